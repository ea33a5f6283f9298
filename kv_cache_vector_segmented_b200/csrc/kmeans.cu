// Segmented k-means index build of the wave index (sm_100a).
//
// Segmented clustering ("KV缓存技术与RetroInfer系统在长上下文推理中的优化实践",
// framerc.cn, §2.1 pseudocode: k-means per 8K-token segment, segments in
// parallel, centroids plus per-cluster value sums) and the cluster-contiguous
// layout (§3.1: the KV vectors of one cluster stored contiguously).
//
// One Lloyd iteration = assignment (tensor cores) + exact fix-up of near ties
// + update (segmented sums).
//
// Assignment: label = argmin_j ||k - mu_j||^2 = argmin_j (||mu_j||^2 - 2 k.mu_j),
// ties to the lower j.  The TMEM accumulator of each (key, centroid) pair
// starts at h_j = -||mu_j||^2 / 2 (fp32, stored by the epilogue) and tcgen05
// MMA adds k . bf16(mu_j) for 128 keys x 256 centroids per instruction group
// (keys are exact in bf16), so w_j = -a_j / 2 and the argmin is the argmax of
// w.  a_j = -2 w_j (exact scaling) differs from the exact criterion by at most
//     eps_j(k) = ||k|| e_j + c_j,
//     e_j = 2 ||mu_j - bf16(mu_j)||  (+ 2^-14 ||mu_j|| for the fp32 accumulation)
//     c_j = 2^-15 (||mu_j||^2 + 1)   (rounding of ||mu_j||^2 and of a_j)
// (Cauchy-Schwarz on the rounding residual; the fp32 accumulation over the
// eight K=16 steps, start value included, stays below 2^-19 (||mu_j||^2 +
// ||k|| ||mu_j||), far inside these terms).  A centroid can be the exact
// argmin only if a_j - eps_j <= min_i (a_i + eps_i); when more than one
// centroid passes, the row is queued and a fix-up kernel decides it exactly
// in fp32.
//
// Update: mu_j = mean of the members (fp32), an empty cluster keeps mu_j; the
// members of a cluster are gathered in position order, so sums are
// deterministic.
#include <float.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace ri {

namespace {

constexpr int kRows = 128;        // keys per tile = MMA M
constexpr int kHalfN = 256;       // centroids per MMA = MMA N
constexpr int kStages = 2;        // key tile ring
constexpr int kEpiWarps = 16;       // assignment epilogue: 4 lane quadrants x 4 column quarters
constexpr int kAssignThreads = 64 + 32 * kEpiWarps;
constexpr int kCand = 8;          // candidate slots per row
constexpr int kUpdateWarps = 2;   // update: one warp per cluster, warps per block (48 per SM)
constexpr int kFinWarps = 2;      // finalise: one warp per cluster, warps per block (24 per SM)
constexpr int kSortThreads = 1024;
constexpr int kGatherRows = 16;   // member rows per cp.async chunk of the update
constexpr int kUpdateSmem = kUpdateWarps * kGatherRows * 128 * 2;  // 8 KB
constexpr int kFinRows = 16;      // member rows (K and V) per cp.async chunk of the finalise
constexpr int kFinSmem = kFinWarps * kFinRows * 512;                // 16 KB
constexpr uint16_t kCandNone = 0xFFFF;
constexpr uint16_t kCandFullScan = 0xFFFE;

// Shared memory of the assignment kernel (from a 1024-byte aligned base).
constexpr uint32_t kSmCent = 0;                                // [2 k-halves][512][128 B]
constexpr uint32_t kCentHalfK = 512 * 128;                     // 64 KB
constexpr uint32_t kSmKeys = 2 * kCentHalfK;                   // 128 KB
constexpr uint32_t kKeyStage = 2 * kRows * 128;                // 32 KB
constexpr uint32_t kNsTileBytes = 512 * 32;                    // [512][16] bf16, plain K-major
constexpr uint32_t kSmNs = kSmKeys + kStages * kKeyStage;      // -||mu_j||^2 / 2 in 3 bf16 parts
constexpr uint32_t kSmOnes = kSmNs + kNsTileBytes;             // [128][16] bf16 (1, 1, 1, 0...)
constexpr uint32_t kSmBar = kSmOnes + kRows * 32;
constexpr int kNumBars = 2 * kStages + 2 + 2 + 2 + 1 + 8;
constexpr uint32_t kSmMisc = kSmBar + kNumBars * 8;
// hand-over from column quarters 0-2 to quarter 3 of a TMEM lane quadrant
constexpr uint32_t kSmXR = (kSmMisc + 64 + 15) / 16 * 16;            // [4][128] f32
constexpr uint32_t kSmXMask = kSmXR + 4 * kRows * 4;                  // [4][4 chunks][128] u32
constexpr uint32_t kSmXSum = kSmXMask + 4 * 4 * kRows * 4;             // [4][128] u32
constexpr uint32_t kAssignSmem = kSmXSum + 4 * kRows * 4 + 1024;       // + alignment
static_assert(kAssignSmem <= 227 * 1024, "assignment kernel shared memory");

// Queue of rows whose label needs an exact decision.
struct FixEntry {
  int32_t row;             // bh * M + position in the middle
  uint16_t cand[kCand];    // candidate cluster ids within the segment
};

struct UnitInfo {
  int bh, s, unit, seg_start, L, Ks, cbase, tile;
};

struct BuildDims {
  int N, M, C, S, seg_len, K_full, L_last, K_last, tiles_full, tiles_last, tiles_bh, m0;
  int total_tiles;
};

__device__ __forceinline__ UnitInfo tile_info(const BuildDims& d, int f) {
  UnitInfo u;
  u.bh = f / d.tiles_bh;
  int rem = f - u.bh * d.tiles_bh;
  int s = rem / d.tiles_full;
  if (s >= d.S - 1) s = d.S - 1;
  u.s = s;
  u.tile = rem - s * d.tiles_full;
  u.unit = u.bh * d.S + s;
  u.seg_start = s * d.seg_len;
  const bool last = s == d.S - 1;
  u.L = last ? d.L_last : d.seg_len;
  u.Ks = last ? d.K_last : d.K_full;
  u.cbase = s * d.K_full;
  return u;
}

__device__ __forceinline__ float col_c(float n) { return 3.0517578125e-05f * (n + 1.f); }

// Entry of centroid j (K half kc) in a unit's [512][16] bf16 tile of
// ||mu||^2 terms, stored in the plain K-major layout of the MMA operand:
// 8-row x 16-byte core matrices, K halves 128 bytes apart, row groups 256.
__device__ __forceinline__ uint4* ns_entry(uint8_t* tile, int j, int kc) {
  return reinterpret_cast<uint4*>(tile + (j >> 3) * 256 + kc * 128 + (j & 7) * 16);
}

// h = -||mu||^2 / 2 as b1 + b2 + b3 (bf16, each the rounded remainder of the
// previous: the subtractions are exact, |h - b1 - b2 - b3| <= 2^-27 |h|),
// packed as the first three K entries.
__device__ __forceinline__ uint4 split3_bf16(float h) {
  const __nv_bfloat16 b1 = __float2bfloat16_rn(h);
  const float r1 = h - __bfloat162float(b1);
  const __nv_bfloat16 b2 = __float2bfloat16_rn(r1);
  const float r2 = r1 - __bfloat162float(b2);
  const __nv_bfloat16 b3 = __float2bfloat16_rn(r2);
  return make_uint4((uint32_t)__bfloat16_as_ushort(b1) | ((uint32_t)__bfloat16_as_ushort(b2) << 16),
                    (uint32_t)__bfloat16_as_ushort(b3), 0u, 0u);
}

// Column constants of one centroid from its fp32 row (lane holds 4 dims):
// the bf16 row (MMA operand) and the entry of -||mu||^2 / 2 in the unit's
// tile.  Returns (e, c) on every lane: e = error coefficient of the bf16
// operand, c = rounding term (see file header).
__device__ __forceinline__ float2 centroid_stats(const float4 m, __nv_bfloat16* bf_row,
                                                 uint8_t* ns_tile, int j, int lane,
                                                 bool write_bf16) {
  const __nv_bfloat162 lo = __floats2bfloat162_rn(m.x, m.y);
  const __nv_bfloat162 hi = __floats2bfloat162_rn(m.z, m.w);
  if (write_bf16) {
    uint2 packed;
    packed.x = *reinterpret_cast<const uint32_t*>(&lo);
    packed.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(bf_row + lane * 4) = packed;
  }
  const float2 l2 = __bfloat1622float2(lo), h2 = __bfloat1622float2(hi);
  const float r0 = m.x - l2.x, r1 = m.y - l2.y, r2 = m.z - h2.x, r3 = m.w - h2.y;
  float sq = m.x * m.x + m.y * m.y + m.z * m.z + m.w * m.w;
  float rr = r0 * r0 + r1 * r1 + r2 * r2 + r3 * r3;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    sq += __shfl_xor_sync(0xffffffffu, sq, off);
    rr += __shfl_xor_sync(0xffffffffu, rr, off);
  }
  if (lane == 0)
    *ns_entry(ns_tile, j, 0) = split3_bf16(-0.5f * sq);
  else if (lane == 1)
    *ns_entry(ns_tile, j, 1) = make_uint4(0u, 0u, 0u, 0u);
  const float e = 2.f * sqrtf(rr) * 1.0001f + 6.1035156e-05f * sqrtf(sq) + 1e-30f;
  return make_float2(e, col_c(sq));
}

// ------------------------------------------------------------- assignment
__global__ void __launch_bounds__(kAssignThreads, 1)
    assign_kernel(const __grid_constant__ CUtensorMap tm_keys,
                  const __grid_constant__ CUtensorMap tm_cent, BuildDims d,
                  const float* __restrict__ knorm, const uint8_t* __restrict__ nsplit,
                  const float* __restrict__ ust, int32_t* __restrict__ labels,
                  FixEntry* __restrict__ queue, int* __restrict__ queue_count, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* cent = sm + kSmCent;
  uint8_t* keys = sm + kSmKeys;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kSmBar);
  uint64_t* full = bars;                       // [kStages] TMA -> MMA
  uint64_t* empty = bars + kStages;            // [kStages] MMA -> TMA
  uint64_t* cent_full = bars + 2 * kStages;    // TMA -> MMA (centroids + ||mu||^2 terms)
  uint64_t* cent_empty = cent_full + 1;        // MMA -> TMA
  uint64_t* tfull = cent_full + 2;             // [2 column halves] MMA -> epilogue
  uint64_t* tempty = tfull + 2;                // [2 column halves] epilogue -> MMA
  uint64_t* drain = tempty + 2;                // MMA drain
  uint64_t* xfull = drain + 1;                 // [4 lane quadrants] quarters 0-2 -> quarter 3
  uint64_t* xempty = xfull + 4;                // [4 lane quadrants] quarter 3 -> quarters 0-2
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kSmMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kSmMisc + 8);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int F = d.total_tiles;
  const int f_begin = (int)((long long)F * blockIdx.x / gridDim.x);
  const int f_end = (int)((long long)F * (blockIdx.x + 1) / gridDim.x);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(cent_full, 1);
    mbar_init(cent_empty, 1);
    for (int h = 0; h < 2; ++h) {
      mbar_init(&tfull[h], 1);
      mbar_init(&tempty[h], kEpiWarps * 32);  // every epilogue warp reads a slice of each half
    }
    mbar_init(drain, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&xfull[i], 3 * 32);
      mbar_init(&xempty[i], 32);
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp >= 2 && warp < 10) {
    // the constant A operand of the extra K step: k' = (1, 1, 1, 0, ..., 0)
    const int e = threadIdx.x - 64;  // 256 threads: (row, K half) pairs
    const int r = e >> 1, kc = e & 1;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (kc == 0) v = make_uint4(0x3F803F80u, 0x00003F80u, 0u, 0u);
    *reinterpret_cast<uint4*>(sm + kSmOnes + (r >> 3) * 256 + kc * 128 + (r & 7) * 16) = v;
    fence_proxy_async_smem();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ----------------------------------------------------------- producer
    tma_prefetch_desc(&tm_keys);
    tma_prefetch_desc(&tm_cent);
    int prev_unit = -1;
    uint32_t ce_phase = 0;
    int it = 0;
    int issued[kStages] = {0, 0};
    int cent_loads = 0;
    for (int f = f_begin; f < f_end; ++f, ++it) {
      if (*abort_flag) break;
      const UnitInfo u = tile_info(d, f);
      if (u.unit != prev_unit) {
        if (prev_unit >= 0) {
          if (!mbar_wait_suspend(cent_empty, ce_phase)) {
            record_status(status, RI_ERR_TIMEOUT);
            *abort_flag = 1;
            break;
          }
          ce_phase ^= 1;
        }
        mbar_arrive_expect_tx(cent_full, 4 * kHalfN * 128 + kNsTileBytes);
        const int crow = u.bh * d.C + u.cbase;
        for (int kh = 0; kh < 2; ++kh)
          for (int h = 0; h < 2; ++h)
            tma_load_2d(cent + kh * kCentHalfK + h * kHalfN * 128, &tm_cent, kh * 64,
                        crow + h * kHalfN, cent_full);
        bulk_load(sm + kSmNs, nsplit + (size_t)u.unit * kNsTileBytes, kNsTileBytes, cent_full);
        ++cent_loads;
        prev_unit = u.unit;
      }
      const int stage = it % kStages;
      if (it >= kStages) {
        if (!mbar_wait_suspend(&empty[stage], (uint32_t)(((it / kStages) - 1) & 1))) {
          record_status(status, RI_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
      }
      mbar_arrive_expect_tx(&full[stage], kKeyStage);
      const int krow = u.bh * d.N + d.m0 + u.seg_start + u.tile * kRows;
      for (int kh = 0; kh < 2; ++kh)
        tma_load_2d(keys + stage * kKeyStage + kh * kRows * 128, &tm_keys, kh * 64, krow,
                    &full[stage]);
      ++issued[stage];
    }
    // wait for every copy this thread started before the block may exit
    for (int st = 0; st < kStages; ++st)
      if (issued[st]) mbar_wait_suspend(&full[st], (uint32_t)((issued[st] - 1) & 1));
    if (cent_loads) mbar_wait_suspend(cent_full, (uint32_t)((cent_loads - 1) & 1));
  } else if (warp == 1 && lane == 0) {
    // ----------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = umma_idesc_bf16_f32(kRows, kHalfN);
    const uint32_t cent_addr = smem_u32(cent);
    const uint32_t keys_addr = smem_u32(keys);
    const uint64_t ones_desc = umma_desc_kmajor_plain(smem_u32(sm + kSmOnes), 128, 256);
    int prev_unit = -1;
    uint32_t cf_phase = 0;
    int it = 0;
    for (int f = f_begin; f < f_end; ++f, ++it) {
      if (*abort_flag) break;
      const UnitInfo u = tile_info(d, f);
      if (u.unit != prev_unit) {
        if (prev_unit >= 0) umma_commit(cent_empty);
        if (!mbar_wait_suspend(cent_full, cf_phase)) {
          record_status(status, RI_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        cf_phase ^= 1;
        prev_unit = u.unit;
      }
      const int stage = it % kStages;
      if (!mbar_wait_suspend(&full[stage], (uint32_t)((it / kStages) & 1))) {
        record_status(status, RI_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      bool ok = true;
      for (int h = 0; h < 2; ++h) {
        // the epilogue has read this half of the previous tile
        if (it > 0 && !mbar_wait_suspend(&tempty[h], (uint32_t)((it - 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t koff = (kk >> 2) * (kRows * 128) + (kk & 3) * 32;
          const uint32_t coff = (kk >> 2) * kCentHalfK + h * (kHalfN * 128) + (kk & 3) * 32;
          const uint64_t adesc = umma_desc_sw128(keys_addr + stage * kKeyStage + koff);
          const uint64_t bdesc = umma_desc_sw128(cent_addr + coff);
          umma_bf16(tmem + h * kHalfN, adesc, bdesc, idesc, kk > 0 ? 1u : 0u);
        }
        // + 1 * (-||mu_j||^2 / 2) as three bf16 parts
        const uint64_t ndesc =
            umma_desc_kmajor_plain(smem_u32(sm + kSmNs) + h * (kHalfN / 8) * 256, 128, 256);
        umma_bf16(tmem + h * kHalfN, ones_desc, ndesc, idesc, 1u);
        umma_commit(&tfull[h]);
      }
      if (!ok) {
        record_status(status, RI_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      umma_commit(&empty[stage]);  // the key stage is free once these MMAs complete
    }
    // every MMA issued by this thread has completed once `drain` flips
    umma_commit(drain);
    mbar_wait_suspend(drain, 0);
  } else if (warp >= 2) {
    // ----------------------------------------------------------- epilogue
    // Warp (lane quadrant q, column slice Qc) reads columns [64 Qc, 64 Qc +
    // 64) of each half (256 columns) of the 32 TMEM lanes of quadrant q once
    // per tile: half 0 first, released to the MMA issuer as soon as all 16
    // warps have read it, so the next tile's MMA into half 0 overlaps the
    // epilogue of half 1.  Per 32-column chunk: its maximum, and the mask of
    // entries within the window of the running maximum R (w_j >= R - delta;
    // a threshold at or below the row's final one keeps every candidate).
    // Masks of chunks whose maximum ends below R_slice - delta are dropped:
    // what remains holds every entry with w_j >= R_slice - delta, and an
    // entry outside that window only in a chunk whose own maximum is a second
    // candidate.  Three slices hand (R, masks) to the fourth (slice
    // tile mod 4), which decides the row: a slice takes part iff its
    // maximum is within delta of the row
    // maximum W (then its entries are candidates, or the row has two or more
    // candidates anyway).  Chunk c of slice Qc covers columns
    // 256 (c >> 1) + 64 Qc + 32 (c & 1).
    const int ew = warp - 2;
    const int Qc = ew >> 2;  // column slice
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int row = q * 32 + lane;
    const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(Qc * 64);
    float* xR = reinterpret_cast<float*>(sm + kSmXR);             // [3][128]
    uint32_t* xm = reinterpret_cast<uint32_t*>(sm + kSmXMask);    // [3][4][128]
    uint32_t* xs = reinterpret_cast<uint32_t*>(sm + kSmXSum);     // [3][128]
    int prev_unit = -1;
    float uE = 0.f, uC = 0.f;
    int it = 0;
    for (int f = f_begin; f < f_end; ++f, ++it) {
      const UnitInfo u = tile_info(d, f);
      if (u.unit != prev_unit) {
        prev_unit = u.unit;
        uE = ust[2 * u.unit];
        uC = ust[2 * u.unit + 1];
      }
      const int t = u.tile * kRows + row;  // token within the segment
      const bool valid = t < u.L;
      const float kn = valid ? knorm[(size_t)u.bh * d.M + u.seg_start + t] : 0.f;
      if (*abort_flag) break;
      // half the window a_j <= min a + 2 (||k|| E + C), in units of w = -a / 2
      const float delta = kn * uE + uC;
      float cm[4];
      uint32_t hit[4];
      float R = -FLT_MAX;
      bool timed_out = false;
#pragma unroll
      for (int cp = 0; cp < 2; ++cp) {  // cp = half of the accumulator
        if (!mbar_wait_suspend(&tfull[cp], (uint32_t)(it & 1))) {
          timed_out = true;
          break;
        }
        tc_fence_after();
        uint32_t r0[32], r1[32];
        tmem_ld32_nowait(taddr + cp * kHalfN, r0);
        tmem_ld32_nowait(taddr + cp * kHalfN + 32, r1);
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&tempty[cp]);  // these columns are free for the next tile
        // both chunk maxima first (independent chains), one threshold
        float m4[4] = {-FLT_MAX, -FLT_MAX, -FLT_MAX, -FLT_MAX};
        float n4[4] = {-FLT_MAX, -FLT_MAX, -FLT_MAX, -FLT_MAX};
#pragma unroll
        for (int i = 0; i < 32; i += 2) {
          const int k = (i >> 1) & 3;
          m4[k] = fmax3f(m4[k], __uint_as_float(r0[i]), __uint_as_float(r0[i + 1]));
          n4[k] = fmax3f(n4[k], __uint_as_float(r1[i]), __uint_as_float(r1[i + 1]));
        }
        cm[2 * cp] = fmax3f(m4[0], m4[1], fmaxf(m4[2], m4[3]));
        cm[2 * cp + 1] = fmax3f(n4[0], n4[1], fmaxf(n4[2], n4[3]));
        R = fmax3f(R, cm[2 * cp], cm[2 * cp + 1]);
        // w_i >= tr iff the sign bit of the rounded difference w_i - tr is
        // clear (rounding keeps the sign; w_i == tr gives +0).  The one
        // exception, -0 - (+0) = -0, is avoided by taking a zero threshold
        // as -0.  A funnel shift moves each sign bit into an accumulator: one
        // integer instruction per entry, the subtraction on the FP32 pipe.
        // Two chains per chunk (entries 15..0 and 31..16, the last one
        // shifted in lands in bit 0).
        const float tr0 = R - delta;
        const float tr = tr0 == 0.f ? -0.f : tr0;
        uint32_t alo = 0u, ahi = 0u, blo = 0u, bhi = 0u;
#pragma unroll
        for (int i = 15; i >= 0; --i) {
          alo = __funnelshift_l(__float_as_uint(__fsub_rn(__uint_as_float(r0[i]), tr)), alo, 1);
          ahi = __funnelshift_l(__float_as_uint(__fsub_rn(__uint_as_float(r0[i + 16]), tr)), ahi, 1);
          blo = __funnelshift_l(__float_as_uint(__fsub_rn(__uint_as_float(r1[i]), tr)), blo, 1);
          bhi = __funnelshift_l(__float_as_uint(__fsub_rn(__uint_as_float(r1[i + 16]), tr)), bhi, 1);
        }
        hit[2 * cp] = ~(alo | (ahi << 16));
        hit[2 * cp + 1] = ~(blo | (bhi << 16));
      }
      if (timed_out) {
        record_status(status, RI_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      const float thr = R - delta;
      // the slice's candidates: how many, and the first in column order
      // (chunk c = 2 h + j of this slice is column chunk 8 h + 2 Qc + j)
      int ncand = 0, first = 512;
#pragma unroll
      for (int c = 3; c >= 0; --c) {
        if (cm[c] < thr) hit[c] = 0u;
        ncand += __popc(hit[c]);
        if (hit[c]) first = (8 * (c >> 1) + 2 * Qc + (c & 1)) * 32 + __ffs(hit[c]) - 1;
      }
      const uint32_t summ = (uint32_t)first | ((uint32_t)ncand << 16);
      // the slice that decides the rows of this quadrant rotates with the
      // tile, so the decision work is shared by the four slices' warps
      const int dq = it & 3;
      if (Qc != dq) {
        if (it >= 1 && !mbar_wait_suspend(&xempty[q], (uint32_t)((it - 1) & 1))) {
          record_status(status, RI_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        xR[Qc * kRows + row] = R;
        xs[Qc * kRows + row] = summ;
#pragma unroll
        for (int c = 0; c < 4; ++c) xm[(Qc * 4 + c) * kRows + row] = hit[c];
        mbar_arrive(&xfull[q]);
        continue;
      }
      if (!mbar_wait_suspend(&xfull[q], (uint32_t)(it & 1))) {
        record_status(status, RI_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      float Rq[4];
      uint32_t sq[4], mq[16];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (k == Qc) {
          Rq[k] = R;
          sq[k] = summ;
#pragma unroll
          for (int c = 0; c < 4; ++c) mq[k * 4 + c] = hit[c];
        } else {
          Rq[k] = xR[k * kRows + row];
          sq[k] = xs[k * kRows + row];
#pragma unroll
          for (int c = 0; c < 4; ++c) mq[k * 4 + c] = xm[(k * 4 + c) * kRows + row];
        }
      }
      mbar_arrive(&xempty[q]);
      if (!valid) continue;
      const float W = fmaxf(fmaxf(Rq[0], Rq[1]), fmaxf(Rq[2], Rq[3]));
      const float wt = W - delta;
      // a slice whose maximum is below W - delta holds no candidate; the
      // others' counts add up and the first candidate is the least first one
      int ntot = 0, lab = 512;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (!(Rq[k] < wt)) {
          ntot += (int)(sq[k] >> 16);
          lab = min(lab, (int)(sq[k] & 0xFFFFu));
        }
      }
      const int grow = u.bh * d.M + u.seg_start + t;
      labels[grow] = lab < 512 ? lab : 0;
      if (ntot != 1) {
        // chunks in column order: column chunk cc = 8 h + 2 Qc + j is chunk
        // 2 h + j of slice Qc
        uint32_t mc[16];
#pragma unroll
        for (int cc = 0; cc < 16; ++cc) {
          const int k = (cc & 7) >> 1, c = ((cc >> 3) << 1) | (cc & 1);
          mc[cc] = Rq[k] < wt ? 0u : mq[k * 4 + c];  // slice without candidates
        }
        // two or more candidates (ids in increasing order): exact fix-up
        FixEntry e;
        e.row = grow;
#pragma unroll
        for (int i = 0; i < kCand; ++i) e.cand[i] = kCandNone;
        if (ntot > kCand || ntot == 0) {
          e.cand[0] = kCandFullScan;
        } else {
          int k = 0;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            uint32_t m = mc[c];
            while (m) {
              const int b = __ffs(m) - 1;
              m &= m - 1u;
              e.cand[k++] = (uint16_t)(c * 32 + b);
            }
          }
        }
        const int qi = atomicAdd(queue_count, 1);
        queue[qi] = e;
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// Exact fp32 decision for the queued rows: one warp per row, lane l holds
// dims 4l..4l+3; distances in the direct difference form, reduced by a xor
// butterfly (identical result on every lane), ties to the lower id.
__global__ void __launch_bounds__(256)
    fixup_kernel(const __nv_bfloat16* __restrict__ K, const float* __restrict__ mu, BuildDims d,
                 const FixEntry* __restrict__ queue, const int* __restrict__ queue_count,
                 int32_t* __restrict__ labels) {
  const int lane = threadIdx.x & 31;
  const int gw = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
  const int nw = (int)((gridDim.x * blockDim.x) >> 5);
  const int n = *queue_count;
  for (int e = gw; e < n; e += nw) {
    const FixEntry en = queue[e];
    const int bh = en.row / d.M;
    const int m = en.row - bh * d.M;
    const int s = m / d.seg_len;
    const int Ks = s == d.S - 1 ? d.K_last : d.K_full;
    const uint2 raw = *reinterpret_cast<const uint2*>(
        K + ((size_t)bh * d.N + d.m0 + m) * kHeadDim + lane * 4);
    const __nv_bfloat162* hk = reinterpret_cast<const __nv_bfloat162*>(&raw);
    const float2 k01 = __bfloat1622float2(hk[0]), k23 = __bfloat1622float2(hk[1]);
    const float* mub = mu + ((size_t)bh * d.C + (size_t)s * d.K_full) * kHeadDim + lane * 4;
    float best = FLT_MAX;
    int bj = 0;
    auto consider = [&](int j) {
      const float4 mm = *reinterpret_cast<const float4*>(mub + (size_t)j * kHeadDim);
      const float t0 = k01.x - mm.x, t1 = k01.y - mm.y, t2 = k23.x - mm.z, t3 = k23.y - mm.w;
      float p = t0 * t0 + t1 * t1 + t2 * t2 + t3 * t3;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) p += __shfl_xor_sync(0xffffffffu, p, off);
      if (p < best || (p == best && j < bj)) {
        best = p;
        bj = j;
      }
    };
    if (en.cand[0] == kCandFullScan) {
      for (int j = 0; j < Ks; ++j) consider(j);
    } else {
#pragma unroll
      for (int i = 0; i < kCand; ++i)
        if (en.cand[i] != kCandNone && en.cand[i] < Ks) consider(en.cand[i]);
    }
    if (lane == 0) labels[en.row] = bj;
  }
}

// ------------------------------------------------------------- prep
// ||k|| of every middle token (four lanes per row, 16-byte loads), rounded
// up so bounds that use it stay upper bounds.
__global__ void knorm_kernel(const __nv_bfloat16* __restrict__ K, float* __restrict__ knorm,
                             int N, int M, int m0, long long rows) {
  const long long r = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 2;
  const int part = threadIdx.x & 3;
  float s = 0.f;
  if (r < rows) {
    const long long bh = r / M, m = r % M;
    const uint4* src = reinterpret_cast<const uint4*>(K + ((size_t)bh * N + m0 + m) * kHeadDim);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float f[8];
      bf16x8_to_float(ldg_nc_v4(src + i * 4 + part), f);
#pragma unroll
      for (int k = 0; k < 8; ++k) s += f[k] * f[k];
    }
  }
  s += __shfl_xor_sync(0xffffffffu, s, 1);
  s += __shfl_xor_sync(0xffffffffu, s, 2);
  if (r < rows && part == 0) knorm[r] = sqrtf(s) * 1.0001f;
}

// Seeds: mu_j = k at the given (or strided) position of the segment.  One
// warp per (bh, s, j in [0, 512)); j >= K_s only pads the column table.
__global__ void init_kernel(const __nv_bfloat16* __restrict__ K,
                            const int32_t* __restrict__ init_pos, BuildDims d,
                            float* __restrict__ mu, __nv_bfloat16* __restrict__ mu_bf16,
                            uint8_t* __restrict__ nsplit, float2* __restrict__ ecs, int* status,
                            long long total) {
  // blocks of 8 warps: kMaxClustersPerSeg is a multiple of 8, so a block's
  // warps share one unit and `total` fills whole blocks
  const long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  const int unit = (int)(w / kMaxClustersPerSeg);
  const int j = (int)(w % kMaxClustersPerSeg);
  const int bh = unit / d.S, s = unit % d.S;
  const bool last = s == d.S - 1;
  const int L = last ? d.L_last : d.seg_len;
  const int Ks = last ? d.K_last : d.K_full;
  uint8_t* ns = nsplit + (size_t)unit * kNsTileBytes;
  if (w < total && j >= Ks) {
    // padding column: w_j = -inf, never a candidate
    if (lane < 2)
      *ns_entry(ns, j, lane) =
          lane == 0 ? make_uint4(0xFF80u, 0u, 0u, 0u) : make_uint4(0u, 0u, 0u, 0u);
  } else if (w < total) {
    const int c = s * d.K_full + j;
    int p;
    if (init_pos) {
      p = init_pos[(size_t)bh * d.C + c];
      if (p < 0 || p >= L) {
        if (lane == 0) record_status(status, RI_ERR_INVALID_ARG);
        p = p < 0 ? 0 : L - 1;
      }
    } else {
      p = (int)(((long long)j * L) / Ks);
    }
    const __nv_bfloat16* src =
        K + ((size_t)bh * d.N + d.m0 + (size_t)s * d.seg_len + p) * kHeadDim + lane * 4;
    const uint2 raw = *reinterpret_cast<const uint2*>(src);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
    const float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
    const float4 m = make_float4(a.x, a.y, b.x, b.y);
    *reinterpret_cast<float4*>(mu + ((size_t)bh * d.C + c) * kHeadDim + lane * 4) = m;
    const float2 ec =
        centroid_stats(m, mu_bf16 + ((size_t)bh * d.C + c) * kHeadDim, ns, j, lane, true);
    if (lane == 0) ecs[w] = ec;
  }
}

// Per unit: E = max e_j, Cmax = max c_j over its K_s centroids (one warp per
// unit, from the per-centroid values the update wrote).
__global__ void unit_max_kernel(const float2* __restrict__ ecs, BuildDims d,
                                float* __restrict__ ust, int units) {
  const int unit = (int)(blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5));
  const int lane = threadIdx.x & 31;
  if (unit >= units) return;
  const int Ks = unit % d.S == d.S - 1 ? d.K_last : d.K_full;
  float2 r = make_float2(0.f, 0.f);
  for (int j = lane; j < Ks; j += 32) {
    const float2 v = ecs[(size_t)unit * kMaxClustersPerSeg + j];
    r.x = fmaxf(r.x, v.x);
    r.y = fmaxf(r.y, v.y);
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    r.x = fmaxf(r.x, __shfl_xor_sync(0xffffffffu, r.x, off));
    r.y = fmaxf(r.y, __shfl_xor_sync(0xffffffffu, r.y, off));
  }
  if (lane == 0) {
    ust[2 * unit] = r.x;
    ust[2 * unit + 1] = r.y;
  }
}

// ------------------------------------------------------------- update / finalise
// Stable counting sort of one segment's positions by label (one block of
// kSortThreads per unit): members[unit rows] lists the positions of cluster 0,
// then cluster 1, ..., each cluster's in increasing position; mstart[unit][j]
// is the first entry of cluster j (mstart[unit][512] = L).  Warp w owns
// positions [w P, w P + P): per-warp histograms, a column scan over warps,
// then each warp places its positions in order (ranks among equal labels of
// one 32-position step by match_any).
// Block 0 also zeroes the fix-up queue count of the next assignment pass
// (the fix-up that read it ran before this kernel).
// Shared memory: lab[L] u16, cnt[32][512] i32, tot scan scratch.
__global__ void __launch_bounds__(kSortThreads)
    sort_kernel(const int32_t* __restrict__ labels, BuildDims d, int32_t* __restrict__ members,
                int32_t* __restrict__ mstart, int* __restrict__ queue_count) {
  extern __shared__ __align__(16) uint8_t smem_s[];
  constexpr int NW = kSortThreads / 32;
  int* cnt = reinterpret_cast<int*>(smem_s);                                  // [NW][512]
  int* cstart = cnt + NW * kMaxClustersPerSeg;                                // [513]
  int* wsum = cstart + kMaxClustersPerSeg + 1;                                // [NW]
  uint16_t* lab = reinterpret_cast<uint16_t*>(wsum + NW);                     // [L]
  const int unit = blockIdx.x;
  const int bh = unit / d.S, s = unit % d.S;
  const bool last = s == d.S - 1;
  const int L = last ? d.L_last : d.seg_len;
  const int seg_start = s * d.seg_len;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int32_t* src = labels + (size_t)bh * d.M + seg_start;
  if (unit == 0 && threadIdx.x == 0) *queue_count = 0;  // for the next assignment pass
  for (int i = threadIdx.x; i < NW * kMaxClustersPerSeg; i += kSortThreads) cnt[i] = 0;
  for (int i = threadIdx.x; i < L; i += kSortThreads) lab[i] = (uint16_t)src[i];
  __syncthreads();
  const int P = ((L + NW - 1) / NW + 31) & ~31;  // positions per warp, whole steps
  const int p0 = warp * P, p1 = min(L, p0 + P);
  int* mycnt = cnt + warp * kMaxClustersPerSeg;
  for (int p = p0 + lane; p < p1; p += 32) atomicAdd(&mycnt[lab[p]], 1);
  __syncthreads();
  // column scan: cnt[w][c] <- first slot of warp w's members of cluster c
  int run = 0;
  const int c = threadIdx.x;
  if (c < kMaxClustersPerSeg) {
    for (int w = 0; w < NW; ++w) {
      const int v = cnt[w * kMaxClustersPerSeg + c];
      cnt[w * kMaxClustersPerSeg + c] = run;
      run += v;
    }
  }
  // exclusive scan of the cluster totals (run) over c: warp sums, then offsets
  int incl = run;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (c < kMaxClustersPerSeg) {
    int before = 0;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    const int first = before + incl - run;
    cstart[c] = first;
    for (int w = 0; w < NW; ++w) cnt[w * kMaxClustersPerSeg + c] += first;
  }
  if (c == 0) cstart[kMaxClustersPerSeg] = L;
  __syncthreads();
  // placement in position order
  int32_t* out = members + (size_t)bh * d.M + seg_start;
  const unsigned lt = (1u << lane) - 1u;
  for (int base = p0; base < p1; base += 32) {
    const int p = base + lane;
    const bool in = p < p1;
    const int cl = in ? (int)lab[p] : -1 - lane;  // out-of-range lanes match nobody
    const unsigned grp = __match_any_sync(0xffffffffu, cl);
    if (in) {
      const int slot = mycnt[cl] + __popc(grp & lt);
      out[slot] = p;
    }
    __syncwarp();
    if (in && (grp & lt) == 0) mycnt[cl] += __popc(grp);
    __syncwarp();
  }
  int32_t* ms = mstart + (size_t)unit * (kMaxClustersPerSeg + 1);
  for (int i = threadIdx.x; i <= kMaxClustersPerSeg; i += kSortThreads) ms[i] = cstart[i];
}

// One warp per cluster: mu_j = mean of the members (fp32, summed in position
// order; an empty cluster keeps mu_j), the column constants of the new
// centroid and the cluster size.  Members are fetched 16 rows at a time with
// 16-byte cp.async copies into the warp's 4 KB of shared memory (the
// transfers need no registers, so a warp keeps a whole chunk in flight).
// Blocks of two warps: a block holds its shared memory until its slower
// warp is done, so small blocks keep a large cluster from idling many warps.
__global__ void __launch_bounds__(kUpdateWarps * 32, 48 / kUpdateWarps)
    update_kernel(const __nv_bfloat16* __restrict__ K, const int32_t* __restrict__ members,
                  const int32_t* __restrict__ mstart, BuildDims d, float* __restrict__ mu,
                  __nv_bfloat16* __restrict__ mu_bf16, uint8_t* __restrict__ nsplit,
                  float2* __restrict__ ecs, int32_t* __restrict__ counts, int update_mu) {
  extern __shared__ __align__(16) uint8_t smem_g[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int unit = blockIdx.x, j = blockIdx.y * kUpdateWarps + warp;
  const int bh = unit / d.S, s = unit % d.S;
  const int Ks = s == d.S - 1 ? d.K_last : d.K_full;
  if (j >= Ks) return;
  uint8_t* wb = smem_g + (size_t)warp * kGatherRows * kHeadDim * 2;  // [16 rows][256 B]
  const int seg_start = s * d.seg_len;
  const int32_t* ms = mstart + (size_t)unit * (kMaxClustersPerSeg + 1);
  const int b = ms[j], e = ms[j + 1];
  const int32_t* mem = members + (size_t)bh * d.M + seg_start;
  const __nv_bfloat16* kseg = K + ((size_t)bh * d.N + d.m0 + seg_start) * kHeadDim;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int i = b; i < e; i += kGatherRows) {
    const int nb = min(kGatherRows, e - i);
    const int pos = lane < nb ? mem[i + lane] : 0;  // the chunk's member positions, one load
    // row r = 2 k + (lane >> 4), 16-byte chunk lane & 15
#pragma unroll
    for (int k = 0; k < kGatherRows / 2; ++k) {
      const int r = 2 * k + (lane >> 4);
      const int p = __shfl_sync(0xffffffffu, pos, r);
      if (r < nb)
        cp_async16(wb + r * (kHeadDim * 2) + (lane & 15) * 16,
                   kseg + (size_t)p * kHeadDim + (lane & 15) * 8);
    }
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();
    for (int r = 0; r < nb; ++r) {
      const uint2 raw = *reinterpret_cast<const uint2*>(wb + r * (kHeadDim * 2) + lane * 8);
      const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
      const float2 a = __bfloat1622float2(h[0]), bb = __bfloat1622float2(h[1]);
      acc[0] += a.x;
      acc[1] += a.y;
      acc[2] += bb.x;
      acc[3] += bb.y;
    }
    __syncwarp();  // the buffer is refilled by the next chunk
  }
  const size_t row = (size_t)bh * d.C + (size_t)s * d.K_full + j;
  uint8_t* ns = nsplit + (size_t)unit * kNsTileBytes;
  const int n = e - b;
  float2 ec;
  if (update_mu && n > 0) {
    const float fn = (float)n;
    const float4 m = make_float4(acc[0] / fn, acc[1] / fn, acc[2] / fn, acc[3] / fn);
    *reinterpret_cast<float4*>(mu + row * kHeadDim + lane * 4) = m;
    ec = centroid_stats(m, mu_bf16 + row * kHeadDim, ns, j, lane, true);
  } else {
    const float4 m = *reinterpret_cast<const float4*>(mu + row * kHeadDim + lane * 4);
    ec = centroid_stats(m, mu_bf16 + row * kHeadDim, ns, j, lane, false);
  }
  if (lane == 0) {
    counts[row] = n;
    ecs[(size_t)unit * kMaxClustersPerSeg + j] = ec;
  }
}

// Cluster-contiguous layout of the final labels (members / mstart from the
// last sort): one warp per cluster copies its members' K and V rows in
// (cluster, position) order, with the permutation, offsets, sizes, value
// sums, the bf16 centroid and the members' squared distances.
__global__ void __launch_bounds__(kFinWarps * 32, 24 / kFinWarps)
    finalise_kernel(const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V,
                    const int32_t* __restrict__ labels, const int32_t* __restrict__ members,
                    const int32_t* __restrict__ mstart, BuildDims d,
                    const float* __restrict__ mu, ri_index out) {
  extern __shared__ __align__(16) uint8_t smem_f[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  {
    const int unit = blockIdx.x, j = blockIdx.y * kFinWarps + warp;
    const int bh = unit / d.S, s = unit % d.S;
    const int Ks = s == d.S - 1 ? d.K_last : d.K_full;
    const int L = s == d.S - 1 ? d.L_last : d.seg_len;
    if (out.labels)  // the unit's blocks share the copy of its labels
      for (int t = blockIdx.y * blockDim.x + threadIdx.x; t < L; t += gridDim.y * blockDim.x)
        out.labels[(size_t)bh * d.M + s * d.seg_len + t] =
            labels[(size_t)bh * d.M + s * d.seg_len + t];
    if (blockIdx.y == 0 && s == d.S - 1 && threadIdx.x == 0)
      out.offsets[(size_t)bh * (d.C + 1) + d.C] = d.M;
    if (j >= Ks) return;
    const int seg_start = s * d.seg_len;
    const int32_t* ms = mstart + (size_t)unit * (kMaxClustersPerSeg + 1);
    const int b = ms[j], e = ms[j + 1];
    const int32_t* mem = members + (size_t)bh * d.M + seg_start;
    const size_t bhN = (size_t)bh * d.N + d.m0 + seg_start;
    const size_t bhM = (size_t)bh * d.M + seg_start;
    const size_t crow = (size_t)bh * d.C + (size_t)s * d.K_full + j;
    // lane l < 16 moves 16-byte chunk l of each member's K row, lane 16 + l
    // chunk l of its V row: 16 rows per cp.async chunk through the warp's 8 KB
    uint8_t* wb = smem_f + (size_t)warp * kFinRows * 512;  // [16 rows][K 256 B | V 256 B]
    const int ch = lane & 15;
    const bool is_v = lane >= 16;
    float mk[8];  // this lane's 8 centroid dims (K lanes)
    {
      const float4 m0v = *reinterpret_cast<const float4*>(mu + crow * kHeadDim + ch * 8);
      const float4 m1v = *reinterpret_cast<const float4*>(mu + crow * kHeadDim + ch * 8 + 4);
      mk[0] = m0v.x; mk[1] = m0v.y; mk[2] = m0v.z; mk[3] = m0v.w;
      mk[4] = m1v.x; mk[5] = m1v.y; mk[6] = m1v.z; mk[7] = m1v.w;
    }
    float acc8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // V sums (V lanes)
    float obj = 0.f;                                           // squared distances (K lanes)
    const __nv_bfloat16* src_base = (is_v ? V : K) + bhN * kHeadDim + ch * 8;
    __nv_bfloat16* dst_base = static_cast<__nv_bfloat16*>(is_v ? out.Vp : out.Kp) + ch * 8;
    for (int i = b; i < e; i += kFinRows) {
      const int nb = min(kFinRows, e - i);
      const int pos = lane < nb ? mem[i + lane] : 0;
      if (lane < nb) out.perm[bhM + i + lane] = d.m0 + seg_start + pos;
#pragma unroll
      for (int r = 0; r < kFinRows; ++r) {
        const int pr = __shfl_sync(0xffffffffu, pos, r);
        if (r < nb) cp_async16(wb + r * 512 + lane * 16, src_base + (size_t)pr * kHeadDim);
      }
      cp_async_commit();
      cp_async_wait<0>();
      __syncwarp();
      for (int r = 0; r < nb; ++r) {
        const uint4 raw = *reinterpret_cast<const uint4*>(wb + r * 512 + lane * 16);
        *reinterpret_cast<uint4*>(dst_base + (bhM + i + r) * kHeadDim) = raw;  // (cluster, position) order
        float f[8];
        bf16x8_to_float(raw, f);
        if (is_v) {
#pragma unroll
          for (int k = 0; k < 8; ++k) acc8[k] += f[k];
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const float dd = f[k] - mk[k];
            obj = fmaf(dd, dd, obj);
          }
        }
      }
      __syncwarp();  // the buffer is refilled by the next chunk
    }
    if (is_v) {
      float4* vdst = reinterpret_cast<float4*>(out.vsum + crow * kHeadDim + ch * 8);
      vdst[0] = make_float4(acc8[0], acc8[1], acc8[2], acc8[3]);
      vdst[1] = make_float4(acc8[4], acc8[5], acc8[6], acc8[7]);
    }
    const float4 m = *reinterpret_cast<const float4*>(mu + crow * kHeadDim + lane * 4);
    const __nv_bfloat162 lo = __floats2bfloat162_rn(m.x, m.y);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(m.z, m.w);
    uint2 packed;
    packed.x = *reinterpret_cast<const uint32_t*>(&lo);
    packed.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out.centroid) + crow * kHeadDim +
                              lane * 4) = packed;
    if (lane == 0) {
      out.counts[crow] = e - b;
      out.offsets[(size_t)bh * (d.C + 1) + (size_t)s * d.K_full + j] = seg_start + b;
    }
    if (out.objective) {
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) obj += __shfl_xor_sync(0xffffffffu, obj, off);
      if (lane == 0) atomicAdd(&out.objective[unit], obj);
    }
  }
}

// Steady-zone buffers: tokens [0, s0) and [N - s1, N) (all tokens if N <= s0 + s1).
__global__ void steady_kernel(const __nv_bfloat16* __restrict__ K,
                              const __nv_bfloat16* __restrict__ V, __nv_bfloat16* __restrict__ Ks,
                              __nv_bfloat16* __restrict__ Vs, int N, int s0, int s1,
                              int n_steady) {
  const int bh = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int t = warp; t < n_steady; t += blockDim.x >> 5) {
    const int pos = (N <= s0 + s1 || t < s0) ? t : N - s1 + (t - s0);
    const size_t src = ((size_t)bh * N + pos) * kHeadDim + lane * 4;
    const size_t dst = ((size_t)bh * n_steady + t) * kHeadDim + lane * 4;
    *reinterpret_cast<uint2*>(Ks + dst) = *reinterpret_cast<const uint2*>(K + src);
    *reinterpret_cast<uint2*>(Vs + dst) = *reinterpret_cast<const uint2*>(V + src);
  }
}

// ------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 map over [rows][128] with boxes of box_rows x 64 (128-byte swizzle).
bool make_map_bf16(CUtensorMap* map, const void* base, unsigned long long rows, int box_rows) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace

#define RI_CUDA_TRY(expr)                                      \
  do {                                                         \
    cudaError_t e_ = (expr);                                   \
    if (e_ != cudaSuccess) {                                   \
      set_error("%s: %s", #expr, cudaGetErrorString(e_));      \
      return RI_ERR_CUDA;                                      \
    }                                                          \
  } while (0)

size_t build_queue_bytes(long long rows) { return (size_t)rows * sizeof(FixEntry); }

ri_status launch_build(const Geometry& g, const BuildLayout& L, const BuildArgs& a,
                       cudaStream_t st) {
  char* ws = a.ws;
  int* status = reinterpret_cast<int*>(ws);
  int* queue_count = reinterpret_cast<int*>(ws + 64);
  const __nv_bfloat16* K = static_cast<const __nv_bfloat16*>(a.K);
  const __nv_bfloat16* V = static_cast<const __nv_bfloat16*>(a.V);
  const long long BH = g.BH();
  if (g.n_steady > 0)
    steady_kernel<<<(unsigned)BH, 256, 0, st>>>(K, V, static_cast<__nv_bfloat16*>(a.out.Ks),
                                                static_cast<__nv_bfloat16*>(a.out.Vs), g.N, g.s0,
                                                g.s1, g.n_steady);
  RI_CUDA_TRY(cudaGetLastError());
  if (g.M == 0) {
    RI_CUDA_TRY(cudaMemsetAsync(a.out.offsets, 0, BH * sizeof(int32_t), st));
    return RI_OK;
  }
  BuildDims d;
  d.N = g.N; d.M = g.M; d.C = g.C; d.S = g.S; d.seg_len = g.seg_len; d.K_full = g.K_full;
  d.L_last = g.L_last; d.K_last = g.K_last; d.tiles_full = g.tiles_full;
  d.tiles_last = g.tiles_last; d.tiles_bh = g.tiles_bh; d.m0 = g.m0;
  if (BH * g.tiles_bh > 0x7fffffffLL) {
    set_error("too many key tiles (%lld)", BH * g.tiles_bh);
    return RI_ERR_UNSUPPORTED;
  }
  d.total_tiles = (int)(BH * g.tiles_bh);
  float* mu = reinterpret_cast<float*>(ws + L.off_mu);
  __nv_bfloat16* mu_bf16 = reinterpret_cast<__nv_bfloat16*>(ws + L.off_mu_bf16);
  uint8_t* nsplit = reinterpret_cast<uint8_t*>(ws + L.off_nsplit);
  float* ust = reinterpret_cast<float*>(ws + L.off_ust);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + L.off_counts);
  int32_t* labels = reinterpret_cast<int32_t*>(ws + L.off_labels);
  float* knorm = reinterpret_cast<float*>(ws + L.off_knorm);
  FixEntry* queue = reinterpret_cast<FixEntry*>(ws + L.off_queue);
  int32_t* members = reinterpret_cast<int32_t*>(ws + L.off_members);
  int32_t* mstart = reinterpret_cast<int32_t*>(ws + L.off_mstart);
  float2* ecs = reinterpret_cast<float2*>(ws + L.off_ecs);
  const long long units = BH * g.S;

  CUtensorMap tm_keys, tm_cent;
  if (!make_map_bf16(&tm_keys, a.K, (unsigned long long)BH * g.N, kRows) ||
      !make_map_bf16(&tm_cent, mu_bf16, (unsigned long long)BH * g.C, kHalfN)) {
    set_error("cuTensorMapEncodeTiled failed");
    return RI_ERR_CUDA;
  }
  const long long rows = BH * g.M;
  knorm_kernel<<<(unsigned)((rows + 63) / 64), 256, 0, st>>>(K, knorm, g.N, g.M, g.m0, rows);
  RI_CUDA_TRY(cudaGetLastError());
  const long long init_total = units * kMaxClustersPerSeg;
  init_kernel<<<(unsigned)((init_total + 7) / 8), 256, 0, st>>>(K, a.init_pos, d, mu, mu_bf16,
                                                                 nsplit, ecs, status, init_total);
  RI_CUDA_TRY(cudaGetLastError());
  unit_max_kernel<<<(unsigned)((units + 7) / 8), 256, 0, st>>>(ecs, d, ust, (int)units);
  RI_CUDA_TRY(cudaGetLastError());

  RI_CUDA_TRY(set_smem_once(0, reinterpret_cast<const void*>(assign_kernel), (int)kAssignSmem));
  auto sort_smem = [](int L) {
    constexpr int NW = kSortThreads / 32;
    return (size_t)(NW * kMaxClustersPerSeg + kMaxClustersPerSeg + 1 + NW) * sizeof(int) +
           (size_t)L * sizeof(uint16_t);
  };
  RI_CUDA_TRY(set_smem_once(1, reinterpret_cast<const void*>(sort_kernel),
                            (int)sort_smem(kMaxSegLen)));
  RI_CUDA_TRY(set_smem_once(2, reinterpret_cast<const void*>(update_kernel), kUpdateSmem));
  RI_CUDA_TRY(set_smem_once(3, reinterpret_cast<const void*>(finalise_kernel), kFinSmem));
  const int sms = num_sms();
  const unsigned grid_assign = (unsigned)(d.total_tiles < sms ? d.total_tiles : sms);
  const dim3 grid_upd((unsigned)units, (unsigned)(kMaxClustersPerSeg / kUpdateWarps));
  const dim3 grid_fin((unsigned)units, (unsigned)(kMaxClustersPerSeg / kFinWarps));
  const int rounds = g.iters > 0 ? g.iters : 1;
  RI_CUDA_TRY(cudaMemsetAsync(queue_count, 0, sizeof(int), st));  // later passes: the sort
  for (int t = 0; t < rounds; ++t) {
    assign_kernel<<<grid_assign, kAssignThreads, kAssignSmem, st>>>(
        tm_keys, tm_cent, d, knorm, nsplit, ust, labels, queue, queue_count, status);
    RI_CUDA_TRY(cudaGetLastError());
    fixup_kernel<<<(unsigned)(4 * sms), 256, 0, st>>>(K, mu, d, queue, queue_count, labels);
    RI_CUDA_TRY(cudaGetLastError());
    sort_kernel<<<(unsigned)units, kSortThreads, sort_smem(g.seg_len), st>>>(
        labels, d, members, mstart, queue_count);
    RI_CUDA_TRY(cudaGetLastError());
    update_kernel<<<grid_upd, kUpdateWarps * 32, kUpdateSmem, st>>>(
        K, members, mstart, d, mu, mu_bf16, nsplit, ecs, counts, g.iters > 0 ? 1 : 0);
    RI_CUDA_TRY(cudaGetLastError());
    unit_max_kernel<<<(unsigned)((units + 7) / 8), 256, 0, st>>>(ecs, d, ust, (int)units);
    RI_CUDA_TRY(cudaGetLastError());
  }
  if (a.out.objective)
    RI_CUDA_TRY(cudaMemsetAsync(a.out.objective, 0, units * sizeof(float), st));
  finalise_kernel<<<grid_fin, kFinWarps * 32, kFinSmem, st>>>(K, V, labels, members, mstart,
                                                                 d, mu, a.out);
  RI_CUDA_TRY(cudaGetLastError());
  return RI_OK;
}

}  // namespace ri
