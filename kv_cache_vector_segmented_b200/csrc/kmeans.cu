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
// ties to the lower j.  tcgen05 MMA computes v_j = k . bf16(mu_j) for 128 keys x
// 256 centroids per instruction group (keys are exact in bf16; fp32
// accumulators in TMEM).  a_j = ||mu_j||^2 - 2 v_j then differs from the exact
// criterion by at most
//     eps_j(k) = ||k|| e_j + c_j,
//     e_j = 2 ||mu_j - bf16(mu_j)||  (+ 2^-14 ||mu_j|| for the fp32 accumulation)
//     c_j = 2^-15 (||mu_j||^2 + 1)   (rounding of ||mu_j||^2 and of a_j)
// (Cauchy-Schwarz on the rounding residual; n * 2^-23 accumulation bounds with
// a factor-2 margin).  A centroid can be the exact argmin only if
// a_j - eps_j <= min_i (a_i + eps_i); when more than one centroid passes, the
// row is queued and a fix-up kernel decides it exactly in fp32.
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
constexpr int kAssignThreads = 192;
constexpr int kCand = 8;          // candidate slots per row
constexpr int kUpdateWarps = 8;
constexpr int kClustersPerWarp = 4;
constexpr int kClustersPerBlock = kUpdateWarps * kClustersPerWarp;  // 32
constexpr uint16_t kCandNone = 0xFFFF;
constexpr uint16_t kCandFullScan = 0xFFFE;

// Shared memory of the assignment kernel (from a 1024-byte aligned base).
constexpr uint32_t kSmCent = 0;                                // [2 k-halves][512][128 B]
constexpr uint32_t kCentHalfK = 512 * 128;                     // 64 KB
constexpr uint32_t kSmKeys = 2 * kCentHalfK;                   // 128 KB
constexpr uint32_t kKeyStage = 2 * kRows * 128;                // 32 KB
constexpr uint32_t kSmCol = kSmKeys + kStages * kKeyStage;     // [2 buf][2][512] fp32
constexpr uint32_t kColBytes = 2 * 512 * 4;                    // n_j then e_j
constexpr uint32_t kSmBar = kSmCol + 2 * kColBytes;
constexpr int kNumBars = 2 * kStages + 2 + 2 + 2 + 2 + 2 + 1;
constexpr uint32_t kSmMisc = kSmBar + kNumBars * 8;
constexpr uint32_t kAssignSmem = kSmMisc + 64 + 1024;          // + alignment slack

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
  long long total_tiles;
};

__device__ __forceinline__ UnitInfo tile_info(const BuildDims& d, long long f) {
  UnitInfo u;
  u.bh = (int)(f / d.tiles_bh);
  int rem = (int)(f - (long long)u.bh * d.tiles_bh);
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

__device__ __forceinline__ void atomic_max_pos(float* addr, float v) {
  atomicMax(reinterpret_cast<int*>(addr), __float_as_int(v));  // v >= 0
}

// Column constants of one centroid from its fp32 row (lane holds 4 dims):
// n = ||mu||^2, e = error coefficient of the bf16 operand (see file header).
// Writes the packed bf16 row and the table entries; lane 0 raises the unit's
// maxima (E, Cmax).
__device__ __forceinline__ void centroid_stats(const float4 m, __nv_bfloat16* bf_row,
                                               float* col_n, float* col_e, float* ust_unit,
                                               int lane, bool write_bf16) {
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
  if (lane == 0) {
    const float e = 2.f * sqrtf(rr) * 1.0001f + 6.1035156e-05f * sqrtf(sq) + 1e-30f;
    *col_n = sq;
    *col_e = e;
    atomic_max_pos(&ust_unit[0], e);
    atomic_max_pos(&ust_unit[1], col_c(sq));
  }
}

// ------------------------------------------------------------- assignment
__global__ void __launch_bounds__(kAssignThreads, 1)
    assign_kernel(const __grid_constant__ CUtensorMap tm_keys,
                  const __grid_constant__ CUtensorMap tm_cent, BuildDims d,
                  const float* __restrict__ knorm, const float* __restrict__ colt,
                  const float* __restrict__ ust, int32_t* __restrict__ labels,
                  FixEntry* __restrict__ queue, int* __restrict__ queue_count, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* cent = sm + kSmCent;
  uint8_t* keys = sm + kSmKeys;
  float* colsm = reinterpret_cast<float*>(sm + kSmCol);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kSmBar);
  uint64_t* full = bars;                       // [kStages] TMA -> MMA
  uint64_t* empty = bars + kStages;            // [kStages] epilogue -> TMA
  uint64_t* cent_full = bars + 2 * kStages;    // TMA -> MMA
  uint64_t* cent_empty = cent_full + 1;        // MMA -> TMA
  uint64_t* tfull = cent_full + 2;             // [2] MMA -> epilogue
  uint64_t* tempty = tfull + 2;                // [2] epilogue -> MMA
  uint64_t* nfull = tempty + 2;                // [2] TMA -> epilogue (column table)
  uint64_t* nempty = nfull + 2;                // [2] epilogue -> TMA
  uint64_t* drain = nempty + 2;                // MMA drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + kSmMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + kSmMisc + 8);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const long long F = d.total_tiles;
  const long long f_begin = F * blockIdx.x / gridDim.x;
  const long long f_end = F * (blockIdx.x + 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 128);
    }
    mbar_init(cent_full, 1);
    mbar_init(cent_empty, 1);
    for (int h = 0; h < 2; ++h) {
      mbar_init(&tfull[h], 1);
      mbar_init(&tempty[h], 128);
      mbar_init(&nfull[h], 1);
      mbar_init(&nempty[h], 128);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
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
    int prev_unit = -1, nunits = 0;
    uint32_t ce_phase = 0;
    long long it = 0;
    int issued[kStages] = {0, 0};
    int cent_loads = 0, col_loads[2] = {0, 0};
    for (long long f = f_begin; f < f_end; ++f, ++it) {
      if (*abort_flag) break;
      const UnitInfo u = tile_info(d, f);
      if (u.unit != prev_unit) {
        if (prev_unit >= 0) {
          if (!mbar_wait(cent_empty, ce_phase)) {
            record_status(status, RI_ERR_TIMEOUT);
            *abort_flag = 1;
            break;
          }
          ce_phase ^= 1;
        }
        mbar_arrive_expect_tx(cent_full, 4 * kHalfN * 128);
        const int crow = u.bh * d.C + u.cbase;
        for (int kh = 0; kh < 2; ++kh)
          for (int h = 0; h < 2; ++h)
            tma_load_2d(cent + kh * kCentHalfK + h * kHalfN * 128, &tm_cent, kh * 64,
                        crow + h * kHalfN, cent_full);
        ++cent_loads;
        const int nb = nunits & 1;
        if (nunits >= 2) {
          if (!mbar_wait(&nempty[nb], ((nunits >> 1) - 1) & 1)) {
            record_status(status, RI_ERR_TIMEOUT);
            *abort_flag = 1;
            break;
          }
        }
        mbar_arrive_expect_tx(&nfull[nb], kColBytes);
        bulk_load(colsm + nb * 1024, colt + (size_t)u.unit * 1024, kColBytes, &nfull[nb]);
        ++col_loads[nb];
        ++nunits;
        prev_unit = u.unit;
      }
      const int stage = (int)(it % kStages);
      if (it >= kStages) {
        if (!mbar_wait(&empty[stage], (uint32_t)(((it / kStages) - 1) & 1))) {
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
      if (issued[st]) mbar_wait(&full[st], (uint32_t)((issued[st] - 1) & 1));
    if (cent_loads) mbar_wait(cent_full, (uint32_t)((cent_loads - 1) & 1));
    for (int nb = 0; nb < 2; ++nb)
      if (col_loads[nb]) mbar_wait(&nfull[nb], (uint32_t)((col_loads[nb] - 1) & 1));
  } else if (warp == 1 && lane == 0) {
    // ----------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc = umma_idesc_bf16_f32(kRows, kHalfN);
    const uint32_t cent_addr = smem_u32(cent);
    const uint32_t keys_addr = smem_u32(keys);
    int prev_unit = -1;
    uint32_t cf_phase = 0;
    long long it = 0;
    for (long long f = f_begin; f < f_end; ++f, ++it) {
      if (*abort_flag) break;
      const UnitInfo u = tile_info(d, f);
      if (u.unit != prev_unit) {
        if (prev_unit >= 0) umma_commit(cent_empty);
        if (!mbar_wait(cent_full, cf_phase)) {
          record_status(status, RI_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        cf_phase ^= 1;
        prev_unit = u.unit;
      }
      const int stage = (int)(it % kStages);
      if (!mbar_wait(&full[stage], (uint32_t)((it / kStages) & 1))) {
        record_status(status, RI_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      tc_fence_after();
      bool ok = true;
      for (int h = 0; h < 2; ++h) {
        if (it > 0 && !mbar_wait(&tempty[h], (uint32_t)((it - 1) & 1))) {
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
        umma_commit(&tfull[h]);
      }
      if (!ok) {
        record_status(status, RI_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
    }
    // every MMA issued by this thread has completed once `drain` flips
    umma_commit(drain);
    mbar_wait(drain, 0);
  } else if (warp >= 2) {
    // ----------------------------------------------------------- epilogue
    const int quad = warp & 3;  // TMEM lane quadrant this warp may access
    const int row = quad * 32 + lane;
    int prev_unit = -1, nunits = 0;
    float uE = 0.f, uC = 0.f;
    long long it = 0;
    for (long long f = f_begin; f < f_end; ++f, ++it) {
      if (*abort_flag) break;
      const UnitInfo u = tile_info(d, f);
      if (u.unit != prev_unit) {
        if (prev_unit >= 0) mbar_arrive(&nempty[(nunits - 1) & 1]);
        if (!mbar_wait(&nfull[nunits & 1], (uint32_t)((nunits >> 1) & 1))) {
          record_status(status, RI_ERR_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        uE = ust[2 * u.unit];
        uC = ust[2 * u.unit + 1];
        ++nunits;
        prev_unit = u.unit;
      }
      const float* cn = colsm + ((nunits - 1) & 1) * 1024;  // n_j
      const float* ce = cn + 512;                             // e_j
      const int t = u.tile * kRows + row;  // token within the segment
      const bool valid = t < u.L;
      const float kn = valid ? knorm[(size_t)u.bh * d.M + u.seg_start + t] : 0.f;
      const float loose = 2.f * (kn * uE + uC);  // window around the row minimum
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16);
      // pass 1: a_j = ||mu_j||^2 - 2 k.mu_j; per 32-column chunk its minimum,
      // over the row the minimum m (four independent min chains)
      float cm[16];
      float m = FLT_MAX;
      bool ok = true;
#pragma unroll 1
      for (int cp = 0; cp < 8; ++cp) {  // columns 64 cp .. 64 cp + 63 (half cp / 4)
        if ((cp & 3) == 0) {
          if (!mbar_wait(&tfull[cp >> 2], (uint32_t)(it & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        uint32_t r0[32], r1[32];
        tmem_ld32_nowait(taddr + cp * 64, r0);
        tmem_ld32_nowait(taddr + cp * 64 + 32, r1);
        tmem_wait_ld();
        const int jb = cp * 64;
        float m4[4] = {FLT_MAX, FLT_MAX, FLT_MAX, FLT_MAX};
        float n4[4] = {FLT_MAX, FLT_MAX, FLT_MAX, FLT_MAX};
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          m4[i & 3] = fminf(m4[i & 3], fmaf(-2.f, __uint_as_float(r0[i]), cn[jb + i]));
          n4[i & 3] = fminf(n4[i & 3], fmaf(-2.f, __uint_as_float(r1[i]), cn[jb + 32 + i]));
        }
        cm[2 * cp] = fminf(fminf(m4[0], m4[1]), fminf(m4[2], m4[3]));
        cm[2 * cp + 1] = fminf(fminf(n4[0], n4[1]), fminf(n4[2], n4[3]));
        m = fminf(m, fminf(cm[2 * cp], cm[2 * cp + 1]));
      }
      // pass 2: the candidates a_j <= m + loose, from the chunks that can hold
      // one (warp-uniform: the TMEM loads are warp-collective); in id order,
      // at most kCand kept, the rest counted
      const float thr = m + loose;
      int cj[kCand];
      float ca[kCand];
      int nc = 0, best = -1;
      float besta = FLT_MAX;
#pragma unroll
      for (int i = 0; i < kCand; ++i) {
        cj[i] = -1;
        ca[i] = FLT_MAX;
      }
      if (ok) {
#pragma unroll 1
        for (int c = 0; c < 16; ++c) {
          const bool need = cm[c] <= thr;
          if (!__any_sync(0xffffffffu, need)) continue;
          float v[32];
          tmem_ld32(taddr + c * 32, v);
          if (!need) continue;
          const int jb = c * 32;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float a = fmaf(-2.f, v[i], cn[jb + i]);
            if (a <= thr) {
              if (a < besta) {
                besta = a;
                best = jb + i;
              }
#pragma unroll
              for (int k = 0; k < kCand; ++k)
                if (k == nc) {
                  cj[k] = jb + i;
                  ca[k] = a;
                }
              ++nc;
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&tempty[0]);
        mbar_arrive(&tempty[1]);
      }
      if (!ok) {
        record_status(status, RI_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      if (valid) {
        // exact-argmin candidates: lower bound <= least upper bound
        float U = FLT_MAX;
#pragma unroll
        for (int i = 0; i < kCand; ++i)
          if (cj[i] >= 0) U = fminf(U, ca[i] + kn * ce[cj[i]] + col_c(cn[cj[i]]));
        int nsurv = 0;
        uint16_t cands[kCand];
#pragma unroll
        for (int i = 0; i < kCand; ++i) cands[i] = kCandNone;
#pragma unroll
        for (int i = 0; i < kCand; ++i) {
          const bool sv = cj[i] >= 0 && cj[i] < u.Ks &&
                          ca[i] - kn * ce[cj[i]] - col_c(cn[cj[i]]) <= U;
          if (sv) {
#pragma unroll
            for (int k = 0; k < kCand; ++k)
              if (k == nsurv) cands[k] = (uint16_t)cj[i];
            ++nsurv;
          }
        }
        // more candidates than slots: decide by a full scan
        const bool overflow = nc > kCand;
        const int grow = u.bh * d.M + u.seg_start + t;
        labels[grow] = (best >= 0 && best < u.Ks) ? best : 0;
        if (overflow || nsurv != 1) {
          FixEntry e;
          e.row = grow;
#pragma unroll
          for (int i = 0; i < kCand; ++i) e.cand[i] = cands[i];
          if (overflow || nsurv == 0) e.cand[0] = kCandFullScan;
          const int qi = atomicAdd(queue_count, 1);
          queue[qi] = e;
        }
      }
      mbar_arrive(&empty[(int)(it % kStages)]);
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
// ||k|| of every middle token (one warp per row), rounded up so bounds that
// use it stay upper bounds.
__global__ void knorm_kernel(const __nv_bfloat16* __restrict__ K, float* __restrict__ knorm,
                             int N, int M, int m0, long long rows) {
  const long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= rows) return;
  const long long bh = w / M, m = w % M;
  const __nv_bfloat16* src = K + ((size_t)bh * N + m0 + m) * kHeadDim + lane * 4;
  const uint2 raw = *reinterpret_cast<const uint2*>(src);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
  const float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
  float s = a.x * a.x + a.y * a.y + b.x * b.x + b.y * b.y;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
  if (lane == 0) knorm[w] = sqrtf(s) * 1.0001f;
}

// Seeds: mu_j = k at the given (or strided) position of the segment.  One
// warp per (bh, s, j in [0, 512)); j >= K_s only pads the column table.
__global__ void init_kernel(const __nv_bfloat16* __restrict__ K,
                            const int32_t* __restrict__ init_pos, BuildDims d,
                            float* __restrict__ mu, __nv_bfloat16* __restrict__ mu_bf16,
                            float* __restrict__ colt, float* __restrict__ ust, int* status,
                            long long total) {
  const long long w = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= total) return;
  const int unit = (int)(w / kMaxClustersPerSeg);
  const int j = (int)(w % kMaxClustersPerSeg);
  const int bh = unit / d.S, s = unit % d.S;
  const bool last = s == d.S - 1;
  const int L = last ? d.L_last : d.seg_len;
  const int Ks = last ? d.K_last : d.K_full;
  float* cn = colt + (size_t)unit * 1024;
  if (j >= Ks) {
    if (lane == 0) {
      cn[j] = INFINITY;
      cn[512 + j] = 0.f;
    }
    return;
  }
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
  centroid_stats(m, mu_bf16 + ((size_t)bh * d.C + c) * kHeadDim, &cn[j], &cn[512 + j],
                 ust + 2 * unit, lane, true);
}

// ------------------------------------------------------------- update / finalise
// Members of the block's clusters [j0, j0 + ncl) of one segment, in position
// order, grouped by cluster: sorted[start[c] .. start[c+1]) are the positions
// (within the segment) of cluster j0 + c.  Returns the member total.
// Shared memory: list[L], sorted[L], start[33], wtot[8].
__device__ int gather_members(const int32_t* __restrict__ lab, int L, int j0, int ncl,
                              int* list, int* sorted, int* start, int* wtot) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const unsigned lt = (1u << lane) - 1u;
  int run = 0;
  // 1) compaction of (position, cluster) pairs, position order
  for (int base = 0; base < L; base += blockDim.x) {
    const int t = base + threadIdx.x;
    const int c = t < L ? lab[t] - j0 : -1;
    const bool mine = c >= 0 && c < ncl;
    const unsigned m = __ballot_sync(0xffffffffu, mine);
    if (lane == 0) wtot[warp] = __popc(m);
    __syncthreads();
    int before = 0, tot = 0;
    for (int w = 0; w < kUpdateWarps; ++w) {
      before += w < warp ? wtot[w] : 0;
      tot += wtot[w];
    }
    if (mine) list[run + before + __popc(m & lt)] = (t << 5) | c;
    run += tot;
    __syncthreads();
  }
  // 2) per-cluster counts and starts
  if (threadIdx.x < 33) start[threadIdx.x] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < run; i += blockDim.x) atomicAdd(&start[(list[i] & 31) + 1], 1);
  __syncthreads();
  if (threadIdx.x == 0)
    for (int c = 1; c <= 32; ++c) start[c] += start[c - 1];
  __syncthreads();
  // 3) stable grouping: warp w moves the members of clusters 4w..4w+3
  for (int cc = 0; cc < kClustersPerWarp; ++cc) {
    const int c = warp * kClustersPerWarp + cc;
    int pos = start[c];
    for (int base = 0; base < run; base += 32) {
      const int i = base + lane;
      const int e = i < run ? list[i] : -1;
      const bool mine = e >= 0 && (e & 31) == c;
      const unsigned m = __ballot_sync(0xffffffffu, mine);
      if (mine) sorted[pos + __popc(m & lt)] = e >> 5;
      pos += __popc(m);
    }
  }
  __syncthreads();
  return run;
}

__global__ void __launch_bounds__(kUpdateWarps * 32)
    update_kernel(const __nv_bfloat16* __restrict__ K, const int32_t* __restrict__ labels,
                  BuildDims d, float* __restrict__ mu, __nv_bfloat16* __restrict__ mu_bf16,
                  float* __restrict__ colt, float* __restrict__ ust,
                  int32_t* __restrict__ counts, int update_mu) {
  extern __shared__ __align__(16) uint8_t smem_u[];
  __shared__ int start[33], wtot[kUpdateWarps];
  const int unit = blockIdx.x;
  const int bh = unit / d.S, s = unit % d.S;
  const bool last = s == d.S - 1;
  const int L = last ? d.L_last : d.seg_len;
  const int Ks = last ? d.K_last : d.K_full;
  const int j0 = blockIdx.y * kClustersPerBlock;
  if (j0 >= Ks) return;
  const int ncl = min(kClustersPerBlock, Ks - j0);
  int* list = reinterpret_cast<int*>(smem_u);
  int* sorted = list + d.seg_len;
  const int seg_start = s * d.seg_len;
  gather_members(labels + (size_t)bh * d.M + seg_start, L, j0, ncl, list, sorted, start, wtot);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const __nv_bfloat16* kbase = K + ((size_t)bh * d.N + d.m0 + seg_start) * kHeadDim + lane * 4;
  float* cn = colt + (size_t)unit * 1024;
  for (int cc = 0; cc < kClustersPerWarp; ++cc) {
    const int c = warp * kClustersPerWarp + cc;
    if (c >= ncl) break;
    const int b = start[c], e = start[c + 1];
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int i = b; i < e; i += 16) {
      uint2 raw[16];
#pragma unroll
      for (int u = 0; u < 16; ++u)
        raw[u] = i + u < e
                     ? *reinterpret_cast<const uint2*>(kbase + (size_t)sorted[i + u] * kHeadDim)
                     : make_uint2(0, 0);
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        if (i + u < e) {
          const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
          const float2 a = __bfloat1622float2(h[0]), bb = __bfloat1622float2(h[1]);
          acc[0] += a.x;
          acc[1] += a.y;
          acc[2] += bb.x;
          acc[3] += bb.y;
        }
      }
    }
    const int j = j0 + c;
    const size_t row = (size_t)bh * d.C + (size_t)s * d.K_full + j;
    const int n = e - b;
    if (update_mu && n > 0) {
      const float fn = (float)n;
      const float4 m = make_float4(acc[0] / fn, acc[1] / fn, acc[2] / fn, acc[3] / fn);
      *reinterpret_cast<float4*>(mu + row * kHeadDim + lane * 4) = m;
      centroid_stats(m, mu_bf16 + row * kHeadDim, &cn[j], &cn[512 + j], ust + 2 * unit, lane,
                     true);
    } else {
      const float4 m = *reinterpret_cast<const float4*>(mu + row * kHeadDim + lane * 4);
      centroid_stats(m, mu_bf16 + row * kHeadDim, &cn[j], &cn[512 + j], ust + 2 * unit, lane,
                     false);
    }
    if (lane == 0) counts[row] = n;
  }
}

__global__ void __launch_bounds__(kUpdateWarps * 32)
    finalise_kernel(const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V,
                    const int32_t* __restrict__ labels, BuildDims d, const float* __restrict__ mu,
                    ri_index out) {
  extern __shared__ __align__(16) uint8_t smem_u[];
  __shared__ int start[33], wtot[kUpdateWarps], before_sm;
  const int unit = blockIdx.x;
  const int bh = unit / d.S, s = unit % d.S;
  const bool last = s == d.S - 1;
  const int L = last ? d.L_last : d.seg_len;
  const int Ks = last ? d.K_last : d.K_full;
  const int j0 = blockIdx.y * kClustersPerBlock;
  if (j0 >= Ks) return;
  const int ncl = min(kClustersPerBlock, Ks - j0);
  int* list = reinterpret_cast<int*>(smem_u);
  int* sorted = list + d.seg_len;
  const int seg_start = s * d.seg_len;
  const int cbase = s * d.K_full;
  const int32_t* lab = labels + (size_t)bh * d.M + seg_start;
  if (out.labels && blockIdx.y == 0)
    for (int t = threadIdx.x; t < L; t += blockDim.x)
      out.labels[(size_t)bh * d.M + seg_start + t] = lab[t];
  if (blockIdx.y == 0 && s == d.S - 1 && threadIdx.x == 0)
    out.offsets[(size_t)bh * (d.C + 1) + d.C] = d.M;
  // rows of the segment taken by clusters before j0: tokens with label < j0
  if (threadIdx.x == 0) before_sm = 0;
  __syncthreads();
  {
    int cnt = 0;
    for (int t = threadIdx.x; t < L; t += blockDim.x) cnt += lab[t] < j0;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    if ((threadIdx.x & 31) == 0) atomicAdd(&before_sm, cnt);
  }
  gather_members(lab, L, j0, ncl, list, sorted, start, wtot);
  const int before = before_sm;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const size_t bhN = (size_t)bh * d.N + d.m0 + seg_start;
  const size_t bhM = (size_t)bh * d.M + seg_start;
  float obj = 0.f;
  for (int cc = 0; cc < kClustersPerWarp; ++cc) {
    const int c = warp * kClustersPerWarp + cc;
    if (c >= ncl) break;
    const int b = start[c], e = start[c + 1];
    const size_t crow = (size_t)bh * d.C + cbase + j0 + c;
    const float4 m = *reinterpret_cast<const float4*>(mu + crow * kHeadDim + lane * 4);
    float vs[4] = {0.f, 0.f, 0.f, 0.f};
    for (int i = b; i < e; i += 8) {
      uint2 kr[8], vr[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const bool in = i + u < e;
        const size_t src = (bhN + (in ? sorted[i + u] : 0)) * kHeadDim + lane * 4;
        kr[u] = in ? *reinterpret_cast<const uint2*>(K + src) : make_uint2(0, 0);
        vr[u] = in ? *reinterpret_cast<const uint2*>(V + src) : make_uint2(0, 0);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (i + u < e) {
          const int r = before + i + u;  // rows are in (cluster, position) order
          const size_t dst = (bhM + r) * kHeadDim + lane * 4;
          *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out.Kp) + dst) = kr[u];
          *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out.Vp) + dst) = vr[u];
          if (lane == 0) out.perm[bhM + r] = d.m0 + seg_start + sorted[i + u];
          const __nv_bfloat162* kh = reinterpret_cast<const __nv_bfloat162*>(&kr[u]);
          const __nv_bfloat162* vh = reinterpret_cast<const __nv_bfloat162*>(&vr[u]);
          const float2 ka = __bfloat1622float2(kh[0]), kb = __bfloat1622float2(kh[1]);
          const float2 va = __bfloat1622float2(vh[0]), vb = __bfloat1622float2(vh[1]);
          vs[0] += va.x;
          vs[1] += va.y;
          vs[2] += vb.x;
          vs[3] += vb.y;
          const float d0 = ka.x - m.x, d1 = ka.y - m.y, d2 = kb.x - m.z, d3 = kb.y - m.w;
          obj += d0 * d0 + d1 * d1 + d2 * d2 + d3 * d3;
        }
      }
    }
    *reinterpret_cast<float4*>(out.vsum + crow * kHeadDim + lane * 4) =
        make_float4(vs[0], vs[1], vs[2], vs[3]);
    const __nv_bfloat162 lo = __floats2bfloat162_rn(m.x, m.y);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(m.z, m.w);
    uint2 packed;
    packed.x = *reinterpret_cast<const uint32_t*>(&lo);
    packed.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out.centroid) + crow * kHeadDim +
                              lane * 4) = packed;
    if (lane == 0) {
      out.counts[crow] = e - b;
      out.offsets[(size_t)bh * (d.C + 1) + cbase + j0 + c] = seg_start + before + b;
    }
  }
  if (out.objective) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) obj += __shfl_xor_sync(0xffffffffu, obj, off);
    if (lane == 0) atomicAdd(&out.objective[unit], obj);
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
  d.total_tiles = BH * g.tiles_bh;
  float* mu = reinterpret_cast<float*>(ws + L.off_mu);
  __nv_bfloat16* mu_bf16 = reinterpret_cast<__nv_bfloat16*>(ws + L.off_mu_bf16);
  float* colt = reinterpret_cast<float*>(ws + L.off_colt);
  float* ust = reinterpret_cast<float*>(ws + L.off_ust);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + L.off_counts);
  int32_t* labels = reinterpret_cast<int32_t*>(ws + L.off_labels);
  float* knorm = reinterpret_cast<float*>(ws + L.off_knorm);
  FixEntry* queue = reinterpret_cast<FixEntry*>(ws + L.off_queue);
  const long long units = BH * g.S;

  CUtensorMap tm_keys, tm_cent;
  if (!make_map_bf16(&tm_keys, a.K, (unsigned long long)BH * g.N, kRows) ||
      !make_map_bf16(&tm_cent, mu_bf16, (unsigned long long)BH * g.C, kHalfN)) {
    set_error("cuTensorMapEncodeTiled failed");
    return RI_ERR_CUDA;
  }
  const long long rows = BH * g.M;
  knorm_kernel<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(K, knorm, g.N, g.M, g.m0, rows);
  RI_CUDA_TRY(cudaGetLastError());
  RI_CUDA_TRY(cudaMemsetAsync(ust, 0, units * 2 * sizeof(float), st));
  const long long init_total = units * kMaxClustersPerSeg;
  init_kernel<<<(unsigned)((init_total + 7) / 8), 256, 0, st>>>(K, a.init_pos, d, mu, mu_bf16,
                                                                 colt, ust, status, init_total);
  RI_CUDA_TRY(cudaGetLastError());

  RI_CUDA_TRY(set_smem_once(reinterpret_cast<const void*>(assign_kernel), (int)kAssignSmem));
  const size_t upd_smem = (size_t)g.seg_len * 2 * sizeof(int);
  const int upd_smem_max = (int)(kMaxSegLen * 2 * sizeof(int));
  RI_CUDA_TRY(set_smem_once(reinterpret_cast<const void*>(update_kernel), upd_smem_max));
  RI_CUDA_TRY(set_smem_once(reinterpret_cast<const void*>(finalise_kernel), upd_smem_max));
  const int sms = num_sms();
  const unsigned grid_assign = (unsigned)(d.total_tiles < (long long)sms ? d.total_tiles : sms);
  const dim3 grid_upd((unsigned)units, (unsigned)((g.K_full + kClustersPerBlock - 1) /
                                                  kClustersPerBlock));
  const int rounds = g.iters > 0 ? g.iters : 1;
  for (int t = 0; t < rounds; ++t) {
    RI_CUDA_TRY(cudaMemsetAsync(queue_count, 0, sizeof(int), st));
    assign_kernel<<<grid_assign, kAssignThreads, kAssignSmem, st>>>(
        tm_keys, tm_cent, d, knorm, colt, ust, labels, queue, queue_count, status);
    RI_CUDA_TRY(cudaGetLastError());
    fixup_kernel<<<(unsigned)(4 * sms), 256, 0, st>>>(K, mu, d, queue, queue_count, labels);
    RI_CUDA_TRY(cudaGetLastError());
    RI_CUDA_TRY(cudaMemsetAsync(ust, 0, units * 2 * sizeof(float), st));
    update_kernel<<<grid_upd, kUpdateWarps * 32, upd_smem, st>>>(
        K, labels, d, mu, mu_bf16, colt, ust, counts, g.iters > 0 ? 1 : 0);
    RI_CUDA_TRY(cudaGetLastError());
  }
  if (a.out.objective)
    RI_CUDA_TRY(cudaMemsetAsync(a.out.objective, 0, units * sizeof(float), st));
  finalise_kernel<<<grid_upd, kUpdateWarps * 32, upd_smem, st>>>(K, V, labels, d, mu, a.out);
  RI_CUDA_TRY(cudaGetLastError());
  return RI_OK;
}

}  // namespace ri
