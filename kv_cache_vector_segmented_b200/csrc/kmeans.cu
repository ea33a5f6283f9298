// Segmented k-means index build of the wave index (sm_100a).
//
// Segmented clustering ("KV缓存技术与RetroInfer系统在长上下文推理中的优化实践",
// framerc.cn, §2.1 pseudocode: k-means per 8K-token segment, segments in
// parallel, centroids plus per-cluster value sums) and the cluster-contiguous
// layout (§3.1: the KV vectors of one cluster stored contiguously).
//
// One Lloyd iteration = assignment (tensor cores) + update (segmented sums).
//   assignment: label_i = argmin_j ||k_i - mu_j||^2
//             = argmin_j (||mu_j||^2 - 2 k_i . mu_j), ties to the lower j.
//     tcgen05 MMA: 128 keys x 256 centroids x 128 dims per instruction group,
//     bf16 operands (keys exact in bf16, centroids rounded to bf16), fp32
//     accumulators in TMEM.  The bf16 centroid costs at most
//     2^-7 ||k|| ||mu_j|| in the distance (|mu - bf16(mu)| <= 2^-8 |mu| per
//     element, Cauchy-Schwarz), plus fp32 accumulation error; every centroid
//     whose approximate distance lies within twice that bound of the best is
//     re-evaluated exactly in fp32 (direct difference form).
//   update: mu_j = mean of members (fp32), an empty cluster keeps mu_j.
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
constexpr int kUpdateWarps = 8;
constexpr int kClustersPerWarp = 4;
constexpr int kClustersPerBlock = kUpdateWarps * kClustersPerWarp;  // 32
constexpr int kMemberBuf = 256;   // member token queue per warp (update/finalise)

// Shared memory of the assignment kernel (from a 1024-byte aligned base).
constexpr uint32_t kSmCent = 0;                                // [2 k-halves][512][128 B]
constexpr uint32_t kCentHalfK = 512 * 128;                     // 64 KB
constexpr uint32_t kSmKeys = 2 * kCentHalfK;                   // 128 KB
constexpr uint32_t kKeyStage = 2 * kRows * 128;                // 32 KB
constexpr uint32_t kSmNrm = kSmKeys + kStages * kKeyStage;     // [2][512] fp32
constexpr uint32_t kSmBar = kSmNrm + 2 * 512 * 4;
constexpr int kNumBars = 2 * kStages + 2 + 2 + 2 + 2 + 2 + 1;
constexpr uint32_t kSmMisc = kSmBar + kNumBars * 8;
constexpr uint32_t kAssignSmem = kSmMisc + 64 + 1024;          // + alignment slack

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

// Exact squared distance in fp32 between row `row` of a swizzled key tile in
// shared memory (two 64-column halves of 128-byte rows) and an fp32 centroid.
__device__ __forceinline__ float exact_dist(const uint8_t* tile, int row, const float* mu) {
  float acc = 0.f;
#pragma unroll 4
  for (int c = 0; c < 16; ++c) {
    const int kh = c >> 3, ch = c & 7;
    const uint4 raw = *reinterpret_cast<const uint4*>(tile + kh * (kRows * 128) + row * 128 +
                                                      ((ch ^ (row & 7)) << 4));
    float k[8];
    bf16x8_to_float(raw, k);
    const float4 m0 = *reinterpret_cast<const float4*>(mu + c * 8);
    const float4 m1 = *reinterpret_cast<const float4*>(mu + c * 8 + 4);
    const float mm[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float t = k[i] - mm[i];
      acc = fmaf(t, t, acc);
    }
  }
  return acc;
}

// ------------------------------------------------------------- assignment
__global__ void __launch_bounds__(kAssignThreads, 1)
    assign_kernel(const __grid_constant__ CUtensorMap tm_keys,
                  const __grid_constant__ CUtensorMap tm_cent, BuildDims d,
                  const float* __restrict__ knorm, const float* __restrict__ norm2,
                  const float* __restrict__ mumax, const float* __restrict__ mu,
                  int32_t* __restrict__ labels, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* cent = sm + kSmCent;
  uint8_t* keys = sm + kSmKeys;
  float* nrm = reinterpret_cast<float*>(sm + kSmNrm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + kSmBar);
  uint64_t* full = bars;                       // [kStages] TMA -> MMA
  uint64_t* empty = bars + kStages;            // [kStages] epilogue -> TMA
  uint64_t* cent_full = bars + 2 * kStages;    // TMA -> MMA
  uint64_t* cent_empty = cent_full + 1;        // MMA -> TMA
  uint64_t* tfull = cent_full + 2;             // [2] MMA -> epilogue
  uint64_t* tempty = tfull + 2;                // [2] epilogue -> MMA
  uint64_t* nfull = tempty + 2;                // [2] TMA -> epilogue (norms)
  uint64_t* nempty = nfull + 2;                // [2] epilogue -> TMA  (uses 1 slot each)
  uint64_t* drain = nfull + 4;                 // MMA drain
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
    int cent_loads = 0, nrm_loads[2] = {0, 0};
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
        // per-unit squared centroid norms for the epilogue (double buffer)
        const int nb = nunits & 1;
        if (nunits >= 2) {
          if (!mbar_wait(&nempty[nb], ((nunits >> 1) - 1) & 1)) {
            record_status(status, RI_ERR_TIMEOUT);
            *abort_flag = 1;
            break;
          }
        }
        mbar_arrive_expect_tx(&nfull[nb], 512 * 4);
        bulk_load(nrm + nb * 512, norm2 + (size_t)u.unit * 512, 512 * 4, &nfull[nb]);
        ++nrm_loads[nb];
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
      if (nrm_loads[nb]) mbar_wait(&nfull[nb], (uint32_t)((nrm_loads[nb] - 1) & 1));
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
    float mx = 0.f;
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
        mx = mumax[u.unit];
        ++nunits;
        prev_unit = u.unit;
      }
      const float* nr = nrm + ((nunits - 1) & 1) * 512;
      const int t = u.tile * kRows + row;  // token within the segment
      const bool valid = t < u.L;
      const float kn = valid ? knorm[(size_t)u.bh * d.M + u.seg_start + t] : 0.f;
      // bound on |approx - exact| of one distance, doubled for the window
      const float eps = 0.0078125f * 1.0157f * kn * mx + 3.0517578e-5f * (kn * kn + mx * mx);
      const float win = 2.f * eps;
      float a0 = FLT_MAX, a1 = FLT_MAX, a2 = FLT_MAX, a3 = FLT_MAX;
      int j0 = -1, j1 = -1, j2 = -1, j3 = -1;
      float dropped = FLT_MAX, thr = FLT_MAX;
      bool ok = true;
      for (int h = 0; h < 2; ++h) {
        if (!mbar_wait(&tfull[h], (uint32_t)(it & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int ch = 0; ch < 8; ++ch) {
          float v[32];
          tmem_ld32(tmem + ((uint32_t)(quad * 32) << 16) + h * kHalfN + ch * 32, v);
          const int jb = h * kHalfN + ch * 32;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float a = fmaf(-2.f, v[i], nr[jb + i]);
            if (a <= thr) {
              float na = a;
              int nj = jb + i;
              if (na < a0) { float tf = a0; a0 = na; na = tf; int ti = j0; j0 = nj; nj = ti; }
              if (na < a1) { float tf = a1; a1 = na; na = tf; int ti = j1; j1 = nj; nj = ti; }
              if (na < a2) { float tf = a2; a2 = na; na = tf; int ti = j2; j2 = nj; nj = ti; }
              if (na < a3) { float tf = a3; a3 = na; na = tf; int ti = j3; j3 = nj; nj = ti; }
              dropped = fminf(dropped, na);
              thr = a0 + win;
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&tempty[h]);
      }
      if (!ok) {
        record_status(status, RI_ERR_TIMEOUT);
        *abort_flag = 1;
        break;
      }
      const int stage = (int)(it % kStages);
      const uint8_t* tile = keys + stage * kKeyStage;
      int label = (j0 < 0 || j0 >= u.Ks) ? 0 : j0;
      if (valid && j0 >= 0 && j0 < u.Ks) {
        const float lim = a0 + win;
        const int nc = (a1 <= lim) + (a2 <= lim) + (a3 <= lim);
        const float* mub = mu + ((size_t)u.bh * d.C + u.cbase) * kHeadDim;
        if (dropped <= lim) {
          // more near-ties than the candidate list holds: exact scan
          float best = FLT_MAX;
          for (int j = 0; j < u.Ks; ++j) {
            const float e = exact_dist(tile, row, mub + (size_t)j * kHeadDim);
            if (e < best) {
              best = e;
              label = j;
            }
          }
        } else if (nc > 0) {
          float best = exact_dist(tile, row, mub + (size_t)j0 * kHeadDim);
          label = j0;
          const int cj[3] = {j1, j2, j3};
#pragma unroll
          for (int c = 0; c < 3; ++c) {
            if (c < nc && cj[c] >= 0 && cj[c] < u.Ks) {
              const float e = exact_dist(tile, row, mub + (size_t)cj[c] * kHeadDim);
              if (e < best || (e == best && cj[c] < label)) {
                best = e;
                label = cj[c];
              }
            }
          }
        }
      }
      if (valid) labels[(size_t)u.bh * d.M + u.seg_start + t] = label;
      mbar_arrive(&empty[stage]);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------- prep
// ||k|| of every middle token (one warp per row).
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
  if (lane == 0) knorm[w] = sqrtf(s);
}

__device__ __forceinline__ void atomic_max_pos(float* addr, float v) {
  atomicMax(reinterpret_cast<int*>(addr), __float_as_int(v));  // v >= 0
}

// Seeds: mu_j = k at the given (or strided) position of the segment.  One
// warp per (bh, s, j in [0, 512)); j >= K_s only pads the norm table.
__global__ void init_kernel(const __nv_bfloat16* __restrict__ K,
                            const int32_t* __restrict__ init_pos, BuildDims d,
                            float* __restrict__ mu, __nv_bfloat16* __restrict__ mu_bf16,
                            float* __restrict__ norm2, float* __restrict__ mumax, int* status,
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
  if (j >= Ks) {
    if (lane == 0) norm2[(size_t)unit * 512 + j] = INFINITY;
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
  const __nv_bfloat16* src = K + ((size_t)bh * d.N + d.m0 + s * d.seg_len + p) * kHeadDim + lane * 4;
  const uint2 raw = *reinterpret_cast<const uint2*>(src);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
  const float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
  float* dst = mu + ((size_t)bh * d.C + c) * kHeadDim + lane * 4;
  *reinterpret_cast<float4*>(dst) = make_float4(a.x, a.y, b.x, b.y);
  *reinterpret_cast<uint2*>(mu_bf16 + ((size_t)bh * d.C + c) * kHeadDim + lane * 4) = raw;
  float sq = a.x * a.x + a.y * a.y + b.x * b.x + b.y * b.y;
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
  if (lane == 0) {
    norm2[(size_t)unit * 512 + j] = sq;
    atomic_max_pos(&mumax[unit], sqrtf(sq));
  }
}

// ------------------------------------------------------------- update / finalise
// Member scan shared by update and finalise: the warp walks the segment's
// labels (shared memory, uint16) in position order and queues the tokens of
// its clusters [jw, jw + 4); `visit(t, cl)` is called for each member in
// position order, 8 row loads in flight at a time by the caller's batching.
struct MemberQueue {
  int buf[kMemberBuf];  // (t << 2) | cl
};

template <typename Visit>
__device__ __forceinline__ void scan_members(const uint16_t* lab, int L, int jw, int nclw,
                                             MemberQueue& q, Visit&& visit) {
  const int lane = threadIdx.x & 31;
  int pos = 0;
  while (pos < L) {
    int n = 0;
    while (pos < L && n <= kMemberBuf - 32) {
      const int t = pos + lane;
      const int c = t < L ? (int)lab[t] - jw : -1;
      const bool mine = c >= 0 && c < nclw;
      const unsigned m = __ballot_sync(0xffffffffu, mine);
      if (mine) q.buf[n + __popc(m & ((1u << lane) - 1u))] = (t << 2) | c;
      n += __popc(m);
      pos += 32;
    }
    __syncwarp();
    visit(n);
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kUpdateWarps * 32)
    update_kernel(const __nv_bfloat16* __restrict__ K, const int32_t* __restrict__ labels,
                  BuildDims d, float* __restrict__ mu, __nv_bfloat16* __restrict__ mu_bf16,
                  float* __restrict__ norm2, float* __restrict__ mumax,
                  int32_t* __restrict__ counts, int update_mu) {
  extern __shared__ __align__(16) uint8_t smem_u[];
  uint16_t* lab = reinterpret_cast<uint16_t*>(smem_u);
  MemberQueue* queues = reinterpret_cast<MemberQueue*>(smem_u + (((size_t)d.seg_len * 2 + 15) & ~(size_t)15));
  const int unit = blockIdx.x;
  const int bh = unit / d.S, s = unit % d.S;
  const bool last = s == d.S - 1;
  const int L = last ? d.L_last : d.seg_len;
  const int Ks = last ? d.K_last : d.K_full;
  const int j0 = blockIdx.y * kClustersPerBlock;
  if (j0 >= Ks) return;
  const int seg_start = s * d.seg_len;
  const int32_t* lsrc = labels + (size_t)bh * d.M + seg_start;
  for (int t = threadIdx.x; t < L; t += blockDim.x) lab[t] = (uint16_t)lsrc[t];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int jw = j0 + warp * kClustersPerWarp;
  const int nclw = max(0, min(kClustersPerWarp, Ks - jw));
  if (nclw == 0) return;
  MemberQueue& q = queues[warp];
  float acc[kClustersPerWarp][4];
  int n[kClustersPerWarp];
#pragma unroll
  for (int c = 0; c < kClustersPerWarp; ++c) {
    n[c] = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[c][i] = 0.f;
  }
  const __nv_bfloat16* kbase = K + ((size_t)bh * d.N + d.m0 + seg_start) * kHeadDim + lane * 4;
  scan_members(lab, L, jw, nclw, q, [&](int cnt) {
    for (int i = 0; i < cnt; i += 8) {
      uint2 raw[8];
      int cl[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int e = i + u < cnt ? q.buf[i + u] : -1;
        cl[u] = e < 0 ? -1 : (e & 3);
        raw[u] = e < 0 ? make_uint2(0, 0)
                       : *reinterpret_cast<const uint2*>(kbase + (size_t)(e >> 2) * kHeadDim);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw[u]);
        const float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
#pragma unroll
        for (int c = 0; c < kClustersPerWarp; ++c) {
          if (cl[u] == c) {
            acc[c][0] += a.x;
            acc[c][1] += a.y;
            acc[c][2] += b.x;
            acc[c][3] += b.y;
            n[c] += 1;
          }
        }
      }
    }
  });
  float wmax = 0.f;
#pragma unroll
  for (int c = 0; c < kClustersPerWarp; ++c) {
    if (c >= nclw) break;
    const int j = jw + c;
    const size_t row = (size_t)bh * d.C + s * d.K_full + j;
    float* mrow = mu + row * kHeadDim + lane * 4;
    float4 m;
    if (update_mu && n[c] > 0) {
      const float fn = (float)n[c];
      m = make_float4(acc[c][0] / fn, acc[c][1] / fn, acc[c][2] / fn, acc[c][3] / fn);
      *reinterpret_cast<float4*>(mrow) = m;
      __nv_bfloat162 lo = __floats2bfloat162_rn(m.x, m.y), hi = __floats2bfloat162_rn(m.z, m.w);
      uint2 packed;
      packed.x = *reinterpret_cast<uint32_t*>(&lo);
      packed.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(mu_bf16 + row * kHeadDim + lane * 4) = packed;
    } else {
      m = *reinterpret_cast<const float4*>(mrow);
    }
    float sq = m.x * m.x + m.y * m.y + m.z * m.z + m.w * m.w;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
    if (lane == 0) {
      norm2[(size_t)unit * 512 + j] = sq;
      counts[row] = n[c];
    }
    wmax = fmaxf(wmax, sqrtf(sq));
  }
  if (lane == 0) atomic_max_pos(&mumax[unit], wmax);
}

__global__ void __launch_bounds__(kUpdateWarps * 32)
    finalise_kernel(const __nv_bfloat16* __restrict__ K, const __nv_bfloat16* __restrict__ V,
                    const int32_t* __restrict__ labels, BuildDims d, const float* __restrict__ mu,
                    const int32_t* __restrict__ counts_ws, ri_index out) {
  extern __shared__ __align__(16) uint8_t smem_u[];
  uint16_t* lab = reinterpret_cast<uint16_t*>(smem_u);
  MemberQueue* queues = reinterpret_cast<MemberQueue*>(smem_u + (((size_t)d.seg_len * 2 + 15) & ~(size_t)15));
  const int unit = blockIdx.x;
  const int bh = unit / d.S, s = unit % d.S;
  const bool last = s == d.S - 1;
  const int L = last ? d.L_last : d.seg_len;
  const int Ks = last ? d.K_last : d.K_full;
  const int j0 = blockIdx.y * kClustersPerBlock;
  if (j0 >= Ks) return;
  const int seg_start = s * d.seg_len;
  const int cbase = s * d.K_full;
  const int32_t* lsrc = labels + (size_t)bh * d.M + seg_start;
  for (int t = threadIdx.x; t < L; t += blockDim.x) {
    const int v = lsrc[t];
    lab[t] = (uint16_t)v;
    if (out.labels && blockIdx.y == 0) out.labels[(size_t)bh * d.M + seg_start + t] = v;
  }
  if (blockIdx.y == 0 && s == d.S - 1 && threadIdx.x == 0)
    out.offsets[(size_t)bh * (d.C + 1) + d.C] = d.M;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int jw = j0 + warp * kClustersPerWarp;
  const int nclw = max(0, min(kClustersPerWarp, Ks - jw));
  if (nclw == 0) return;
  const int32_t* cnt = counts_ws + (size_t)bh * d.C + cbase;
  // rows before cluster jw within the segment
  int before = 0;
  for (int j = lane; j < jw; j += 32) before += cnt[j];
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) before += __shfl_xor_sync(0xffffffffu, before, off);
  int rowstart[kClustersPerWarp];
  {
    int r = before;
#pragma unroll
    for (int c = 0; c < kClustersPerWarp; ++c) {
      rowstart[c] = r;
      if (c < nclw) r += cnt[jw + c];
    }
  }
  int rank[kClustersPerWarp] = {0, 0, 0, 0};
  float vs[kClustersPerWarp][4];
  float obj = 0.f;
  float mrow[kClustersPerWarp][4];
#pragma unroll
  for (int c = 0; c < kClustersPerWarp; ++c) {
#pragma unroll
    for (int i = 0; i < 4; ++i) vs[c][i] = 0.f;
    if (c < nclw) {
      const float4 m = *reinterpret_cast<const float4*>(
          mu + ((size_t)bh * d.C + cbase + jw + c) * kHeadDim + lane * 4);
      mrow[c][0] = m.x; mrow[c][1] = m.y; mrow[c][2] = m.z; mrow[c][3] = m.w;
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) mrow[c][i] = 0.f;
    }
  }
  const size_t bhN = (size_t)bh * d.N + d.m0 + seg_start;
  const size_t bhM = (size_t)bh * d.M + seg_start;
  MemberQueue& q = queues[warp];
  scan_members(lab, L, jw, nclw, q, [&](int cntq) {
    for (int i = 0; i < cntq; i += 8) {
      uint2 kr[8], vr[8];
      int e[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        e[u] = i + u < cntq ? q.buf[i + u] : -1;
        const size_t src = (bhN + (e[u] < 0 ? 0 : (e[u] >> 2))) * kHeadDim + lane * 4;
        kr[u] = e[u] < 0 ? make_uint2(0, 0) : *reinterpret_cast<const uint2*>(K + src);
        vr[u] = e[u] < 0 ? make_uint2(0, 0) : *reinterpret_cast<const uint2*>(V + src);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (e[u] < 0) continue;
        const int t = e[u] >> 2, c = e[u] & 3;
        int r = 0;
#pragma unroll
        for (int cc = 0; cc < kClustersPerWarp; ++cc)
          if (cc == c) r = rowstart[cc] + rank[cc]++;
        const size_t dst = (bhM + r) * kHeadDim + lane * 4;
        *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out.Kp) + dst) = kr[u];
        *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out.Vp) + dst) = vr[u];
        if (lane == 0) out.perm[bhM + r] = d.m0 + seg_start + t;
        const __nv_bfloat162* kh = reinterpret_cast<const __nv_bfloat162*>(&kr[u]);
        const __nv_bfloat162* vh = reinterpret_cast<const __nv_bfloat162*>(&vr[u]);
        const float2 ka = __bfloat1622float2(kh[0]), kb = __bfloat1622float2(kh[1]);
        const float2 va = __bfloat1622float2(vh[0]), vb = __bfloat1622float2(vh[1]);
#pragma unroll
        for (int cc = 0; cc < kClustersPerWarp; ++cc) {
          if (cc == c) {
            vs[cc][0] += va.x; vs[cc][1] += va.y; vs[cc][2] += vb.x; vs[cc][3] += vb.y;
            const float d0 = ka.x - mrow[cc][0], d1 = ka.y - mrow[cc][1];
            const float d2 = kb.x - mrow[cc][2], d3 = kb.y - mrow[cc][3];
            obj += d0 * d0 + d1 * d1 + d2 * d2 + d3 * d3;
          }
        }
      }
    }
  });
#pragma unroll
  for (int c = 0; c < kClustersPerWarp; ++c) {
    if (c >= nclw) break;
    const size_t row = (size_t)bh * d.C + cbase + jw + c;
    *reinterpret_cast<float4*>(out.vsum + row * kHeadDim + lane * 4) =
        make_float4(vs[c][0], vs[c][1], vs[c][2], vs[c][3]);
    __nv_bfloat162 lo = __floats2bfloat162_rn(mrow[c][0], mrow[c][1]);
    __nv_bfloat162 hi = __floats2bfloat162_rn(mrow[c][2], mrow[c][3]);
    uint2 packed;
    packed.x = *reinterpret_cast<uint32_t*>(&lo);
    packed.y = *reinterpret_cast<uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(out.centroid) + row * kHeadDim +
                              lane * 4) = packed;
    if (lane == 0) {
      out.counts[row] = cnt[jw + c];
      out.offsets[(size_t)bh * (d.C + 1) + cbase + jw + c] = seg_start + rowstart[c];
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

ri_status launch_build(const Geometry& g, const BuildLayout& L, const BuildArgs& a,
                       cudaStream_t st) {
  char* ws = a.ws;
  int* status = reinterpret_cast<int*>(ws);
  const __nv_bfloat16* K = static_cast<const __nv_bfloat16*>(a.K);
  const __nv_bfloat16* V = static_cast<const __nv_bfloat16*>(a.V);
  const long long BH = g.BH();
  // steady buffers
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
  float* norm2 = reinterpret_cast<float*>(ws + L.off_norm2);
  float* mumax = reinterpret_cast<float*>(ws + L.off_mumax);
  int32_t* counts = reinterpret_cast<int32_t*>(ws + L.off_counts);
  int32_t* labels = reinterpret_cast<int32_t*>(ws + L.off_labels);
  float* knorm = reinterpret_cast<float*>(ws + L.off_knorm);
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
  RI_CUDA_TRY(cudaMemsetAsync(mumax, 0, units * sizeof(float), st));
  const long long init_total = units * kMaxClustersPerSeg;
  init_kernel<<<(unsigned)((init_total + 7) / 8), 256, 0, st>>>(K, a.init_pos, d, mu, mu_bf16,
                                                                 norm2, mumax, status, init_total);
  RI_CUDA_TRY(cudaGetLastError());

  RI_CUDA_TRY(set_smem_once(reinterpret_cast<const void*>(assign_kernel), (int)kAssignSmem));
  const size_t upd_smem = align_up(g.seg_len * 2, 16) + kUpdateWarps * sizeof(MemberQueue);
  const int upd_smem_max = (int)(32768 * 2 + kUpdateWarps * sizeof(MemberQueue));
  RI_CUDA_TRY(set_smem_once(reinterpret_cast<const void*>(update_kernel), upd_smem_max));
  RI_CUDA_TRY(set_smem_once(reinterpret_cast<const void*>(finalise_kernel), upd_smem_max));
  const unsigned grid_assign =
      (unsigned)(d.total_tiles < (long long)num_sms() ? d.total_tiles : num_sms());
  const dim3 grid_upd((unsigned)units, (unsigned)((g.K_full + kClustersPerBlock - 1) /
                                                  kClustersPerBlock));
  const int rounds = g.iters > 0 ? g.iters : 1;
  for (int t = 0; t < rounds; ++t) {
    assign_kernel<<<grid_assign, kAssignThreads, kAssignSmem, st>>>(
        tm_keys, tm_cent, d, knorm, norm2, mumax, mu, labels, status);
    RI_CUDA_TRY(cudaGetLastError());
    RI_CUDA_TRY(cudaMemsetAsync(mumax, 0, units * sizeof(float), st));
    update_kernel<<<grid_upd, kUpdateWarps * 32, upd_smem, st>>>(
        K, labels, d, mu, mu_bf16, norm2, mumax, counts, g.iters > 0 ? 1 : 0);
    RI_CUDA_TRY(cudaGetLastError());
  }
  if (a.out.objective)
    RI_CUDA_TRY(cudaMemsetAsync(a.out.objective, 0, units * sizeof(float), st));
  finalise_kernel<<<grid_upd, kUpdateWarps * 32, upd_smem, st>>>(K, V, labels, d, mu,
                                                                  counts, a.out);
  RI_CUDA_TRY(cudaGetLastError());
  return RI_OK;
}

}  // namespace ri
