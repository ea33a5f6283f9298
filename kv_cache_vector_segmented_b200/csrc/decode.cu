// Tripartite decode attention over the wave index (sm_100a): one persistent,
// cooperative kernel launch per decode step, one block per SM.
//
// Steps (RetroInfer; "KV缓存技术与RetroInfer系统在长上下文推理中的优化实践",
// framerc.cn, §2.1 zones, §2.2 step 1 index query, §3.3 attention over the
// zones and merge of the partial results):
//   S1 centroid scoring   s[g][c] = q_g . centroid_c / sqrt(d), key r_c = sum_g s
//   S2 cluster selection  R = top k_r by (r desc, id asc), E = the next k_e
//   S4 exact partials     split-K flash decode over steady + R tokens
//   S5 estimation term    each c in E adds n_c e^{s} / e^{s} Vsum_c
//   S6 merge              log-sum-exp over the split partials
//
// A unit is one (sequence, KV head).  Work flows between blocks through
// per-unit counters in the workspace; no block ever waits for a block that
// could be waiting for it, and the cooperative launch keeps every block
// resident, so the waits below always end (they are bounded in any case).
//   A) Every block scores 128-centroid tiles t = blockIdx + k gridDim of the
//      flattened (unit, tile) list on the tensor cores: TMA brings the tile
//      and the unit's query rows (128-byte swizzle), one thread issues
//      tcgen05.mma (M = 128 centroids, N = 16 query rows, K = 128), four
//      warps read the fp32 scores from TMEM, store s and r and fold r into
//      the unit's key range; a fifth warp counts finished tiles per unit.
//   B) Block NB - 1 - u ranks unit u's C keys exactly once its tiles are all
//      scored (value histogram over the key range, exact order inside the
//      two boundary buckets), writes R and E in id order and the R clusters'
//      token prefix and first rows, then raises the unit's ready flag.
//   C) Every block takes (unit, slice) pairs: the unit's steady tokens, R
//      tokens and E clusters form one item list cut into S equal slices, and
//      each warp of the block a contiguous run of the slice.  A warp streams
//      its items through a private ring of shared-memory slots with 16-byte
//      cp.async copies (the ring's depth in flight) and folds each into one
//      online-softmax state: a token adds e^{x} v after its logit x, an E
//      cluster adds n_c e^{s} and e^{s} Vsum_c.  The block combines its warps
//      into the slice's partial (m, l, o) in the workspace.
//   D) The block that finishes a unit's last slice (atomic ticket) merges the
//      S partials by log-sum-exp and writes out and lse.
#include <float.h>
#include <math.h>
#include <string.h>

#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"
#include "internal.h"

namespace ri {

namespace {

constexpr float kScale = 0.08838834764831845f;  // 1/sqrt(128)
constexpr int kTileC = 128;          // centroids per MMA tile (M)
constexpr int kQRows = 16;           // MMA N: query rows (the unit's G, then others)
constexpr int kStagesA = 4;
constexpr uint32_t kTileBytes = kTileC * kHeadDim * 2;  // 32 KB
constexpr uint32_t kQBytes = kQRows * kHeadDim * 2;     // 4 KB
constexpr uint32_t kStageBytes = kTileBytes + kQBytes;  // 1024-byte multiple
constexpr int kNB = 2048;            // value buckets of the selection
constexpr int kBoundaryCap = 256;    // keys ranked exactly in a boundary bucket
constexpr int kRound = 8192;         // keys per selection round (all threads)
constexpr int kMaxWarps = 32;
constexpr int kRoundItems = 134;      // work items (token or E cluster) per copy round
constexpr uint32_t kBufBytes = 81920;  // one round: tokens (padded to 16) x 512 B + E x 548 B
constexpr uint32_t kRegionBytes = 2 * kBufBytes;
constexpr float kRescale = 8.f;      // online softmax: new reference only when the max
                                     // grows by more than this (terms stay <= e^8)
static_assert(kStagesA * kStageBytes <= kRegionBytes, "stages");
static_assert(16 * 512 + (kRoundItems - 1) * 548 <= (int)kBufBytes &&
                  (kRoundItems + 15) * 512 <= (int)kBufBytes, "round");

// Threads per block (registers: up to 128 each).
template <int G>
struct Shape {
  static constexpr int kThreads = 512;
  static constexpr int kWarps = kThreads / 32;
  static constexpr int kPer = kRound / kThreads;  // keys per thread and round
};

// Shared memory map (byte offsets from a 1024-byte aligned base).
constexpr uint32_t kOffRpre = kRegionBytes;                        // int [kMaxRetrieval + 4]
constexpr uint32_t kOffRrow = kOffRpre + (kMaxRetrieval + 4) * 4;  // int [kMaxRetrieval]
constexpr uint32_t kOffMisc = kOffRrow + kMaxRetrieval * 4;
constexpr uint32_t kMiscBytes = 3072;
constexpr uint32_t kSmemBytes = kOffMisc + kMiscBytes + 1024;  // + base alignment slack
static_assert(kSmemBytes <= 232448, "shared memory");
static_assert(kOffMisc % 16 == 0, "misc alignment");

// Selection scratch inside the region (free outside steps A and C).
constexpr uint32_t kOffHist = 0;
constexpr uint32_t kOffCand = kOffHist + kNB * 4;                // [2][kBoundaryCap] u64
constexpr uint32_t kOffSelCnt = kOffCand + 2 * kBoundaryCap * 8;  // int [kRound]
constexpr uint32_t kOffSelOff = kOffSelCnt + kRound * 4;          // int [kRound]
constexpr uint32_t kOffSelE = kOffSelOff + kRound * 4;            // int [kRound]
constexpr uint32_t kOffSelRid = kOffSelE + kRound * 4;            // int [kMaxRetrieval]
constexpr uint32_t kOffSelRcnt = kOffSelRid + kMaxRetrieval * 4;  // int [kMaxRetrieval]
static_assert(kOffSelRcnt + kMaxRetrieval * 4 <= kRegionBytes, "selection scratch");

enum Mode { kModeFull = 0, kModeSelect = 1, kModeAttend = 2 };

struct Params {
  const __nv_bfloat16* q;
  const int32_t* counts;
  const int32_t* offsets;
  const float* vsum;
  const __nv_bfloat16* Kr;  // retrieval rows: Kp (in place) or the execution buffer
  const __nv_bfloat16* Vr;
  const __nv_bfloat16* Ks;
  const __nv_bfloat16* Vs;
  __nv_bfloat16* out;
  float* lse;
  int32_t* sel_user;
  int32_t* rpre_user;
  float* score;    // ws [BH][C][8]
  float* rkey;     // ws [BH][C]
  int32_t* sel;    // ws [BH][k_r + k_e]
  int32_t* rpre;   // ws [BH][k_r + 1]
  int32_t* rrow;   // ws [BH][k_r]
  float* part;     // ws [BH][S][G][kPartStride]
  int* status;     // ws status word
  int* done;       // ws [BH] scored tiles
  int* ready;      // ws [BH] selection published
  int* ticket;     // ws [BH] finished slices
  uint32_t* kmax;  // ws [BH] max order key of the finite selection keys
  uint32_t* kmin;  // ws [BH] max of the complemented order keys (= min key)
  int* ninf;       // ws [BH] empty clusters (key -inf)
  int BH, C, M, n_steady, k_r, k_e, kr, ke, S, exec_rows, mode;
  int nbp;         // blocks that take attention slices (the rest are selectors)
};

struct Misc {
  uint64_t full[kStagesA], empty[kStagesA], tfull[2], tempty[2], drain;
  uint32_t tmem;
  int abort_flag;
  int epi_done;  // epilogue's finished tiles (step A)
  int flag;
  int bucket[2], above[2], ncand[2];
  uint32_t Tu[2];
  int Tid[2];
  int wtot[2][kMaxWarps];
  int scan[kMaxWarps + 4];
  float wm[kMaxWarps][8];  // per-warp partial maxima (block combine)
  float wl[kMaxWarps][8];  // per-warp partial denominators
};
static_assert(sizeof(Misc) <= kMiscBytes, "misc area");

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_acquire_cta(const int* p) {
  int v;
  asm volatile("ld.acquire.cta.shared.b32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_cta(int* p, int v) {
  asm volatile("st.release.cta.shared.b32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}
__device__ __forceinline__ int ld_volatile(const int* p) {
  return *reinterpret_cast<const volatile int*>(p);
}

__device__ __forceinline__ float float_from_order_key(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

// 64-bit selection order: larger key first, lower id first among equal keys.
__device__ __forceinline__ unsigned long long ord64(uint32_t u, int id) {
  return ((unsigned long long)u << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)id);
}

// Value bucket of a finite key (monotone in the key), -1 for -inf.
__device__ __forceinline__ int bucket_of(float r, float lo, float scale) {
  if (r == -INFINITY) return -1;
  int b = (int)((r - lo) * scale);
  return b < 0 ? 0 : (b >= kNB ? kNB - 1 : b);
}

// ---- warp-level tensor-core helpers (mma.sync m16n8k16, bf16 in, fp32 acc)
__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// d += A . B with A 16x16 row-major (regs a0..a3), B 16x8 column-major (b0, b1)
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0,
                                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
// 2^x by the hardware approximation (ex2.approx; -inf gives +0)
__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The k-th (1-based, from the top) key of value bucket b with its id, by an
// MSD radix walk over the bucket's keys (for crowded buckets: heavy ties).
template <int NT>
__device__ void kth_in_bucket_slow(const float* keys, int C, int b, float lo, float scale, int k,
                                   Misc* ms, int* hist, uint32_t* Tu, int* Tid) {
  constexpr int NW = NT / 32;
  uint32_t prefix = 0, mask = 0;
  int remaining = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += NT) hist[i] = 0;
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += NT) {
      const float r = __ldcg(keys + c);
      if (bucket_of(r, lo, scale) != b) continue;
      const uint32_t u = float_order_key(r);
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int cum = 0, dg = 255;
      for (; dg > 0; --dg) {
        if (cum + hist[dg] >= remaining) break;
        cum += hist[dg];
      }
      ms->scan[0] = dg;
      ms->scan[1] = remaining - cum;
    }
    __syncthreads();
    prefix |= (uint32_t)ms->scan[0] << shift;
    mask |= 255u << shift;
    remaining = ms->scan[1];
    __syncthreads();
  }
  // the remaining-th smallest id among the bucket's keys equal to prefix
  if (threadIdx.x == 0) ms->scan[2] = -1;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int run = 0;
  for (int base = 0; base < C; base += NT) {
    const int c = base + threadIdx.x;
    const float r = c < C ? __ldcg(keys + c) : 0.f;
    const bool eq = c < C && bucket_of(r, lo, scale) == b && float_order_key(r) == prefix;
    const unsigned mk = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) ms->wtot[0][warp] = __popc(mk);
    __syncthreads();
    int before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      before += w < warp ? ms->wtot[0][w] : 0;
      tot += ms->wtot[0][w];
    }
    const int rank = run + before + __popc(mk & ((1u << lane) - 1u));
    if (eq && rank == remaining - 1) ms->scan[2] = c;
    run += tot;
    __syncthreads();
  }
  *Tu = prefix;
  *Tid = ms->scan[2];
  __syncthreads();
}

// Block-wide exclusive prefix of one int per thread (thread order); the
// block total goes to *total.  One warp scans the per-warp totals.
template <int NT>
__device__ __forceinline__ int block_scan(int v, int* scratch /* [NT / 32 + 1] */, int* total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += t;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int wt = lane < NW ? scratch[lane] : 0;
    int wi = wt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += t;
    }
    if (lane < NW) scratch[lane] = wi - wt;
    if (lane == 31) scratch[NW] = wi;
  }
  __syncthreads();
  const int excl = scratch[warp] + incl - v;
  *total = scratch[NW];
  __syncthreads();  // scratch is reused by the next scan
  return excl;
}

// OR of a predicate over the 128 threads of warps 4-7 (named barrier 1).
__device__ __forceinline__ bool epilogue_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "barrier.red.or.pred q, 1, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)v)
      : "memory");
  return r != 0;
}

// Bounded wait of one thread until a counter other blocks raise reaches
// `target`; gives up early when any block has recorded a failure.
__device__ bool wait_count(const int* counter, int target, const int* status) {
  if (ld_acquire(counter) >= target) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    if (ld_acquire(counter) >= target) return true;
    if (ld_volatile(status) != 0) return false;
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
    __nanosleep(32);
  }
}

// ------------------------------------------------------------------ kernel
template <int G>
__global__ void __launch_bounds__(Shape<G>::kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tm_cent,
                  const __grid_constant__ CUtensorMap tm_q, const Params p) {
  constexpr int NT = Shape<G>::kThreads;
  constexpr int NW = Shape<G>::kWarps;
  constexpr int kPer = Shape<G>::kPer;

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  Misc* ms = reinterpret_cast<Misc*>(sm + kOffMisc);
  int32_t* rpre_sm = reinterpret_cast<int32_t*>(sm + kOffRpre);
  int32_t* rrow_sm = reinterpret_cast<int32_t*>(sm + kOffRrow);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int C = p.C;
  const int kr = p.kr, ke = p.ke;
  const int tiles_h = C > 0 ? (C + kTileC - 1) / kTileC : 0;

  if (threadIdx.x == 0) {
    ms->abort_flag = 0;
    ms->epi_done = 0;
    for (int i = 0; i < kStagesA; ++i) {
      mbar_init(&ms->full[i], 1);
      mbar_init(&ms->empty[i], 1);
    }
    for (int h = 0; h < 2; ++h) {
      mbar_init(&ms->tfull[h], 1);
      mbar_init(&ms->tempty[h], 128);
    }
    mbar_init(&ms->drain, 1);
    fence_barrier_init();
  }
  __syncthreads();

  // ============================================================ step A
  if (p.mode != kModeAttend && tiles_h > 0) {
    const int total_tiles = p.BH * tiles_h;
    const int nt = total_tiles > (int)blockIdx.x
                       ? (total_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1
                       : 0;
    if (nt > 0) {
      if (warp == 1) {
        tmem_alloc(&ms->tmem, 32);
        tmem_relinquish();
      }
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      const uint32_t tmem = ms->tmem;
      if (warp == 0 && lane == 0) {
        // TMA producer: centroid tile and the unit's query rows per stage
        tma_prefetch_desc(&tm_cent);
        tma_prefetch_desc(&tm_q);
        int issued[kStagesA] = {0, 0, 0, 0};
        for (int it = 0; it < nt; ++it) {
          if (ld_volatile(&ms->abort_flag)) break;
          const int st = it % kStagesA;
          if (it >= kStagesA && !mbar_wait(&ms->empty[st], ((it / kStagesA) - 1) & 1)) {
            record_status(p.status, RI_ERR_TIMEOUT);
            ms->abort_flag = 1;
            break;
          }
          const int t = (int)blockIdx.x + it * (int)gridDim.x;
          const int u = t / tiles_h, ti = t - u * tiles_h;
          uint8_t* stage = sm + st * kStageBytes;
          mbar_arrive_expect_tx(&ms->full[st], kStageBytes);
          const int row = u * C + ti * kTileC;
          for (int kh = 0; kh < 2; ++kh) {
            tma_load_2d(stage + kh * (kTileC * 128), &tm_cent, kh * 64, row, &ms->full[st]);
            tma_load_2d(stage + kTileBytes + kh * (kQRows * 128), &tm_q, kh * 64, u * G,
                        &ms->full[st]);
          }
          ++issued[st];
        }
        for (int st = 0; st < kStagesA; ++st)
          if (issued[st]) mbar_wait(&ms->full[st], (uint32_t)((issued[st] - 1) & 1));
      } else if (warp == 1 && lane == 0) {
        // MMA issuer: D[128 x 16] = tile[128 x 128] . Q[16 x 128]^T
        constexpr uint32_t idesc = umma_idesc_bf16_f32(kTileC, kQRows);
        const uint32_t base = smem_u32(sm);
        for (int it = 0; it < nt; ++it) {
          if (ld_volatile(&ms->abort_flag)) break;
          const int st = it % kStagesA, buf = it & 1;
          if (!mbar_wait(&ms->full[st], (uint32_t)((it / kStagesA) & 1)) ||
              (it >= 2 && !mbar_wait(&ms->tempty[buf], (uint32_t)(((it >> 1) - 1) & 1)))) {
            record_status(p.status, RI_ERR_TIMEOUT);
            ms->abort_flag = 1;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = base + st * kStageBytes;
          const uint32_t b_addr = a_addr + kTileBytes;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t aoff = (kk >> 2) * (kTileC * 128) + (kk & 3) * 32;
            const uint32_t boff = (kk >> 2) * (kQRows * 128) + (kk & 3) * 32;
            umma_bf16(tmem + buf * kQRows, umma_desc_sw128(a_addr + aoff),
                      umma_desc_sw128(b_addr + boff), idesc, kk > 0 ? 1u : 0u);
          }
          umma_commit(&ms->empty[st]);
          umma_commit(&ms->tfull[buf]);
        }
        umma_commit(&ms->drain);
        mbar_wait(&ms->drain, 0);
      } else if (warp == 2 && lane == 0) {
        // publisher: counts the epilogue's finished tiles into the units'
        // tile counters (one gpu-scope fence per batch of tiles)
        int published = 0;
        const unsigned long long t0 = globaltimer_ns();
        while (published < nt) {
          const int e = ld_acquire_cta(&ms->epi_done);
          if (e > published) {
            __threadfence();
            for (int i = published; i < e; ++i) {
              const int t = (int)blockIdx.x + i * (int)gridDim.x;
              atomicAdd(p.done + t / tiles_h, 1);
            }
            published = e;
          } else if (ld_volatile(&ms->abort_flag)) {
            break;
          } else if (globaltimer_ns() - t0 > kWaitLimitNs) {
            record_status(p.status, RI_ERR_TIMEOUT);
            ms->abort_flag = 1;
            break;
          }
        }
      } else if (warp >= 4 && warp < 8) {
        // epilogue: one centroid per thread; the unit's key range on the side
        const int quad = warp & 3;
        const int r = quad * 32 + lane;
        for (int it = 0; it < nt; ++it) {
          const int buf = it & 1;
          const int t = (int)blockIdx.x + it * (int)gridDim.x;
          const int u = t / tiles_h, ti = t - u * tiles_h;
          const int c = ti * kTileC + r;
          // issued before the wait so the load overlaps the MMA
          const int cnt = c < C ? __ldg(p.counts + (size_t)u * C + c) : 0;
          const bool ok = mbar_wait(&ms->tfull[buf], (uint32_t)((it >> 1) & 1));
          // the 128 epilogue threads leave together (they share named barrier 1)
          if (epilogue_any(!ok)) {
            if (!ok) record_status(p.status, RI_ERR_TIMEOUT);
            ms->abort_flag = 1;
            break;
          }
          tc_fence_after();
          float v[16];
          tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + buf * kQRows, v);
          tc_fence_before();
          mbar_arrive(&ms->tempty[buf]);
          uint32_t kmx = 0, kmn = 0;
          bool empty = false;
          if (c < C) {
            float s[8];
            float rs = 0.f;
#pragma unroll
            for (int g = 0; g < 8; ++g) {
              s[g] = g < G ? v[g] * kScale : 0.f;
              if (g < G) rs += s[g];
            }
            float4* dst = reinterpret_cast<float4*>(p.score + ((size_t)u * C + c) * 8);
            dst[0] = make_float4(s[0], s[1], s[2], s[3]);
            dst[1] = make_float4(s[4], s[5], s[6], s[7]);
            p.rkey[(size_t)u * C + c] = cnt > 0 ? rs : -INFINITY;
            if (cnt > 0) {
              kmx = float_order_key(rs);
              kmn = ~kmx;
            } else {
              empty = true;
            }
          }
          kmx = __reduce_max_sync(0xffffffffu, kmx);
          kmn = __reduce_max_sync(0xffffffffu, kmn);
          const int ne = __popc(__ballot_sync(0xffffffffu, empty));
          if (lane == 0) {
            if (kmx) atomicMax(p.kmax + u, kmx);
            if (kmn) atomicMax(p.kmin + u, kmn);
            if (ne) atomicAdd(p.ninf + u, ne);
          }
          asm volatile("bar.sync 1, 128;" ::: "memory");
          if (threadIdx.x == 128) st_release_cta(&ms->epi_done, it + 1);
        }
      }
      __syncwarp();
      tc_fence_before();
      __syncthreads();
      tc_fence_after();
      if (warp == 1) tmem_dealloc(tmem, 32);
    }
  }

  // ============================================================ step B
  // Exact selection over the C keys of unit u by this block alone.  Keys are
  // taken in rounds of kRound ids; thread t holds ids round_base + kPer t + j
  // in registers (16-byte loads).  The key range comes from step A.
  auto select_unit = [&](int u) {
    int* hist = reinterpret_cast<int*>(sm + kOffHist);        // [kNB]
    unsigned long long* cand = reinterpret_cast<unsigned long long*>(sm + kOffCand);
    int* cnt_sm = reinterpret_cast<int*>(sm + kOffSelCnt);    // [kRound] sizes of the round
    int* off_sm = reinterpret_cast<int*>(sm + kOffSelOff);    // [kRound] first rows of the round
    int* ecomp = reinterpret_cast<int*>(sm + kOffSelE);       // [kRound] E ids of the round
    int* rid_sm = reinterpret_cast<int*>(sm + kOffSelRid);    // [kMaxRetrieval] R ids
    int* rcnt_sm = reinterpret_cast<int*>(sm + kOffSelRcnt);  // [kMaxRetrieval] R sizes
    const float* rk = p.rkey + (size_t)u * C;
    const int32_t* cg = p.counts + (size_t)u * C;
    const int32_t* og = p.offsets + (size_t)u * (C + 1);
    const int rounds = (C + kRound - 1) / kRound;
    const bool vec = (C & 3) == 0;
    float kk[kPer];
    // keys of round rd into registers; sizes and first rows into shared memory
    auto load_round = [&](int rd, bool with_meta) {
      const int c0 = rd * kRound + threadIdx.x * kPer;
      if (vec && c0 + kPer <= C) {
#pragma unroll
        for (int i = 0; i < kPer; i += 4) {
          const float4 v = __ldcg(reinterpret_cast<const float4*>(rk + c0 + i));
          kk[i] = v.x;
          kk[i + 1] = v.y;
          kk[i + 2] = v.z;
          kk[i + 3] = v.w;
        }
        if (with_meta) {
          // every load issued before the first store (no load waits on a store)
          int4 cv[kPer / 4];
          int ov[kPer];
#pragma unroll
          for (int i = 0; i < kPer / 4; ++i) cv[i] = __ldg(reinterpret_cast<const int4*>(cg + c0) + i);
#pragma unroll
          for (int i = 0; i < kPer; ++i) ov[i] = __ldg(og + c0 + i);
#pragma unroll
          for (int i = 0; i < kPer / 4; ++i)
            *reinterpret_cast<int4*>(cnt_sm + threadIdx.x * kPer + 4 * i) = cv[i];
#pragma unroll
          for (int i = 0; i < kPer; ++i) off_sm[threadIdx.x * kPer + i] = ov[i];
        }
      } else {
        int cv[kPer], ov[kPer];
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
          const bool in = c0 + i < C;
          kk[i] = in ? __ldcg(rk + c0 + i) : 0.f;
          cv[i] = (with_meta && in) ? __ldg(cg + c0 + i) : 0;
          ov[i] = (with_meta && in) ? __ldg(og + c0 + i) : 0;
        }
        if (with_meta) {
#pragma unroll
          for (int i = 0; i < kPer; ++i) {
            cnt_sm[threadIdx.x * kPer + i] = cv[i];
            off_sm[threadIdx.x * kPer + i] = ov[i];
          }
        }
      }
    };
    load_round(0, false);
    for (int i = threadIdx.x; i < kNB; i += NT) hist[i] = 0;
    if (threadIdx.x < 2) ms->ncand[threadIdx.x] = 0;
    const uint32_t kmx = __ldcg(p.kmax + u), kmn = __ldcg(p.kmin + u);
    const int ninf = __ldcg(p.ninf + u);
    const int nfin = C - ninf;
    const float lo = nfin > 0 ? float_from_order_key(~kmn) : 0.f;
    const float hi = nfin > 0 ? float_from_order_key(kmx) : 0.f;
    const float scale = (nfin > 0 && hi > lo) ? (float)kNB / (hi - lo) : 0.f;
    __syncthreads();
    // 1) histogram over value buckets (monotone in the key)
    for (int rd = 0; rd < rounds; ++rd) {
      if (rd > 0) load_round(rd, false);
      const int c0 = rd * kRound + threadIdx.x * kPer;
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const int b = bucket_of(kk[j], lo, scale);
        if (c0 + j < C && b >= 0) atomicAdd(&hist[b], 1);
      }
    }
    __syncthreads();
    // 2) boundary buckets of ranks kr and kr + ke from the top: thread t
    //    owns kNB / NT consecutive buckets, the highest for t = 0
    {
      constexpr int BPT = kNB / NT;
      int hc[BPT];
      int sum = 0;
#pragma unroll
      for (int i = 0; i < BPT; ++i) {
        hc[i] = hist[kNB - 1 - BPT * threadIdx.x - i];
        sum += hc[i];
      }
      if (threadIdx.x < 2) {
        const int k = threadIdx.x == 0 ? kr : kr + ke;
        ms->bucket[threadIdx.x] = k <= 0 ? -2 : (k > nfin ? -1 : -3);
        ms->above[threadIdx.x] = k > nfin ? nfin : 0;
      }
      int total_fin;
      const int excl = block_scan<NT>(sum, ms->scan, &total_fin);
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const int k = w == 0 ? kr : kr + ke;
        if (k > 0 && k <= nfin && excl < k && excl + sum >= k) {
          int cum = excl;
#pragma unroll
          for (int i = 0; i < BPT; ++i) {
            if (cum + hc[i] >= k) {
              ms->bucket[w] = kNB - 1 - BPT * threadIdx.x - i;
              ms->above[w] = cum;
              break;
            }
            cum += hc[i];
          }
        }
      }
      __syncthreads();
    }
    // 3) exact order inside each boundary bucket: the members of both
    //    buckets are gathered (warp-aggregated slots) and sorted by
    //    (key desc, id asc): a warp-wide bitonic sort when <= 32, else ranking
    int bk[2];
    bool small[2];
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      bk[w] = ms->bucket[w];
      const int nb = bk[w] >= 0 ? hist[bk[w]] : (bk[w] == -1 ? ninf : 0);
      small[w] = bk[w] != -2 && nb <= kBoundaryCap;
    }
    if (small[0] || small[1]) {
      for (int rd = 0; rd < rounds; ++rd) {
        if (rounds > 1) load_round(rd, false);
        const int c0 = rd * kRound + threadIdx.x * kPer;
        uint32_t cm[2] = {0u, 0u};
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
          const int b = bucket_of(kk[j], lo, scale);
#pragma unroll
          for (int w = 0; w < 2; ++w)
            if (small[w] && b == bk[w] && c0 + j < C) cm[w] |= 1u << j;
        }
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if (!small[w]) continue;
          const int cnt = __popc(cm[w]);
          int incl = cnt;
#pragma unroll
          for (int off = 1; off < 32; off <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += t;
          }
          const int wtot = __shfl_sync(0xffffffffu, incl, 31);
          int base = 0;
          if (lane == 0 && wtot > 0) base = atomicAdd(&ms->ncand[w], wtot);
          base = __shfl_sync(0xffffffffu, base, 0) + incl - cnt;
          uint32_t m = cm[w];
          while (m) {
            const int j = __ffs(m) - 1;
            m &= m - 1;
            cand[w * kBoundaryCap + base++] = ord64(float_order_key(kk[j]), c0 + j);
          }
        }
      }
      __syncthreads();
      if (warp < 2 && small[warp]) {
        const int w = warp;
        const int k = (w == 0 ? kr : kr + ke) - ms->above[w];  // 1-based rank in the bucket
        const int n = ms->ncand[w];
        if (n <= 32) {
          unsigned long long v = lane < n ? cand[w * kBoundaryCap + lane] : 0ull;
#pragma unroll
          for (int kb = 2; kb <= 32; kb <<= 1)
#pragma unroll
            for (int jb = kb >> 1; jb > 0; jb >>= 1) {
              const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, jb);
              const bool keep_max = ((lane & jb) == 0) == ((lane & kb) == 0);
              v = keep_max ? (v > o ? v : o) : (v < o ? v : o);
            }
          if (lane == k - 1) {
            ms->Tu[w] = (uint32_t)(v >> 32);
            ms->Tid[w] = (int)(0xFFFFFFFFu - (uint32_t)(v & 0xFFFFFFFFull));
          }
        } else {
          for (int i = lane; i < n; i += 32) {
            const unsigned long long me = cand[w * kBoundaryCap + i];
            int rank = 0;
            for (int t = 0; t < n; ++t) rank += cand[w * kBoundaryCap + t] > me;
            if (rank == k - 1) {
              ms->Tu[w] = (uint32_t)(me >> 32);
              ms->Tid[w] = (int)(0xFFFFFFFFu - (uint32_t)(me & 0xFFFFFFFFull));
            }
          }
        }
      }
    }
    for (int w = 0; w < 2; ++w) {
      if (bk[w] == -2 || small[w]) continue;
      uint32_t Tu;
      int Tid;
      const int k = (w == 0 ? kr : kr + ke) - ms->above[w];
      kth_in_bucket_slow<NT>(rk, C, bk[w], lo, scale, k, ms, hist, &Tu, &Tid);
      if (threadIdx.x == 0) {
        ms->Tu[w] = Tu;
        ms->Tid[w] = Tid;
      }
    }
    __syncthreads();
    const bool selA = bk[0] != -2, selB = bk[1] != -2;
    const uint32_t TuA = ms->Tu[0], TuB = ms->Tu[1];
    const int TidA = ms->Tid[0], TidB = ms->Tid[1];
    // 4) membership (order key, then id) and compaction in id order: R ids,
    //    sizes and first rows to shared memory, E ids per round to shared
    //    memory and then out in coalesced stores
    int32_t* selg = p.sel + (size_t)u * (p.k_r + p.k_e);
    int32_t* selu = p.sel_user ? p.sel_user + (size_t)u * (p.k_r + p.k_e) : nullptr;
    int baseR = 0, baseE = 0;
    for (int rd = 0; rd < rounds; ++rd) {
      if (rounds > 1) {
        __syncthreads();  // previous round's E ids are written out
        load_round(rd, false);
      }
      const int c0 = rd * kRound + threadIdx.x * kPer;
      uint32_t mR = 0, mE = 0;
#pragma unroll
      for (int j = 0; j < kPer; ++j) {
        const uint32_t o = float_order_key(kk[j]);
        const int c = c0 + j;
        const bool inR = c < C && selA && (o > TuA || (o == TuA && c <= TidA));
        const bool inE = c < C && !inR && selB && (o > TuB || (o == TuB && c <= TidB));
        mR |= (uint32_t)inR << j;
        mE |= (uint32_t)inE << j;
      }
      int tot;
      const int excl = block_scan<NT>((__popc(mR) << 16) | __popc(mE), ms->scan, &tot);
      int pr = baseR + (excl >> 16), pe = excl & 0xFFFF;
      while (mR) {
        const int j = __ffs(mR) - 1;
        mR &= mR - 1;
        rid_sm[pr] = c0 + j;
        ++pr;
      }
      while (mE) {
        const int j = __ffs(mE) - 1;
        mE &= mE - 1;
        ecomp[pe++] = c0 + j;
      }
      __syncthreads();
      const int nE = tot & 0xFFFF;
      for (int i = threadIdx.x; i < nE; i += NT) {
        selg[p.k_r + baseE + i] = ecomp[i];
        if (selu) selu[p.k_r + baseE + i] = ecomp[i];
      }
      baseR += tot >> 16;
      baseE += nE;
    }
    for (int i = threadIdx.x; i < p.k_r; i += NT) {
      const int v = i < kr ? rid_sm[i] : -1;
      selg[i] = v;
      if (selu) selu[i] = v;
    }
    for (int i = ke + threadIdx.x; i < p.k_e; i += NT) {
      selg[p.k_r + i] = -1;
      if (selu) selu[p.k_r + i] = -1;
    }
    // 5) R token prefix (execution-buffer rows) and first rows, id order:
    //    sizes and first rows of the R clusters gathered (loads issued
    //    together), then one block scan
    {
      constexpr int kPerR = kMaxRetrieval / NT;
      const int per = (kr + NT - 1) / NT;
      const int i0 = min(kr, (int)threadIdx.x * per), i1 = min(kr, i0 + per);
      int cn[kPerR], of[kPerR];
#pragma unroll
      for (int w = 0; w < kPerR; ++w) {
        const int i = i0 + w;
        const int c = i < i1 ? rid_sm[i] : 0;
        cn[w] = i < i1 ? __ldg(cg + c) : 0;
        of[w] = i < i1 ? __ldg(og + c) : 0;
      }
      int loc = 0;
#pragma unroll
      for (int w = 0; w < kPerR; ++w) {
        const int i = i0 + w;
        if (i < i1) {
          rcnt_sm[i] = cn[w];
          rrow_sm[i] = of[w];
        }
        loc += cn[w];
      }
      int total;
      int run = block_scan<NT>(loc, ms->scan, &total);
      int32_t* rp = p.rpre + (size_t)u * (p.k_r + 1);
      int32_t* rr = p.rrow + (size_t)u * (p.k_r > 0 ? p.k_r : 1);
      int32_t* ru = p.rpre_user ? p.rpre_user + (size_t)u * (p.k_r + 1) : nullptr;
      for (int i = i0; i < i1; ++i) {
        rp[i] = run;
        if (ru) ru[i] = run;
        run += rcnt_sm[i];
      }
      for (int i = threadIdx.x; i < kr; i += NT) rr[i] = rrow_sm[i];
      for (int i = kr + threadIdx.x; i <= p.k_r; i += NT) {
        rp[i] = total;
        if (ru) ru[i] = total;
      }
    }
    // 6) publish: one fence after the block barrier covers the block's stores
    __syncthreads();
    if (threadIdx.x == 0) {
      __threadfence();
      st_release(p.ready + u, 1);
    }
  };

  // Unit u is selected by block NB - 1 - (u mod NB) once its tiles are all
  // scored (the blocks at the end of the grid score the fewest tiles).
  if (p.mode != kModeAttend && tiles_h > 0) {
    for (int u = (int)gridDim.x - 1 - (int)blockIdx.x; u < p.BH; u += (int)gridDim.x) {
      if (threadIdx.x == 0) {
        const bool ok = wait_count(p.done + u, tiles_h, p.status);
        if (!ok) record_status(p.status, RI_ERR_TIMEOUT);
        ms->flag = ok;
      }
      __syncthreads();
      if (!ms->flag) break;
      __threadfence();
      select_unit(u);
    }
  }
  if (p.mode == kModeSelect) return;

  // ============================================================ step C
  const int npairs = p.BH * p.S;
  const bool exec = p.exec_rows > 0;
  const long long lim_rows = exec ? p.exec_rows : p.M;
  const long long row_base_stride = exec ? p.exec_rows : p.M;
  const int gid = lane >> 2, tig = lane & 3;  // mma fragment coordinates
  for (int pi = blockIdx.x; pi < npairs && (int)blockIdx.x < p.nbp; pi += p.nbp) {
    const int u = pi % p.BH, s = pi / p.BH;
    if (p.mode == kModeFull && tiles_h > 0) {
      if (threadIdx.x == 0) {
        const bool ok = wait_count(p.ready + u, 1, p.status);
        if (!ok) record_status(p.status, RI_ERR_TIMEOUT);
        ms->flag = ok;
      }
      __syncthreads();
      if (!ms->flag) break;
    }
    // the unit's R prefix and first rows, coalesced into shared memory
    if (C > 0) {
      const int32_t* rpg = p.rpre + (size_t)u * (p.k_r + 1);
      const int32_t* rrg = p.rrow + (size_t)u * (p.k_r > 0 ? p.k_r : 1);
      for (int i0 = 0; i0 <= kr; i0 += 4 * NT) {
        int a[4], b[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int i = i0 + j * NT + threadIdx.x;
          a[j] = i <= kr ? __ldcg(rpg + i) : 0;
          b[j] = (!exec && i < kr) ? __ldcg(rrg + i) : 0;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int i = i0 + j * NT + threadIdx.x;
          if (i <= kr) rpre_sm[i] = a[j];
          if (i < kr) rrow_sm[i] = b[j];
        }
      }
    } else if (threadIdx.x == 0) {
      rpre_sm[0] = 0;
    }
    // A fragments of Q (rows = query heads, padded to 16 with zeros):
    // qa[kk][0] = Q[gid][16 kk + 2 tig ..], qa[kk][1] = Q[gid][16 kk + 8 + 2 tig ..]
    uint32_t qa[8][2];
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      if (gid < G) {
        const __nv_bfloat16* qr = p.q + ((size_t)u * G + gid) * kHeadDim + kk * 16 + tig * 2;
        qa[kk][0] = *reinterpret_cast<const uint32_t*>(qr);
        qa[kk][1] = *reinterpret_cast<const uint32_t*>(qr + 8);
      } else {
        qa[kk][0] = qa[kk][1] = 0u;
      }
    }
    __syncthreads();
    const int n_st = p.n_steady;
    const int T_R = C > 0 ? rpre_sm[kr] : 0;
    const long long W = (long long)n_st + T_R + ke;
    const long long w0 = W * s / p.S, w1 = W * (s + 1) / p.S;
    const int tok_end = n_st + T_R;  // items below are tokens, above E clusters
    const int nrounds = (int)((w1 - w0 + kRoundItems - 1) / kRoundItems);
    struct Round {
      int ta, ntok, npad, ea, ne;
      uint32_t off_v, off_ev, off_es, off_en;
    };
    auto round_of = [&](int r) {
      const long long a = w0 + (long long)r * kRoundItems;
      const long long b = min(w1, a + kRoundItems);
      Round rd;
      rd.ta = (int)min(a, (long long)tok_end);
      rd.ntok = (int)min(b, (long long)tok_end) - rd.ta;
      rd.npad = (rd.ntok + 15) & ~15;
      rd.ea = (int)(max(a, (long long)tok_end) - tok_end);
      rd.ne = (int)(max(b, (long long)tok_end) - tok_end) - rd.ea;
      rd.off_v = rd.npad * 256;
      rd.off_ev = 2 * rd.npad * 256;
      rd.off_es = rd.off_ev + rd.ne * 512;
      rd.off_en = rd.off_es + rd.ne * 32;
      return rd;
    };
    // 16-byte chunk c of token row t, XOR-swizzled for conflict-free ldmatrix
    auto row_chunk = [](int t, int c) { return (uint32_t)(t * 256 + ((c ^ (t & 7)) << 4)); };

    // ---- copies of round r into buffer r & 1, issued by every warp: warp w
    // takes items [n w / NW, n (w + 1) / NW) of the round; one cp.async group
    // per thread and round.  Token rows: lanes 0-15 copy K, 16-31 copy V.
    auto issue = [&](int r) {
      const Round rd = round_of(r);
      uint8_t* buf = sm + (r & 1) * kBufBytes;
      const int n = rd.ntok + rd.ne;
      const int j0 = n * warp / NW, j1 = n * (warp + 1) / NW;
      // tokens of this warp
      const int t0 = min(j0, rd.ntok), t1 = min(j1, rd.ntok);
      if (t1 > t0) {
        int ci = 0;
        const int first_r = rd.ta + t0 - n_st;  // R index of the first token (if any)
        if (!exec && rd.ta + t1 > n_st && kr > 0) {
          const int r0 = max(first_r, 0);
          int lo = 0, hi = kr - 1;  // last cluster with rpre <= r0
          while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (rpre_sm[mid] <= r0) lo = mid; else hi = mid - 1;
          }
          ci = lo;
        }
        for (int t = t0; t < t1; ++t) {
          const int it = rd.ta + t;
          const __nv_bfloat16* src = nullptr;
          if (it < n_st) {
            src = (lane < 16 ? p.Ks : p.Vs) + ((size_t)u * n_st + it) * kHeadDim;
          } else {
            const int rpos = it - n_st;
            long long row;
            if (exec) {
              row = rpos;
            } else {
              while (ci + 1 < kr && rpre_sm[ci + 1] <= rpos) ++ci;
              row = (long long)rrow_sm[ci] + (rpos - rpre_sm[ci]);
            }
            if (row >= 0 && row < lim_rows)
              src = (lane < 16 ? p.Kr : p.Vr) + ((size_t)u * row_base_stride + row) * kHeadDim;
          }
          const int c = lane & 15;
          uint8_t* dst = buf + (lane < 16 ? 0u : rd.off_v) + row_chunk(t, c);
          if (src) {
            cp_async16(dst, src + c * 8);
          } else {
            *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
            if (lane == 0) record_status(p.status, RI_ERR_INVALID_ARG);
          }
        }
      }
      // padding rows of the last token tile (zeros: no NaN into the MMA)
      if (warp == NW - 1)
        for (int i = lane; i < (rd.npad - rd.ntok) * 32; i += 32) {
          const int t = rd.ntok + (i >> 5), c = i & 15;
          *reinterpret_cast<uint4*>(buf + ((i & 16) ? rd.off_v : 0u) + row_chunk(t, c)) =
              make_uint4(0, 0, 0, 0);
        }
      // E clusters of this warp
      const int e0 = max(j0, rd.ntok) - rd.ntok, e1 = max(j1, rd.ntok) - rd.ntok;
      for (int eb = e0; eb < e1; eb += 32) {
        const int ne = min(32, e1 - eb);
        int idv = -1;
        if (lane < ne) idv = __ldcg(p.sel + (size_t)u * (p.k_r + p.k_e) + p.k_r + rd.ea + eb + lane);
        for (int i = 0; i < ne; ++i) {
          const int c = __shfl_sync(0xffffffffu, idv, i);
          const int e = eb + i;
          if (c >= 0 && c < C) {
            const size_t uc = (size_t)u * C + c;
            cp_async16(buf + rd.off_ev + e * 512 + lane * 16, p.vsum + uc * kHeadDim + lane * 4);
            if (lane < 2) cp_async16(buf + rd.off_es + e * 32 + lane * 16, p.score + uc * 8 + lane * 4);
            if (lane == 2) cp_async4(buf + rd.off_en + e * 4, p.counts + uc);
          } else if (lane == 0) {
            *reinterpret_cast<int*>(buf + rd.off_en + e * 4) = 0;
            record_status(p.status, RI_ERR_INVALID_ARG);
          }
        }
      }
      cp_async_commit();
    };

    // ---- state.  Tokens (tensor cores): O^T[d][g] fragments, lane holds
    // d = 16 j + gid (+8), g = 2 tig (+1); running max / sum of row g = gid
    // in log2 units.  E clusters (CUDA cores): lane owns dims 4 lane .. +3.
    float ot[8][4];
    float tm = -INFINITY, tl = 0.f;
    float ea[G][4], em[G], el[G];
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i) ot[j][i] = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      em[g] = -INFINITY;
      el[g] = 0.f;
#pragma unroll
      for (int i = 0; i < 4; ++i) ea[g][i] = 0.f;
    }
    constexpr float kScale2 = kScale * 1.4426950408889634f;  // to log2 units
    constexpr float kLog2e = 1.4426950408889634f;
    for (int r = 0; r < 2 && r < nrounds; ++r) issue(r);
    for (int r = 0; r < nrounds; ++r) {
      const Round rd = round_of(r);
      const uint8_t* buf = sm + (r & 1) * kBufBytes;
      if (r + 1 < nrounds) cp_async_wait<1>(); else cp_async_wait<0>();
      __syncthreads();
      // token tiles of 16: tile j on warp j % NW
      const int ntiles = rd.npad >> 4;
      for (int tj = warp; tj < ntiles; tj += NW) {
        const uint32_t kbase = smem_u32(buf) + tj * 16 * 256;
        const uint32_t vbase = smem_u32(buf + rd.off_v) + tj * 16 * 256;
        // S = Q K^T for tokens 16 tj .. +15: two n-tiles of 8 tokens
        float sacc[2][4];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int i = 0; i < 4; ++i) sacc[h][i] = 0.f;
#pragma unroll
        for (int kp = 0; kp < 4; ++kp) {  // dims 32 kp .. 32 kp + 31
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            // matrices: (tokens 8h.., dim chunk 4kp + m) for m = 0..3
            const int tr = h * 8 + (lane & 7), ch = kp * 4 + (lane >> 3);
            uint32_t b[4];
            ldmatrix_x4(b, kbase + row_chunk(tr, ch));
            mma_bf16_16816(sacc[h], qa[2 * kp][0], 0u, qa[2 * kp][1], 0u, b[0], b[1]);
            mma_bf16_16816(sacc[h], qa[2 * kp + 1][0], 0u, qa[2 * kp + 1][1], 0u, b[2], b[3]);
          }
        }
        // row g = gid: logits of tokens 8h + 2 tig (+1); mask the padding
        float x[4];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int t = tj * 16 + h * 8 + tig * 2 + i;
            x[h * 2 + i] = t < rd.ntok ? sacc[h][i] * kScale2 : -INFINITY;
          }
        float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        float corr = 1.f;
        if (mx > tm + kRescale * kLog2e) {  // new reference (also the first tile)
          corr = tm == -INFINITY ? 0.f : ex2f(tm - mx);
          tm = mx;
          tl *= corr;
        }
        // O^T columns g = 2 tig, 2 tig + 1 rescale by the factors of rows g
        if (__any_sync(0xffffffffu, corr != 1.f)) {
          const float c0 = __shfl_sync(0xffffffffu, corr, (tig * 2) * 4);
          const float c1 = __shfl_sync(0xffffffffu, corr, (tig * 2 + 1) * 4);
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            ot[j][0] *= c0;
            ot[j][1] *= c1;
            ot[j][2] *= c0;
            ot[j][3] *= c1;
          }
        }
        float pv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          pv[i] = ex2f(x[i] - tm);
          tl += pv[i];
        }
        const uint32_t pb0 = pack_bf16x2(pv[0], pv[1]);  // tokens 2 tig, +1
        const uint32_t pb1 = pack_bf16x2(pv[2], pv[3]);  // tokens 8 + 2 tig, +1
        // O^T += V^T P^T: 8 dim groups of 16
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          // matrices: (tokens 8 (m >> 1).., dim chunk 2 j + (m & 1)) for m = 0..3
          const int m4 = lane >> 3;
          const int tr = (m4 >> 1) * 8 + (lane & 7), ch = j * 2 + (m4 & 1);
          uint32_t a[4];
          ldmatrix_x4_trans(a, vbase + row_chunk(tr, ch));
          mma_bf16_16816(ot[j], a[0], a[1], a[2], a[3], pb0, pb1);
        }
      }
      // E clusters: cluster e on warp e % NW, lane owns dims 4 lane .. 4 lane + 3
      for (int e = warp; e < rd.ne; e += NW) {
        const int n = *reinterpret_cast<const int*>(buf + rd.off_en + e * 4);
        if (n <= 0) continue;
        const float4 v = *reinterpret_cast<const float4*>(buf + rd.off_ev + e * 512 + lane * 16);
        const float* sc = reinterpret_cast<const float*>(buf + rd.off_es + e * 32);
        const float nf = (float)n;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float sg = sc[g] * kLog2e;
          if (sg > em[g] + kRescale * kLog2e) {
            const float c = em[g] == -INFINITY ? 0.f : ex2f(em[g] - sg);
            el[g] *= c;
#pragma unroll
            for (int i = 0; i < 4; ++i) ea[g][i] *= c;
            em[g] = sg;
          }
          const float w = ex2f(sg - em[g]);
          el[g] = fmaf(nf, w, el[g]);
          ea[g][0] = fmaf(w, v.x, ea[g][0]);
          ea[g][1] = fmaf(w, v.y, ea[g][1]);
          ea[g][2] = fmaf(w, v.z, ea[g][2]);
          ea[g][3] = fmaf(w, v.w, ea[g][3]);
        }
      }
      __syncthreads();  // buffer r & 1 is free again
      if (r + 2 < nrounds) issue(r + 2);
    }
    // ---- warp state -> shared memory: per head g the warp's reference
    // maximum (natural log), denominator and numerator [128]
    __syncthreads();
    float* red = reinterpret_cast<float*>(sm);  // [NW][G][128]
    {
      tl += __shfl_xor_sync(0xffffffffu, tl, 1);
      tl += __shfl_xor_sync(0xffffffffu, tl, 2);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float mtg = __shfl_sync(0xffffffffu, tm, g * 4);
        const float ltg = __shfl_sync(0xffffffffu, tl, g * 4);
        const float mw = fmaxf(mtg, em[g]);
        const float ft = mtg == -INFINITY ? 0.f : ex2f(mtg - mw);
        const float fe = em[g] == -INFINITY ? 0.f : ex2f(em[g] - mw);
        if (lane == 0) {
          ms->wm[warp][g] = mw == -INFINITY ? -INFINITY : mw * 0.6931471805599453f;
          ms->wl[warp][g] = ltg * ft + el[g] * fe;
        }
        float4* rw = reinterpret_cast<float4*>(red + ((size_t)warp * G + g) * kHeadDim + lane * 4);
        *rw = make_float4(ea[g][0] * fe, ea[g][1] * fe, ea[g][2] * fe, ea[g][3] * fe);
      }
      __syncwarp();
      // token numerators: lane holds O^T[16 j + gid (+8)][2 tig (+1)]
      float ftv[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int g = tig * 2 + k;
        const float mtg = __shfl_sync(0xffffffffu, tm, (g < 8 ? g : 0) * 4);
        float emg = -INFINITY;
#pragma unroll
        for (int gg = 0; gg < G; ++gg)
          if (gg == g) emg = em[gg];
        const float mw = fmaxf(mtg, emg);
        ftv[k] = (g < G && mtg != -INFINITY) ? ex2f(mtg - mw) : 0.f;
      }
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int g = tig * 2 + k;
          if (g < G) {
            float* rg = red + ((size_t)warp * G + g) * kHeadDim + j * 16 + gid;
            rg[0] += ot[j][k] * ftv[k];
            rg[8] += ot[j][2 + k] * ftv[k];
          }
        }
    }
    __syncthreads();
    float* part = p.part + ((size_t)u * p.S + s) * G * kPartStride;
    // warp g: the block maximum of head g and the warps' factors (in wm)
    if (warp < G) {
      const int g = warp;
      const float wmv = lane < NW ? ms->wm[lane][g] : -INFINITY;
      float mb = wmv;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, off));
      const float f = (wmv == -INFINITY) ? 0.f : __expf(wmv - mb);
      float lw = lane < NW ? f * ms->wl[lane][g] : 0.f;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, off);
      __syncwarp();
      if (lane < NW) ms->wm[lane][g] = f;
      if (lane == 0) {
        part[(size_t)g * kPartStride + 0] = mb;
        part[(size_t)g * kPartStride + 1] = lw;
      }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * kHeadDim; idx += NT) {
      const int g = idx / kHeadDim, d = idx - g * kHeadDim;
      float a = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) a = fmaf(ms->wm[w][g], red[((size_t)w * G + g) * kHeadDim + d], a);
      part[(size_t)g * kPartStride + 4 + d] = a;
    }
    // ============================================================ step D
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) ms->flag = atomicAdd(p.ticket + u, 1) == p.S - 1;
    __syncthreads();
    if (ms->flag) {
      // the last slice of unit u merges the S partials (log-sum-exp)
      __threadfence();
      const float* pu = p.part + (size_t)u * p.S * G * kPartStride;
      float* fq = reinterpret_cast<float*>(sm);  // [S][G] maxima, then weights
      float* tot = fq + p.S * G;                 // [G] max, [G] denominator
      if (warp < G) {
        // warp g: the slices' maxima and denominators of query head g
        const int g = warp;
        float mx = -INFINITY;
        for (int q = lane; q < p.S; q += 32) {
          const float m = __ldcg(pu + ((size_t)q * G + g) * kPartStride);
          fq[q * G + g] = m;
          mx = fmaxf(mx, m);
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        float ls = 0.f;
        for (int q = lane; q < p.S; q += 32) {
          const float m = fq[q * G + g];
          const float f = (mx == -INFINITY || m == -INFINITY) ? 0.f : __expf(m - mx);
          fq[q * G + g] = f;
          ls = fmaf(__ldcg(pu + ((size_t)q * G + g) * kPartStride + 1), f, ls);
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
        if (lane == 0) {
          tot[g] = mx;
          tot[G + g] = ls;
        }
      }
      __syncthreads();
      for (int idx = threadIdx.x; idx < G * kHeadDim; idx += NT) {
        const int g = idx / kHeadDim, d = idx - g * kHeadDim;
        float os = 0.f;
        for (int q0 = 0; q0 < p.S; q0 += 16) {
          float v[16];
#pragma unroll
          for (int k = 0; k < 16; ++k)
            v[k] = q0 + k < p.S ? __ldcg(pu + ((size_t)(q0 + k) * G + g) * kPartStride + 4 + d)
                                : 0.f;
#pragma unroll
          for (int k = 0; k < 16; ++k)
            if (q0 + k < p.S) os = fmaf(fq[(q0 + k) * G + g], v[k], os);
        }
        const float ls = tot[G + g];
        // no token and no cluster contributed (empty steady zone and budgets): 0, lse -inf
        const bool any = ls > 0.f;
        const size_t hq = (size_t)u * G + g;
        p.out[hq * kHeadDim + d] = __float2bfloat16_rn(any ? os / ls : 0.f);
        if (p.lse && d == 0) p.lse[hq] = any ? tot[g] + logf(ls) : -INFINITY;
      }
    }
    __syncthreads();  // the region is reused by the next pair's copies
  }
}

// ------------------------------------------------------------------ host
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// bf16 [rows][128] row-major, boxes of 64 columns x box_rows, 128-byte swizzle
cudaError_t encode_rows(CUtensorMap* map, const void* base, unsigned long long rows,
                        unsigned box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  if (fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  return cudaSuccess;
}

template <int G>
cudaError_t prepare_kernel() {
  return set_smem_once(reinterpret_cast<const void*>(decode_kernel<G>), (int)kSmemBytes);
}

template <int G>
int blocks_per_sm() {
  int n = 0;
  if (prepare_kernel<G>() != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_kernel<G>, Shape<G>::kThreads,
                                                    kSmemBytes) != cudaSuccess)
    n = 0;
  cudaGetLastError();
  return n;
}

int blocks_per_sm_g(int G) {
  switch (G) {
    case 1: return blocks_per_sm<1>();
    case 2: return blocks_per_sm<2>();
    case 3: return blocks_per_sm<3>();
    case 4: return blocks_per_sm<4>();
    case 5: return blocks_per_sm<5>();
    case 6: return blocks_per_sm<6>();
    case 7: return blocks_per_sm<7>();
    default: return blocks_per_sm<8>();
  }
}

template <int G>
cudaError_t launch_g(const Geometry& g, const DecodeLayout& L, const DecodeArgs& a, int mode,
                     cudaStream_t s) {
  Params p;
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.counts = a.counts;
  p.offsets = a.offsets;
  p.vsum = a.vsum;
  const bool exec = a.exec_K != nullptr;
  p.Kr = static_cast<const __nv_bfloat16*>(exec ? a.exec_K : a.Kp);
  p.Vr = static_cast<const __nv_bfloat16*>(exec ? a.exec_V : a.Vp);
  p.Ks = static_cast<const __nv_bfloat16*>(a.Ks);
  p.Vs = static_cast<const __nv_bfloat16*>(a.Vs);
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.lse = a.lse;
  p.sel_user = a.sel_user;
  p.rpre_user = a.rpre_user;
  p.score = reinterpret_cast<float*>(a.ws + L.off_score);
  p.rkey = reinterpret_cast<float*>(a.ws + L.off_rkey);
  p.sel = reinterpret_cast<int32_t*>(a.ws + L.off_sel);
  p.rpre = reinterpret_cast<int32_t*>(a.ws + L.off_rpre);
  p.rrow = reinterpret_cast<int32_t*>(a.ws + L.off_rrow);
  p.part = reinterpret_cast<float*>(a.ws + L.off_part);
  p.status = reinterpret_cast<int*>(a.ws);
  const long long BH = g.BH();
  p.done = reinterpret_cast<int*>(a.ws + L.off_ctrl);
  p.ready = p.done + BH;
  p.ticket = p.ready + BH;
  p.kmax = reinterpret_cast<uint32_t*>(p.ticket + BH);
  p.kmin = p.kmax + BH;
  p.ninf = reinterpret_cast<int*>(p.kmin + BH);
  p.nbp = L.NBP;
  p.BH = (int)BH;
  p.C = g.C;
  p.M = g.M;
  p.n_steady = g.n_steady;
  p.k_r = L.k_r;
  p.k_e = L.k_e;
  p.kr = L.kr;
  p.ke = L.ke;
  p.S = L.S;
  p.exec_rows = exec ? a.exec_rows : 0;
  p.mode = mode;

  CUtensorMap map_c, map_q;
  memset(&map_c, 0, sizeof(map_c));
  memset(&map_q, 0, sizeof(map_q));
  if (g.C > 0 && mode != kModeAttend) {
    cudaError_t e = encode_rows(&map_c, a.centroid, (unsigned long long)BH * g.C, kTileC);
    if (e == cudaSuccess) e = encode_rows(&map_q, a.q, (unsigned long long)BH * G, kQRows);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = prepare_kernel<G>();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)L.NB);
  cfg.blockDim = dim3(Shape<G>::kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_kernel<G>, map_c, map_q, p);
}

cudaError_t launch_mode(const Geometry& g, const DecodeLayout& L, const DecodeArgs& a, int mode,
                        cudaStream_t s) {
  switch (g.G) {
    case 1: return launch_g<1>(g, L, a, mode, s);
    case 2: return launch_g<2>(g, L, a, mode, s);
    case 3: return launch_g<3>(g, L, a, mode, s);
    case 4: return launch_g<4>(g, L, a, mode, s);
    case 5: return launch_g<5>(g, L, a, mode, s);
    case 6: return launch_g<6>(g, L, a, mode, s);
    case 7: return launch_g<7>(g, L, a, mode, s);
    default: return launch_g<8>(g, L, a, mode, s);
  }
}

}  // namespace

// Launch shape of the decode kernel: one block per SM (NB), and S slices of
// the attention work per unit.  S is the smallest count whose makespan
// (ceil(units x S / NB') slices of 1/S of a unit per block) is within 5 % of
// the best over S <= 64, with at least ~32 items per slice; NB' leaves the
// selector blocks free when units <= NB / 2.
bool decode_plan(const Geometry& g, DecodeLayout* L) {
  int nb = 148;
  int dev = -1;
  if (cudaGetDevice(&dev) == cudaSuccess) {
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess &&
        sms > 0) {
      static std::mutex mu;
      static std::map<std::pair<int, int>, int> cache;
      int per;
      {
        std::lock_guard<std::mutex> lk(mu);
        auto key = std::make_pair(dev, g.G);
        auto it = cache.find(key);
        if (it == cache.end()) it = cache.emplace(key, blocks_per_sm_g(g.G)).first;
        per = it->second;
      }
      if (per < 1) {
        set_error("decode kernel cannot be resident on this device");
        return false;
      }
      nb = sms;  // one block per SM
    }
  }
  cudaGetLastError();
  const long long units = g.BH();
  const double avg_r = g.C > 0 ? (double)L->kr * g.M / g.C : 0.0;
  const double w_est = g.n_steady + avg_r + L->ke;
  int s_max = (int)(w_est / 32.0);
  s_max = s_max < 1 ? 1 : (s_max > 64 ? 64 : s_max);
  // with few units the selector blocks (the last `units` blocks) take no slices
  const long long nbp = units <= nb / 2 ? nb - units : nb;
  auto makespan = [&](int S) {
    return (double)((units * S + nbp - 1) / nbp) / (double)S;
  };
  double best = 1e30;
  for (int S = 1; S <= s_max; ++S) best = best < makespan(S) ? best : makespan(S);
  int S = 1;
  while (S < s_max && makespan(S) > 1.05 * best) ++S;
  L->NB = nb;
  L->NBP = (int)nbp;
  L->S = S;
  return true;
}

cudaError_t launch_select(const Geometry& g, const DecodeLayout& L, const DecodeArgs& a,
                          cudaStream_t s) {
  return launch_mode(g, L, a, kModeSelect, s);
}

cudaError_t launch_attend(const Geometry& g, const DecodeLayout& L, const DecodeArgs& a,
                          cudaStream_t s) {
  return launch_mode(g, L, a, kModeAttend, s);
}

cudaError_t launch_decode(const Geometry& g, const DecodeLayout& L, const DecodeArgs& a,
                          cudaStream_t s) {
  return launch_mode(g, L, a, kModeFull, s);
}

// ------------------------------------------------------------------- self-test
__global__ void wait_timeout_kernel(int* status, unsigned long long limit_ns) {
  // Waits for status[1] to become nonzero; nothing sets it.
  volatile int* flag = status + 1;
  const unsigned long long t0 = globaltimer_ns();
  while (*flag == 0) {
    if (globaltimer_ns() - t0 > limit_ns) {
      record_status(status, RI_ERR_TIMEOUT);
      return;
    }
  }
}

cudaError_t launch_wait_timeout_selftest(int* status, unsigned long long limit_ns,
                                         cudaStream_t s) {
  wait_timeout_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace ri
