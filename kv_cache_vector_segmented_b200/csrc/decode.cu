// Tripartite decode attention over the wave index (sm_100a): one thread-block
// cluster per unit (one sequence and KV head), one block per SM.
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
// The CS blocks of a cluster share one unit.  Block b owns the unit's
// 128-centroid tiles b, b + CS, b + 2 CS, ... (dealt round-robin, so the
// blocks' shares differ by at most one tile); the blocks exchange data only
// through distributed shared memory and the cluster barrier, never through
// global counters, so no block waits on another cluster.  Data a block
// needs from the others is pushed into its shared memory before the barrier
// that publishes it wherever possible (a remote load costs a round trip
// after the barrier; a remote store does not).
//   A) Scoring: TMA brings the block's centroid tiles (128-byte swizzle, a
//      ring of 4 stages) and the unit's query rows once; one thread issues
//      tcgen05.mma (M = 128 centroids, N = 16 query rows, K = 128), each tile
//      into its own TMEM columns; four epilogue warps read the fp32 scores,
//      keep the keys r_c in shared memory and write the per-head scores s
//      to the workspace (the estimation term reads them back).  Eight other
//      warps load the clusters' sizes and first rows meanwhile.
//   B) Selection, exact, cluster-wide: the key range (barrier 1), each
//      block's histogram of its own keys over 4096 value buckets with its
//      sums over groups of 32 buckets counted alongside, the group sums
//      pushed to every block (barrier 2); every block finds the two boundary
//      groups (ranks k_r and k_r + k_e from the top), reads those groups' 32
//      bucket counts from every block and finds the boundary buckets.  The
//      members of a boundary bucket are ranked exactly by (key desc, id
//      asc): pushed to every block when there are few of them (barrier 3)
//      and ranked by one warp per boundary, else found by a radix walk over
//      the 32-bit order key and a final id count (crowded buckets, heavy
//      ties).  Each block lists its own R clusters (first row, token prefix)
//      and E clusters (id, size) in id order; when the selection is written
//      out, every block pushes its per-tile counts (barrier 4) and places its
//      ids by the prefixes over all tiles.
//   C) Attention: each block attends over the clusters it scored (its own
//      R and E lists) and an even share of the steady tokens.  Warps 0-7
//      take the token rows in windows: 16-row K and V tiles copied with
//      16-byte cp.async (two whole rows per instruction) into an
//      XOR-swizzled layout, S = Q K^T and O^T += V^T P^T on
//      mma.sync.m16n8k16 bf16 tiles (ldmatrix / ldmatrix.trans, the query
//      rows padded to 16).  Warps 8-15 fold the E clusters four at a time
//      on the tensor cores (mma.sync.m16n8k4, TF32 value sums and weights,
//      fp32 sums; the denominator n_c e^s in fp32 on CUDA cores), each warp
//      streaming value sums and scores through its own ring of slots.  Both
//      keep an online softmax in log2 units, rescaled only when the maximum
//      grows by more than e^8.  After a separate select call, the attend
//      call rebuilds the same lists by the same tile ownership, so both
//      paths fold the same items in the same order.
//   D) Merge: the block's warps are combined in shared memory; block 0
//      releases its ring with a remote mbarrier arrive and the other blocks
//      store their partials (max, denominator, numerator) into it with
//      st.async, whose bytes complete an mbarrier of block 0; block 0 merges
//      them by log-sum-exp into out and lse.  A last cluster barrier, whose
//      arrivals come early, keeps every block alive until the remote arrives
//      have landed.
// Launches go out with programmatic dependent launch: a launch sets up its
// barriers and tensor memory while the launch before it finishes and waits
// for it (griddepcontrol.wait) before its first global access.
// A growing index (index maintenance during decode) is read through
// separate per-unit strides: Cs clusters and Ms rows, of which the first C
// clusters are live.
// Every wait on an mbarrier is bounded; on expiry the block records
// RI_ERR_TIMEOUT in the status word, stops issuing work, lets the copies it
// issued land and still takes part in every cluster barrier.
#include <float.h>
#include <limits.h>
#include <math.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace ri {

namespace {

constexpr float kScale = 0.08838834764831845f;  // 1/sqrt(128)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescale2 = 8.f * kLog2e;  // online softmax: new reference only when the
                                           // maximum grows by more than e^8

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;

constexpr int kTileC = 128;  // centroids per MMA tile (M)
constexpr int kQRows = 16;   // MMA N: the unit's query rows, then padding
constexpr uint32_t kTileBytes = kTileC * kHeadDim * 2;  // 32 KB
constexpr uint32_t kQBytes = kQRows * kHeadDim * 2;     // 4 KB
constexpr int kStagesA = 4;
constexpr int kMaxTilesPerBlock = kMaxIdsPerBlock / kTileC;  // 32
constexpr int kMaxCS = kMaxClusterBlocks;

constexpr int kNB = 4096;  // value buckets of the selection histogram
constexpr int kGroups = kNB / 32;
constexpr int kCand = 256;  // boundary-bucket members ranked directly
constexpr int kKPT = kMaxIdsPerBlock / kThreads;  // own ids per thread (contiguous)

// Step C: warps 0..7 fold the tokens in tiles of 16 on the tensor cores
// (double-buffered, 16 KB each), warps 8..15 the estimation clusters on CUDA
// cores; the token rows of up to kWindowTokens tokens are planned at a time.
constexpr int kTokenWarps = 8;
constexpr int kEWarps = kWarps - kTokenWarps;
constexpr uint32_t kTokenWarpBytes = 16384;
constexpr int kWindowTokens = 1024;
// estimation warps: rings of kESlots slots (value sum 512 B + scores 32 B)
// in the size-and-row area of step A, free by then, and the area after it
constexpr uint32_t kSlotE = 544;
constexpr uint32_t kEWarpBytes = 6912;
constexpr int kESlots = (int)(kEWarpBytes / kSlotE);

// Shared memory map (byte offsets from a 1024-byte aligned base).
constexpr uint32_t kRingBytes = kTokenWarps * kTokenWarpBytes;  // 128 KB
static_assert(kStagesA * kTileBytes == kRingBytes, "ring");
constexpr uint32_t kOffQ = kRingBytes;                          // q tile (4 KB)
constexpr uint32_t kOffKeys = kOffQ + kQBytes;                  // float keys[P], then lists
constexpr uint32_t kOffMeta = kOffKeys + kMaxIdsPerBlock * 8;   // int2 (first row, size)[P]
constexpr uint32_t kERingBytes = kEWarps * kEWarpBytes;  // from kOffMeta, step C
static_assert(kERingBytes >= kMaxIdsPerBlock * 8, "estimation rings cover the meta area");
constexpr uint32_t kOffRuns = kOffMeta + kERingBytes;          // int token rows[kWindowTokens]
constexpr uint32_t kOffMisc = kOffRuns + kWindowTokens * 4;
constexpr uint32_t kMiscBytes = 4096;
constexpr uint32_t kSmemBytes = kOffMisc + kMiscBytes + 1024;  // + base alignment slack
static_assert(kSmemBytes <= 232448, "shared memory");

// Inside the ring between steps A and C.
constexpr uint32_t kRHist = 0;                          // int [kNB] own histogram
constexpr uint32_t kRDig = kRHist + kNB * 4;            // int [4 passes][2][256] digit slices
constexpr uint32_t kRGin = kRDig + 4 * 2 * 256 * 4;     // int [kMaxCS][kGroups] pushed group sums
constexpr uint32_t kRCin = kRGin + kMaxCS * kGroups * 4;  // u64 [2][kMaxCS][kCand] pushed members
constexpr uint32_t kRAll = kRCin + 2 * kMaxCS * kCand * 8;  // u64 [2][kCand] gathered members
constexpr uint32_t kRRid = kRAll + 2 * kCand * 8;       // u16 [P] own R clusters (local index)
constexpr uint32_t kRLgs = kRRid + kMaxIdsPerBlock * 2;  // int [kGroups] own group sums
constexpr uint32_t kRTin = kRLgs + kGroups * 4;  // int [2][512] pushed per-tile equal-key counts
constexpr uint32_t kRTcnt = kRTin + 2 * 512 * 4;  // int4 [512] pushed per-tile list counts
static_assert(kRTcnt + 512 * 16 <= kRingBytes, "selection scratch");

enum Mode { kModeFull = 0, kModeSelect = 1, kModeAttend = 2 };

// Phase timestamps for profiling builds (-DRI_DEBUG_PHASES): %globaltimer of
// phase boundaries per block; nothing is recorded in normal builds.
#ifdef RI_DEBUG_PHASES
constexpr int kStampBlocks = 4096, kStamps = 64;
__device__ unsigned long long g_phase_ns[kStampBlocks][kStamps];
// stamps are kept in shared memory (Misc::stamps) and written out at the
// block's exit, so no global store sits between two phases
#define RI_STAMP(i, t)                                          \
  do {                                                          \
    if (threadIdx.x == (t)) ms->stamps[(i)] = globaltimer_ns(); \
  } while (0)
#define RI_STAMP_VAL(i, t, v)                                          \
  do {                                                                 \
    if (threadIdx.x == (t)) ms->stamps[(i)] = (unsigned long long)(v); \
  } while (0)
#define RI_STAMP_DUMP()                                                        \
  do {                                                                         \
    __syncthreads();                                                           \
    if (threadIdx.x < kStamps && blockIdx.x < kStampBlocks)                    \
      g_phase_ns[blockIdx.x][threadIdx.x] = ms->stamps[threadIdx.x];           \
  } while (0)
#else
#define RI_STAMP(i, t) \
  do {                 \
  } while (0)
#define RI_STAMP_VAL(i, t, v) \
  do {                        \
  } while (0)
#define RI_STAMP_DUMP() \
  do {                  \
  } while (0)
#endif

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
  float* score;   // ws [BH][Cs][Gp]
  int32_t* sel;   // ws [BH][k_r + k_e]
  int32_t* rpre;  // ws [BH][k_r + 1]
  int* status;
  unsigned long long wait_ns;
  int fault;
  int BH, C, Cs, Ms, n_steady, k_r, k_e, kr, ke, tiles, exec_rows, mode;
};

struct Misc {
  uint64_t fullA[kStagesA], emptyA[kStagesA], tdone[kMaxTilesPerBlock], qbar, drain, metabar;
  uint64_t go;   // step D: completed by block 0 once its ring takes partials
  uint64_t mrg;  // step D, block 0: completed by the bytes of the other partials
  uint32_t tmem;
  int abort_flag;
  uint32_t own_kmax, own_kmin;  // this block's key range (order keys) and empty clusters
  int own_ninf;
  int own_ncand[2];
  int own_nR, own_nE, own_tokR;
  int pub_tid[2];
  // pushed by every block of the cluster (slot = the sender's rank)
  uint4 rng_in[kMaxCS];   // (max key, max complemented key, empty clusters, 0)
  int candn_in[2][kMaxCS];
  // cluster-wide values
  int nRp[kMaxCS + 1], nEp[kMaxCS + 1], tokRp[kMaxCS + 1];
  int candp[2][kMaxCS + 1];
  float lo, scale;
  int nfin, ninf;
  int bucket[2], above[2], nmem[2], kp[2], slow[2], digit[2], owner[2];
  unsigned long long thr[2];
  int gsum[kGroups];  // cluster-wide group counts
  int fine[2][32];    // cluster-wide bucket counts of the two boundary groups
  alignas(16) int scan[2 * kWarps];
#ifdef RI_DEBUG_PHASES
  unsigned long long stamps[kStamps];
#endif
  float wm[kWarps][8], wl[kWarps][8];
};
static_assert(sizeof(Misc) <= kMiscBytes, "misc area");

// ---------------------------------------------------------------- helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_nrank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
// Cluster barrier in its .aligned form (whole warps); several call sites
// follow per-thread loops, so each call first reconverges the warp.
__device__ __forceinline__ void cluster_arrive() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  __syncwarp();
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_sync() {
  cluster_arrive();
  cluster_wait();
}
// Arrival that orders none of the thread's memory accesses.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
// Address of the same shared-memory location in block `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ uint32_t ld_cl_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ int4 ld_cl_v4(uint32_t addr) {
  int4 v;
  asm volatile("ld.shared::cluster.v4.s32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void st_cl_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_cl_u64(uint32_t addr, unsigned long long v) {
  asm volatile("st.shared::cluster.u64 [%0], %1;" ::"r"(addr), "l"(v) : "memory");
}
__device__ __forceinline__ void st_cl_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
// Store into another block's shared memory whose bytes complete on an
// mbarrier of that block (both addresses from mapa).
__device__ __forceinline__ void st_async_v4(uint32_t addr, float4 v, uint32_t bar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, [%5];" ::
          "r"(addr),
      "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void st_async_v2(uint32_t addr, float a, float b, uint32_t bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::
                   "r"(addr),
               "f"(a), "f"(b), "r"(bar)
               : "memory");
}
// Arrive (release, cluster scope) on an mbarrier of another block.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Bounded wait with acquire at cluster scope (data or arrivals from other
// blocks of the cluster).
__device__ __forceinline__ bool mbar_wait_cl(uint64_t* bar, uint32_t parity,
                                             unsigned long long limit_ns) {
  auto probe = [&]() {
    uint32_t ok;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
  };
  if (probe()) return true;
  const unsigned long long t0 = globaltimer_ns();
  while (true) {
    if (probe()) return true;
    if (globaltimer_ns() - t0 > limit_ns) return false;
  }
}
__device__ __forceinline__ void red_cl_add(uint32_t addr, uint32_t v) {
  asm volatile("red.shared::cluster.add.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
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

// 2^x by the hardware approximation (ex2.approx; -inf gives +0)
__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Exclusive prefix sum over the block's threads (thread order) and the
// total, with one barrier: each warp scans its lanes and publishes its total
// in scratch[warp]; after the barrier every thread adds up the totals of the
// warps before it.  The scratch array is read after the barrier, so the
// caller separates two uses of one array by a barrier of its own.
__device__ __forceinline__ int block_scan(int v, int* scratch /* [kWarps] */, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += t;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w4 = 0; w4 < kWarps / 4; ++w4) {
    const int4 t = reinterpret_cast<const int4*>(scratch)[w4];
    before += (4 * w4 < warp ? t.x : 0) + (4 * w4 + 1 < warp ? t.y : 0) +
              (4 * w4 + 2 < warp ? t.z : 0) + (4 * w4 + 3 < warp ? t.w : 0);
    all += t.x + t.y + t.z + t.w;
  }
  *total = all;
  return before + incl - v;
}

// Two prefix sums at once (scratch [2 * kWarps]), one barrier.
__device__ __forceinline__ int2 block_scan2(int a, int b, int* scratch, int2* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int ia = a, ib = b;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int ta = __shfl_up_sync(0xffffffffu, ia, off);
    const int tb = __shfl_up_sync(0xffffffffu, ib, off);
    if (lane >= off) {
      ia += ta;
      ib += tb;
    }
  }
  if (lane == 31) reinterpret_cast<int2*>(scratch)[warp] = make_int2(ia, ib);
  __syncthreads();
  int2 before = make_int2(0, 0), all = make_int2(0, 0);
#pragma unroll
  for (int w2 = 0; w2 < kWarps / 2; ++w2) {
    const int4 t = reinterpret_cast<const int4*>(scratch)[w2];  // warps 2 w2, 2 w2 + 1
    if (2 * w2 < warp) {
      before.x += t.x;
      before.y += t.y;
    }
    if (2 * w2 + 1 < warp) {
      before.x += t.z;
      before.y += t.w;
    }
    all.x += t.x + t.z;
    all.y += t.y + t.w;
  }
  *total = all;
  return make_int2(before.x + ia - a, before.y + ib - b);
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

// Bounded wait on an mbarrier phase; the waiting thread is suspended in
// hardware between probes (it resumes as soon as the phase completes), so
// waiting warps leave the issue slots to the warps doing the work.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity,
                                         unsigned long long lim) {
  return mbar_wait_suspend(bar, parity, 20000u, lim);
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
// D += A B on the tensor cores, m16n8k4, TF32 inputs, fp32 accumulation:
// A rows gid, gid + 8 at column tig (a0, a1), B row tig at column gid (b0).
__device__ __forceinline__ void mma_tf32_1684(float (&d)[4], uint32_t a0, uint32_t a1,
                                              uint32_t b0) {
  asm volatile(
      "mma.sync.aligned.m16n8k4.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(b0));
}
__device__ __forceinline__ uint32_t tf32_rn(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}
// 16-byte global -> shared copy; with fill == false the 16 bytes are zeroed
// and nothing is read.
__device__ __forceinline__ void cp_async16_zfill(void* smem, const void* gmem, bool fill) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(smem)), "l"(gmem),
               "r"(fill ? 16 : 0)
               : "memory");
}
// Barrier of the token warps only (named barrier 2, 256 threads).
__device__ __forceinline__ void token_bar() {
  asm volatile("bar.sync 2, 256;" ::: "memory");
}

// Thresholds of the boundary buckets holding more than kCand keys (heavy
// ties): an MSD radix walk over the 32-bit order key, one byte per pass with
// the digit counts reduced into their owner blocks, then the boundary id
// among the keys equal to the key found (per-block counts in id order).
// Called by every thread of every block of the cluster (cluster barriers).
__device__ __noinline__ void crowded_thresholds(const float* keys, int nid, float lo, float scale,
                                                int bk0, int bk1, bool slow0, bool slow1,
                                                Misc* ms, uint32_t dig_a, const int* tin,
                                                uint32_t tin_a, int CS, int b, int ntl,
                                                int tiles, int* status) {
  const int tid = threadIdx.x;
  const int DS = (256 + CS - 1) / CS;
      RI_STAMP(16, 0);
      uint32_t prefix[2] = {0u, 0u}, mask[2] = {0u, 0u};
      int kp[2] = {ms->kp[0], ms->kp[1]};
      for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = tid; i < nid; i += kThreads) {
          const float key = keys[i];
          const int bk = bucket_of(key, lo, scale);
          const uint32_t o = float_order_key(key);
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            if ((w == 0 ? slow0 : slow1) && bk == (w == 0 ? bk0 : bk1) &&
                (o & mask[w]) == prefix[w]) {
              const int d = (int)((o >> shift) & 255u);
              red_cl_add(mapa(dig_a + 4u * (uint32_t)((pass * 2 + w) * 256 + d % DS),
                              (uint32_t)(d / DS)),
                         1u);
            }
          }
        }
        cluster_sync();  // digit counts of this pass complete
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if (!(w == 0 ? slow0 : slow1)) continue;
          const int d = 255 - tid;  // thread order = digits from the top
          int v = 0;
          if (tid < 256)
            v = (int)ld_cl_u32(mapa(dig_a + 4u * (uint32_t)((pass * 2 + w) * 256 + d % DS),
                                    (uint32_t)(d / DS)));
          int tot;
          const int excl = block_scan(v, ms->scan, &tot);
          if (tid < 256 && excl < kp[w] && excl + v >= kp[w]) {
            ms->digit[w] = d;
            ms->above[w] = excl;
          }
          __syncthreads();
          prefix[w] |= (uint32_t)ms->digit[w] << shift;
          mask[w] |= 255u << shift;
          kp[w] -= ms->above[w];
          __syncthreads();
        }
      }
      // members equal to the found key, counted per tile (tiles are in id
      // order and dealt round-robin to the blocks): every block pushes its
      // tiles' counts to every block, a scan over the tiles finds the tile
      // holding the kp-th one, and the block owning that tile names its id
      if (tid < 64) ms->fine[tid >> 5][tid & 31] = 0;
      if (tid < 2) ms->owner[tid] = -1;
      __syncthreads();
      for (int i = tid; i < nid; i += kThreads) {
        const float key = keys[i];
        const int bk = bucket_of(key, lo, scale);
        const uint32_t o = float_order_key(key);
#pragma unroll
        for (int w = 0; w < 2; ++w)
          if ((w == 0 ? slow0 : slow1) && bk == (w == 0 ? bk0 : bk1) && o == prefix[w])
            atomicAdd(&ms->fine[w][i >> 7], 1);
      }
      __syncthreads();
      for (int t = tid; t < CS * ntl * 2; t += kThreads) {
        const int q = t / (ntl * 2), r = t - q * (ntl * 2);
        const int w = r / ntl, lt = r - w * ntl;
        st_cl_u32(mapa(tin_a + 4u * (uint32_t)(w * 512 + b + lt * CS), (uint32_t)q),
                  (uint32_t)ms->fine[w][lt]);
      }
      cluster_sync();  // every tile's count of equal keys pushed
#pragma unroll 1
      for (int w = 0; w < 2; ++w) {
        if (!(w == 0 ? slow0 : slow1)) continue;
        const int v = tid < tiles ? tin[w * 512 + tid] : 0;
        int tot;
        const int excl = block_scan(v, ms->scan, &tot);
        if (tid < tiles && excl < kp[w] && excl + v >= kp[w]) {
          ms->owner[w] = tid;
          ms->candp[w][0] = excl;  // equal keys in earlier tiles
        }
        __syncthreads();
      }
      if (tid < 2 && (tid == 0 ? slow0 : slow1)) {
        const int w = tid, tile = ms->owner[w];
        if (tile >= 0 && tile % CS == b) {
          const int lt = (tile - b) / CS;
          const int r = kp[w] - ms->candp[w][0];  // 1-based inside the tile
          int seen = 0;
          for (int i = lt * kTileC; i < min(nid, (lt + 1) * kTileC); ++i) {
            const float key = keys[i];
            if (bucket_of(key, lo, scale) == (w == 0 ? bk0 : bk1) &&
                float_order_key(key) == prefix[w] && ++seen == r) {
              ms->pub_tid[w] = tile * kTileC + (i & (kTileC - 1));
              break;
            }
          }
        }
      }
      cluster_sync();  // the boundary ids named
      if (tid < 2 && (tid == 0 ? slow0 : slow1)) {
        const int w = tid;
        const int tile = ms->owner[w];
        const int id = tile >= 0 ? (int)ld_cl_u32(mapa(smem_u32(&ms->pub_tid[w]),
                                                       (uint32_t)(tile % CS)))
                                 : -1;
        ms->thr[w] = ord64(prefix[w], id);
        if (tile < 0 || id < 0) record_status(status, RI_ERR_INVALID_ARG);
      }
      __syncthreads();
    }

// ------------------------------------------------------------------ kernel
template <int G>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tm_cent,
                  const __grid_constant__ CUtensorMap tm_q, const Params p) {
  constexpr int Gp = G <= 4 ? 4 : 8;        // scores stored per cluster
  constexpr uint32_t kPartStride = (kHeadDim + 4) * 4;  // step D: a head's partial in block 0
  constexpr uint32_t kPartBytes = G * (kHeadDim + 2) * 4;  // bytes of a block partial sent

  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  Misc* ms = reinterpret_cast<Misc*>(sm + kOffMisc);
  float* keys = reinterpret_cast<float*>(sm + kOffKeys);
  int2* lists = reinterpret_cast<int2*>(sm + kOffKeys);
  int2* meta = reinterpret_cast<int2*>(sm + kOffMeta);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int CS = (int)cluster_nrank();
  const int b = (int)cluster_rank();
  const int u = (int)blockIdx.x / CS;
  const int C = p.C, Cs = p.Cs;  // live clusters, per-unit stride
  const unsigned long long lim = p.wait_ns;
  const bool selecting = p.mode != kModeAttend && C > 0;
  // this block's tiles: b, b + CS, b + 2 CS, ... of the unit's ceil(C / 128)
  // tiles (interleaved, so that relevant clusters crowded into a few
  // segments still spread over the blocks); local id i is cluster id_of(i)
  const int ntiles = (selecting && b < p.tiles) ? (p.tiles - 1 - b) / CS + 1 : 0;
  const bool has_last = ntiles > 0 && (p.tiles - 1 - b) % CS == 0;
  const int nid = ntiles * kTileC - (has_last ? p.tiles * kTileC - C : 0);
  auto id_of = [&](int i) { return (b + (i >> 7) * CS) * kTileC + (i & (kTileC - 1)); };
  const uint32_t sm_base = smem_u32(sm);

#ifdef RI_DEBUG_PHASES
  if (tid < kStamps) ms->stamps[tid] = 0ull;
#endif
  if (tid == 0) {
    ms->abort_flag = 0;
    ms->own_kmax = ms->own_kmin = 0u;
    ms->own_ninf = 0;
    ms->own_ncand[0] = ms->own_ncand[1] = 0;
    ms->pub_tid[0] = ms->pub_tid[1] = -1;
    ms->own_nR = ms->own_nE = ms->own_tokR = 0;
    ms->thr[0] = ms->thr[1] = 0ull;
    for (int i = 0; i < kStagesA; ++i) {
      mbar_init(&ms->fullA[i], 1);
      mbar_init(&ms->emptyA[i], 1);
    }
    for (int i = 0; i < kMaxTilesPerBlock; ++i) mbar_init(&ms->tdone[i], 1);
    mbar_init(&ms->qbar, 1);
    mbar_init(&ms->drain, 1);
    mbar_init(&ms->metabar, 8);
    mbar_init(&ms->go, 1);
    mbar_init(&ms->mrg, 1);
    fence_barrier_init();
    // block 0 takes the other blocks' partials in step D
    if (b == 0) mbar_arrive_expect_tx(&ms->mrg, (uint32_t)(CS - 1) * kPartBytes);
  }
  // tensor memory for step A's accumulators (a column group per tile),
  // before the wait on the launch this one follows
  uint32_t ncols = 32;
  while (ncols < (uint32_t)ntiles * kQRows) ncols <<= 1;
  if (ntiles > 0 && warp == 1) {
    tmem_alloc(&ms->tmem, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // 0: the block has started (waited on before the first remote access)
  cluster_arrive();
  // a launch that follows this one may start its own set-up now; this one
  // touches no global memory before the launch it follows has completed
  // (both are no-ops without a programmatic dependency)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  RI_STAMP(0, 0);
  if (p.mode != kModeSelect && tid == 32 * 3 && p.n_steady > 0) {
    // this block's share of the steady rows into L2 (read in step C)
    const int s0 = p.n_steady * b / CS, s1 = p.n_steady * (b + 1) / CS;
    if (s1 > s0) {
      const size_t r0 = (size_t)u * p.n_steady + s0;
      prefetch_l2_bulk(p.Ks + r0 * kHeadDim, (uint32_t)(s1 - s0) * 256u);
      prefetch_l2_bulk(p.Vs + r0 * kHeadDim, (uint32_t)(s1 - s0) * 256u);
    }
  }

  // ============================================================ step A
  if (ntiles > 0) {
    const uint32_t tmem = ms->tmem;
    if (warp == 0 && lane == 0) {
      // TMA producer: the unit's query rows once, then the block's tiles
      tma_prefetch_desc(&tm_cent);
      tma_prefetch_desc(&tm_q);
      mbar_arrive_expect_tx(&ms->qbar, kQBytes);
      tma_load_2d(sm + kOffQ, &tm_q, 0, u * G, &ms->qbar);
      tma_load_2d(sm + kOffQ + kQRows * 128, &tm_q, 64, u * G, &ms->qbar);
      int issued[kStagesA] = {0, 0, 0, 0};
      for (int it = 0; it < ntiles; ++it) {
        if (ld_volatile(&ms->abort_flag)) break;
        const int st = it % kStagesA;
        if (it >= kStagesA && !wait_bar(&ms->emptyA[st], ((it / kStagesA) - 1) & 1, lim)) {
          record_status(p.status, RI_ERR_TIMEOUT);
          ms->abort_flag = 1;
          break;
        }
        uint8_t* stage = sm + st * kTileBytes;
        mbar_arrive_expect_tx(&ms->fullA[st], kTileBytes);
        const int row = u * Cs + (b + it * CS) * kTileC;
        if (!(p.fault == RI_FAULT_SCORE_COPY && it == 0)) {
          tma_load_2d(stage, &tm_cent, 0, row, &ms->fullA[st]);
          tma_load_2d(stage + kTileC * 128, &tm_cent, 64, row, &ms->fullA[st]);
        }
        ++issued[st];
      }
      // every copy issued lands before its stage is reused or the block exits
      for (int st = 0; st < kStagesA; ++st)
        if (issued[st]) wait_bar(&ms->fullA[st], (uint32_t)((issued[st] - 1) & 1), lim);
      wait_bar(&ms->qbar, 0, lim);
    } else if (warp == 1 && lane == 0) {
      // MMA issuer: D[128 x 16] = tile[128 x 128] . Q[16 x 128]^T per tile
      constexpr uint32_t idesc = umma_idesc_bf16_f32(kTileC, kQRows);
      const uint32_t qaddr = sm_base + kOffQ;
      bool ok = wait_bar(&ms->qbar, 0, lim);
      if (!ok) {
        record_status(p.status, RI_ERR_TIMEOUT);
        ms->abort_flag = 1;
      }
      for (int it = 0; ok && it < ntiles; ++it) {
        if (ld_volatile(&ms->abort_flag)) break;
        const int st = it % kStagesA;
        if (!wait_bar(&ms->fullA[st], (uint32_t)((it / kStagesA) & 1), lim)) {
          record_status(p.status, RI_ERR_TIMEOUT);
          ms->abort_flag = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = sm_base + st * kTileBytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = (kk >> 2) * (kTileC * 128) + (kk & 3) * 32;
          const uint32_t boff = (kk >> 2) * (kQRows * 128) + (kk & 3) * 32;
          umma_bf16(tmem + it * kQRows, umma_desc_sw128(a_addr + aoff),
                    umma_desc_sw128(qaddr + boff), idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&ms->emptyA[st]);
        if (!(p.fault == RI_FAULT_SCORE_COMMIT && it == 0)) umma_commit(&ms->tdone[it]);
      }
      // the MMAs issued have completed before TMEM is released
      umma_commit(&ms->drain);
      if (!wait_bar(&ms->drain, 0, lim)) {
        record_status(p.status, RI_ERR_TIMEOUT);
        ms->abort_flag = 1;
      }
    } else if (warp >= 8) {
      // sizes and first rows of the block's clusters, all loads in flight at
      // once while the tiles arrive
      const int32_t* cg = p.counts + (size_t)u * Cs;
      const int32_t* og = p.offsets + (size_t)u * (Cs + 1);
      for (int i0 = tid - 256; i0 < nid; i0 += 4 * 256) {
        int cv[4], ov[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int i = i0 + r * 256;
          cv[r] = i < nid ? __ldg(cg + id_of(i)) : 0;
          ov[r] = i < nid ? __ldg(og + id_of(i)) : 0;
        }
#pragma unroll
        for (int r = 0; r < 4; ++r)
          if (i0 + r * 256 < nid) meta[i0 + r * 256] = make_int2(ov[r], cv[r]);
      }
      __syncwarp();
      if (lane == 0 && p.fault != RI_FAULT_SCORE_SIZES) mbar_arrive(&ms->metabar);
    } else if (warp >= 4 && warp < 8) {
      // epilogue: one centroid per thread
      const int quad = warp & 3;
      const int rr = quad * 32 + lane;
      uint32_t kmx = 0, kmn = 0;
      int ninf = 0;
      bool ok = wait_bar(&ms->metabar, 0, lim);
      for (int it = 0; it < ntiles; ++it) {
        const int cl = it * kTileC + rr;
        const bool valid = cl < nid;
        const size_t gc = (size_t)u * Cs + id_of(cl);
        ok = ok && wait_bar(&ms->tdone[it], 0, lim);
        if (epilogue_any(!ok)) {  // the 128 threads leave together
          if (!ok) record_status(p.status, RI_ERR_TIMEOUT);
          ms->abort_flag = 1;
          break;
        }
        tc_fence_after();
        float v[8];
        tmem_ld8(tmem + ((uint32_t)(quad * 32) << 16) + it * kQRows, v);
        if (valid) {
          const int cnt = meta[cl].y;
          float s[Gp];
          float rs = 0.f;
#pragma unroll
          for (int g = 0; g < Gp; ++g) {
            s[g] = g < G ? v[g] * kScale : 0.f;
            if (g < G) rs += s[g];
          }
          float4* dst = reinterpret_cast<float4*>(p.score + gc * Gp);
          dst[0] = make_float4(s[0], s[1], s[2], s[3]);
          if constexpr (Gp == 8) dst[1] = make_float4(s[4], s[5], s[6], s[7]);
          keys[cl] = cnt > 0 ? rs : -INFINITY;
          if (cnt > 0) {
            const uint32_t o = float_order_key(rs);
            kmx = max(kmx, o);
            kmn = max(kmn, ~o);
          } else {
            ++ninf;
          }
        }
      }
      kmx = __reduce_max_sync(0xffffffffu, kmx);
      kmn = __reduce_max_sync(0xffffffffu, kmn);
      ninf = __reduce_add_sync(0xffffffffu, ninf);
      if (lane == 0) {
        atomicMax(&ms->own_kmax, kmx);
        atomicMax(&ms->own_kmin, kmn);
        atomicAdd(&ms->own_ninf, ninf);
      }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, ncols);
  }
  __syncthreads();
  RI_STAMP(1, 0);
  if (ms->abort_flag && nid > 0) {
    // a failed scoring pass leaves no usable key: the block's clusters are
    // treated as empty (selected only past every finite key, never attended)
    for (int i = tid; i < nid; i += kThreads) {
      keys[i] = -INFINITY;
      meta[i] = make_int2(0, 0);
    }
    if (tid == 0) {
      ms->own_kmax = ms->own_kmin = 0u;
      ms->own_ninf = nid;
    }
    __syncthreads();
  }
  cluster_wait();  // 0: every block of the cluster has started

  // ============================================================ step B
  const int kA = p.kr, kB = p.kr + p.ke;
  const bool onA = kA > 0, onB = p.ke > 0;
  if (selecting) {
    int* hist = reinterpret_cast<int*>(sm + kRHist);
    int* dig = reinterpret_cast<int*>(sm + kRDig);
    int* lgs = reinterpret_cast<int*>(sm + kRLgs);
    const int* gin = reinterpret_cast<const int*>(sm + kRGin);
    unsigned long long* cin = reinterpret_cast<unsigned long long*>(sm + kRCin);
    unsigned long long* all = reinterpret_cast<unsigned long long*>(sm + kRAll);
    const uint32_t hist_a = sm_base + kRHist, dig_a = sm_base + kRDig;
    // this block's key range and empty count, pushed to every block
    if (tid < CS)
      st_cl_v4(mapa(smem_u32(&ms->rng_in[b]), (uint32_t)tid),
               make_uint4(ms->own_kmax, ms->own_kmin, (uint32_t)ms->own_ninf, 0u));
    for (int i = tid; i < kNB; i += kThreads) hist[i] = 0;
    for (int i = tid; i < 4 * 2 * 256; i += kThreads) dig[i] = 0;
    if (tid < 64) ms->fine[tid >> 5][tid & 31] = 0;
    for (int i = tid; i < kGroups; i += kThreads) lgs[i] = 0;
    cluster_sync();  // 1: key ranges pushed
    RI_STAMP(2, 0);

    // every warp takes the cluster's key range and empty count itself
    float lo, scale;
    int nfin, ninf;
    {
      uint32_t kx = 0, kn = 0;
      int ni = 0;
      if (lane < CS) {
        const uint4 v = ms->rng_in[lane];
        kx = v.x;
        kn = v.y;
        ni = (int)v.z;
      }
      kx = __reduce_max_sync(0xffffffffu, kx);
      kn = __reduce_max_sync(0xffffffffu, kn);
      ni = __reduce_add_sync(0xffffffffu, ni);
      nfin = C - ni;
      ninf = ni;
      lo = nfin > 0 ? float_from_order_key(~kn) : 0.f;
      const float hi = nfin > 0 ? float_from_order_key(kx) : 0.f;
      scale = (nfin > 0 && hi > lo) ? (float)kNB / (hi - lo) : 0.f;
    }
    // the block's histogram of its own keys and its sums over groups of 32
    // buckets; the group sums are pushed
    for (int i = tid; i < nid; i += kThreads) {
      const int bk = bucket_of(keys[i], lo, scale);
      if (bk >= 0) {
        atomicAdd(&hist[bk], 1);
        atomicAdd(&lgs[bk >> 5], 1);
      }
    }
    __syncthreads();
    RI_STAMP(26, 0);
    if (tid < 32 * CS) {
      const int q = tid >> 5, j = tid & 31;  // target block, 16-byte piece
      const int4 v = reinterpret_cast<const int4*>(lgs)[j];
      st_cl_v4(mapa(sm_base + kRGin + 4u * (uint32_t)(b * kGroups + 4 * j), (uint32_t)q),
               make_uint4((uint32_t)v.x, (uint32_t)v.y, (uint32_t)v.z, (uint32_t)v.w));
    }
    cluster_sync();  // 2: group sums pushed; histograms final
    RI_STAMP(3, 0);

    // boundary buckets of ranks kA and kB from the top: first the group,
    // then the bucket inside it
    {
      if (tid < kGroups) {
        int v = 0;
        for (int q = 0; q < CS; ++q) v += gin[q * kGroups + tid];
        ms->gsum[tid] = v;
      }
      if (tid < 2) {
        const int k = tid == 0 ? kA : kB;
        const bool on = tid == 0 ? onA : onB;
        ms->bucket[tid] = !on ? -2 : (k > nfin ? -1 : -3);
        ms->above[tid] = k > nfin ? nfin : 0;
        ms->nmem[tid] = k > nfin ? ninf : 0;
        ms->digit[tid] = -1;  // boundary group (finite case)
      }
      __syncthreads();
      const int gi = kGroups - 1 - tid;  // thread order = groups from the top
      const int gs = tid < kGroups ? ms->gsum[gi] : 0;
      int total_fin;
      const int excl = block_scan(gs, ms->scan, &total_fin);
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const int k = w == 0 ? kA : kB;
        const bool on = w == 0 ? onA : onB;
        if (tid < kGroups && on && k <= nfin && excl < k && excl + gs >= k) {
          ms->digit[w] = gi;
          ms->above[w] = excl;
        }
      }
      __syncthreads();
      RI_STAMP(28, 0);
      // the two boundary groups' bucket counts, summed over the blocks
      if (tid < 2 * 8 * CS) {
        const int w = tid / (8 * CS), r = tid - w * 8 * CS;
        const int q = r >> 3, j = r & 7;
        const int g = ms->digit[w];
        if (g >= 0) {
          const int4 v = ld_cl_v4(mapa(hist_a + 4u * (uint32_t)(g * 32 + 4 * j), (uint32_t)q));
          if (v.x) atomicAdd(&ms->fine[w][4 * j], v.x);
          if (v.y) atomicAdd(&ms->fine[w][4 * j + 1], v.y);
          if (v.z) atomicAdd(&ms->fine[w][4 * j + 2], v.z);
          if (v.w) atomicAdd(&ms->fine[w][4 * j + 3], v.w);
        }
      }
      __syncthreads();
      RI_STAMP(29, 0);
      if (warp < 2 && ms->digit[warp] >= 0) {
        const int w = warp, g = ms->digit[w];
        const int k = w == 0 ? kA : kB;
        const int bkt = g * 32 + 31 - lane;  // lane order = buckets from the top
        const int v = ms->fine[w][31 - lane];
        int incl = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += t;
        }
        const int base = ms->above[w];
        const unsigned hit = __ballot_sync(0xffffffffu, base + incl - v < k && base + incl >= k);
        const int L = __ffs(hit) - 1;
        if (lane == L) {
          ms->bucket[w] = bkt;
          ms->above[w] = base + incl - v;
          ms->nmem[w] = v;
        }
      }
      __syncthreads();
      if (tid < 2) {
        const int k = tid == 0 ? kA : kB;
        ms->kp[tid] = k - ms->above[tid];
        ms->slow[tid] = ms->bucket[tid] != -2 && ms->nmem[tid] > kCand;
      }
      __syncthreads();
      RI_STAMP(12, 0);
      RI_STAMP_VAL(20, 0, ms->nmem[0]);
      RI_STAMP_VAL(21, 0, ms->nmem[1]);
      RI_STAMP_VAL(22, 0, ms->slow[0] * 2 + ms->slow[1]);
    }
    const int bk0 = ms->bucket[0], bk1 = ms->bucket[1];
    const bool fast0 = bk0 != -2 && !ms->slow[0], fast1 = bk1 != -2 && !ms->slow[1];
    const bool slow0 = ms->slow[0], slow1 = ms->slow[1];

    // ---- few members: every block pushes its members of the boundary
    // buckets to every block, which ranks them all directly
    if (fast0 || fast1) {
      for (int i = tid; i < nid; i += kThreads) {
        const float key = keys[i];
        const int bk = bucket_of(key, lo, scale);
#pragma unroll
        for (int w = 0; w < 2; ++w) {
          if ((w == 0 ? fast0 : fast1) && bk == (w == 0 ? bk0 : bk1)) {
            const int slot = atomicAdd(&ms->own_ncand[w], 1);
            if (slot < kCand)
              cin[(w * kMaxCS + b) * kCand + slot] = ord64(float_order_key(key), id_of(i));
          }
        }
      }
      __syncthreads();
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const int n = min(kCand, ms->own_ncand[w]);
        // (target, member) pairs, the count first
        for (int t = tid; t < CS * (n + 1); t += kThreads) {
          const int q = t / (n + 1), j = t - q * (n + 1);
          if (j == n)
            st_cl_u32(mapa(smem_u32(&ms->candn_in[w][b]), (uint32_t)q), (uint32_t)n);
          else if (q != b)
            st_cl_u64(mapa(sm_base + kRCin + 8u * (uint32_t)((w * kMaxCS + b) * kCand + j),
                           (uint32_t)q),
                      cin[(w * kMaxCS + b) * kCand + j]);
        }
      }
      RI_STAMP(13, 0);
      cluster_sync();  // 3: every block's boundary members pushed
      RI_STAMP(14, 0);
      // warp w ranks the members of boundary w: lane q copies block q's
      // members (pushed to cin[w][q][0 .. n_q)) to their place in all[w]
      // (a warp scan over the n_q), then lane i ranks member i by counting
      // the larger ones
      if (warp < 2 && (warp == 0 ? fast0 : fast1)) {
        const int w = warp;
        unsigned long long* aw = all + w * kCand;
        const int cq = lane < CS ? min(kCand, ms->candn_in[w][lane]) : 0;
        int incl = cq;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += t;
        }
        const int n = min(kCand, __shfl_sync(0xffffffffu, incl, 31));
        const unsigned long long* src = cin + (w * kMaxCS + lane) * kCand;
        for (int k = 0; k < cq; ++k) {
          const int pos = incl - cq + k;
          if (pos < kCand) aw[pos] = src[k];
        }
        __syncwarp();
        for (int i = lane; i < n; i += 32) {
          const unsigned long long me = aw[i];
          int greater = 0;
#pragma unroll 8
          for (int t = 0; t < n; ++t) greater += aw[t] > me;
          if (greater == ms->kp[w] - 1) ms->thr[w] = me;  // kp: 1-based rank in the bucket
        }
      }
      __syncthreads();
      RI_STAMP(15, 0);
    }

    // ---- crowded bucket: radix walk over the order key, then the id count
    if (slow0 || slow1)
      crowded_thresholds(keys, nid, lo, scale, bk0, bk1, slow0, slow1, ms, dig_a,
                         reinterpret_cast<const int*>(sm + kRTin), sm_base + kRTin, CS, b,
                         ntiles, p.tiles, p.status);
    const unsigned long long thrA = onA ? ms->thr[0] : ~0ull, thrB = onB ? ms->thr[1] : ~0ull;
    RI_STAMP(4, 0);

    // ---- classification of the block's ids and the id-ordered lists:
    // R entries (first row, token prefix in the block) then E entries (id,
    // size); per own tile the counts (R, E, R tokens) for the outputs
    const bool need_out = p.mode == kModeSelect || p.sel_user || p.rpre_user;
    int* tcl = ms->gsum;  // [32 own tiles][3], free after the boundary search
    for (int i = tid; i < 3 * kMaxTilesPerBlock; i += kThreads) tcl[i] = 0;
    __syncthreads();
    RI_STAMP(30, 0);
    {
      // thread t takes kper consecutive local ids; kper is a power of two, so
      // no thread's ids straddle a tile
      int kper = 1;
      while (kper * kThreads < nid) kper <<= 1;
      const int i0 = tid * kper, i1 = min(i0 + kper, nid);
      float kk[kKPT];
      int2 mm[kKPT];
#pragma unroll
      for (int j = 0; j < kKPT; ++j) {
        if (j >= kper) break;  // kper is the same in every thread
        const int i = i0 + j;
        if (i < i1) {
          kk[j] = keys[i];
          mm[j] = meta[i];
        }
      }
      uint32_t mR = 0, mE = 0;
      int tokr = 0;
      bool bad = false;
#pragma unroll
      for (int j = 0; j < kKPT; ++j) {
        if (j >= kper) break;
        const int i = i0 + j;
        if (i >= i1) continue;
        const unsigned long long o = ord64(float_order_key(kk[j]), id_of(i));
        const bool inR = onA && o >= thrA;
        const bool inE = !inR && onB && o >= thrB;
        if (inR || inE) {
          const int off = mm[j].x, cnt = mm[j].y;
          const bool ok = inR ? (cnt >= 0 && off >= 0 && (long long)off + cnt <= p.Ms)
                              : cnt >= 0;
          if (!ok) {
            bad = true;
            mm[j] = make_int2(0, 0);
          }
        }
        if (inR) tokr += mm[j].y;
        mR |= (uint32_t)inR << j;
        mE |= (uint32_t)inE << j;
      }
      if (bad) record_status(p.status, RI_ERR_INVALID_ARG);
      if (need_out && i0 < i1 && (mR | mE)) {
        const int lt = i0 >> 7;
        atomicAdd(&tcl[3 * lt], __popc(mR));
        atomicAdd(&tcl[3 * lt + 1], __popc(mE));
        atomicAdd(&tcl[3 * lt + 2], tokr);
      }
      RI_STAMP(31, 0);
      int2 tots;
      const int2 exs = block_scan2((__popc(mR) << 16) | __popc(mE), tokr, ms->scan, &tots);
      RI_STAMP(32, 0);
      const int excl = exs.x, tot = tots.x, ttot = tots.y;
      int texcl = exs.y;
      const int nR = tot >> 16, nE = tot & 0xFFFF;
      // keys are all in registers now: the lists take their place
      uint16_t* rid = reinterpret_cast<uint16_t*>(sm + kRRid);
      int pr = excl >> 16, pe = nR + (excl & 0xFFFF);
#pragma unroll
      for (int j = 0; j < kKPT; ++j) {
        if (j >= kper) break;
        if ((mR >> j) & 1u) {
          lists[pr] = make_int2(mm[j].x, texcl);
          rid[pr] = (uint16_t)(i0 + j);
          texcl += mm[j].y;
          ++pr;
        } else if ((mE >> j) & 1u) {
          lists[pe++] = make_int2(id_of(i0 + j), mm[j].y);
        }
      }
      if (tid == 0) {
        ms->own_nR = nR;
        ms->own_nE = nE;
        ms->own_tokR = ttot;
      }
    }
    RI_STAMP(17, 0);
    if (need_out) {
      // every own tile's counts pushed to every block, then the prefixes
      // over all tiles (in id order) place the block's ids
      __syncthreads();
      for (int t = tid; t < CS * ntiles; t += kThreads) {
        const int q = t / ntiles, lt = t - q * ntiles;
        st_cl_v4(mapa(sm_base + kRTcnt + 16u * (uint32_t)(b + lt * CS), (uint32_t)q),
                 make_uint4((uint32_t)tcl[3 * lt], (uint32_t)tcl[3 * lt + 1],
                            (uint32_t)tcl[3 * lt + 2], 0u));
      }
      cluster_sync();  // 4: every tile's counts pushed
      RI_STAMP(5, 0);
      const uint4* tc = reinterpret_cast<const uint4*>(sm + kRTcnt);
      const uint4 v = tid < p.tiles ? tc[tid] : make_uint4(0u, 0u, 0u, 0u);
      int2 tots;
      const int2 exs = block_scan2((int)((v.x << 16) | v.y), (int)v.z, ms->scan, &tots);
      const int exRE = exs.x, exT = exs.y, totRE = tots.x, totT = tots.y;
      // tile prefixes into the tile-count area (only the own tiles are used)
      int4* tp = reinterpret_cast<int4*>(sm + kRTcnt);
      if (tid < p.tiles) tp[tid] = make_int4(exRE >> 16, exRE & 0xFFFF, exT, 0);
      if (tid == 0) {
        ms->nRp[0] = totRE >> 16;  // cluster-wide totals
        ms->nEp[0] = totRE & 0xFFFF;
        ms->tokRp[0] = totT;
      }
      __syncthreads();
      const bool to_ws = p.mode == kModeSelect;
      const int ksel = p.k_r + p.k_e;
      int32_t* selw = to_ws ? p.sel + (size_t)u * ksel : nullptr;
      int32_t* selu = p.sel_user ? p.sel_user + (size_t)u * ksel : nullptr;
      int32_t* rpw = to_ws ? p.rpre + (size_t)u * (p.k_r + 1) : nullptr;
      int32_t* rpu = p.rpre_user ? p.rpre_user + (size_t)u * (p.k_r + 1) : nullptr;
      const uint16_t* rid = reinterpret_cast<const uint16_t*>(sm + kRRid);
      const int nR = ms->own_nR, nE = ms->own_nE;
      // local starts of each own tile's R / E entries and R tokens
      // (tcl becomes the exclusive prefix over own tiles)
      if (tid == 0) {
        int a = 0, e = 0, t = 0;
        for (int lt = 0; lt < ntiles; ++lt) {
          const int ca = tcl[3 * lt], ce = tcl[3 * lt + 1], ct = tcl[3 * lt + 2];
          tcl[3 * lt] = a;
          tcl[3 * lt + 1] = e;
          tcl[3 * lt + 2] = t;
          a += ca;
          e += ce;
          t += ct;
        }
      }
      __syncthreads();
      for (int i = tid; i < nR; i += kThreads) {
        const int lt = rid[i] >> 7;
        const int4 tpv = tp[b + lt * CS];
        const int g = tpv.x + i - tcl[3 * lt];
        if (g >= p.k_r) continue;
        const int id = id_of(rid[i]);
        const int rp = tpv.z + lists[i].y - tcl[3 * lt + 2];
        if (selw) selw[g] = id;
        if (selu) selu[g] = id;
        if (rpw) rpw[g] = rp;
        if (rpu) rpu[g] = rp;
      }
      for (int i = tid; i < nE; i += kThreads) {
        const int id = lists[nR + i].x;
        const int lt = ((id >> 7) - b) / CS;
        const int e = tp[id >> 7].y + i - tcl[3 * lt + 1];
        if (e >= p.k_e) continue;
        if (selw) selw[p.k_r + e] = id;
        if (selu) selu[p.k_r + e] = id;
      }
      if (b == CS - 1) {
        const int KRt = ms->nRp[0], KEt = ms->nEp[0];
        for (int g = KRt + tid; g < p.k_r; g += kThreads) {
          if (selw) selw[g] = -1;
          if (selu) selu[g] = -1;
        }
        for (int e = KEt + tid; e < p.k_e; e += kThreads) {
          if (selw) selw[p.k_r + e] = -1;
          if (selu) selu[p.k_r + e] = -1;
        }
        for (int g = min(KRt, p.k_r) + tid; g <= p.k_r; g += kThreads) {
          if (rpw) rpw[g] = ms->tokRp[0];
          if (rpu) rpu[g] = ms->tokRp[0];
        }
      }
    }
  }
  if (C == 0 && p.mode != kModeAttend && b == 0) {
    // no indexed token: empty zones
    const int ksel = p.k_r + p.k_e;
    for (int i = tid; i < ksel; i += kThreads) {
      if (p.sel_user) p.sel_user[(size_t)u * ksel + i] = -1;
      if (p.mode == kModeSelect) p.sel[(size_t)u * ksel + i] = -1;
    }
    for (int i = tid; i <= p.k_r; i += kThreads) {
      if (p.rpre_user) p.rpre_user[(size_t)u * (p.k_r + 1) + i] = 0;
      if (p.mode == kModeSelect) p.rpre[(size_t)u * (p.k_r + 1) + i] = 0;
    }
  }
  // after barrier 4 nothing reads another block's shared memory in a select
  if (p.mode == kModeSelect) {
    RI_STAMP_DUMP();
    return;
  }

  // ============================================================ step C
  // The block attends over the clusters it scored (its own R and E lists,
  // in shared memory) and over an even share of the steady tokens.  After a
  // separate select, the attend call rebuilds the same lists from the
  // workspace by the same tile ownership, so the one-call decode and the
  // split calls fold the same items in the same order.
  const bool exec = p.exec_rows > 0;
  const long long lim_rows = exec ? p.exec_rows : p.Ms;
  const int n_st = p.n_steady;
  const int st0 = (int)((long long)n_st * b / CS), st1 = (int)((long long)n_st * (b + 1) / CS);
  if (!selecting && C > 0) {
    const int32_t* selg = p.sel + (size_t)u * (p.k_r + p.k_e);
    const int32_t* rpg = p.rpre + (size_t)u * (p.k_r + 1);
    const int32_t* off_u = p.offsets + (size_t)u * (Cs + 1);
    // R: the workspace's retrieval clusters (id order) of this block's tiles
    {
      const int kr = p.kr;
      const int per = (kr + kThreads - 1) / kThreads;  // <= 8 (kr <= 4096)
      const int g0 = min(kr, tid * per), g1 = min(kr, g0 + per);
      int rowv[kKPT], cntv[kKPT];
      uint32_t mk = 0;
      int tok = 0;
      bool bad = false;
#pragma unroll
      for (int j = 0; j < kKPT; ++j) {
        const int g = g0 + j;
        rowv[j] = 0;
        cntv[j] = 0;
        if (g < g1) {
          const int id = __ldcg(selg + g);
          if (id >= 0 && id < C && (id >> 7) % CS == b) {
            const int r0 = __ldcg(rpg + g), cnt = __ldcg(rpg + g + 1) - r0;
            const int row = exec ? r0 : __ldg(off_u + id);
            if (cnt >= 0 && row >= 0 && (long long)row + cnt <= lim_rows) {
              rowv[j] = row;
              cntv[j] = cnt;
            } else {
              bad = true;
            }
            mk |= 1u << j;
            tok += cntv[j];
          } else if (id < -1 || id >= C) {
            bad = true;
          }
        }
      }
      if (bad) record_status(p.status, RI_ERR_INVALID_ARG);
      int2 tots;
      const int2 exs = block_scan2(__popc(mk), tok, ms->scan, &tots);
      const int ex = exs.x, tot = tots.x, ttot = tots.y;
      int tex = exs.y;
      int pos = ex;
#pragma unroll
      for (int j = 0; j < kKPT; ++j)
        if ((mk >> j) & 1u) {
          if (pos < kMaxIdsPerBlock) lists[pos] = make_int2(rowv[j], tex);
          tex += cntv[j];
          ++pos;
        }
      if (tid == 0) {
        ms->own_nR = min(tot, kMaxIdsPerBlock);
        ms->own_tokR = ttot;
      }
    }
    __syncthreads();
    // E: the workspace's estimation clusters of this block's tiles, two
    // passes over each thread's contiguous run (count, then write)
    {
      const int nRo = ms->own_nR;
      const int ke = p.ke;
      const int per = (ke + kThreads - 1) / kThreads;
      const int g0 = min(ke, tid * per), g1 = min(ke, g0 + per);
      int n = 0;
      for (int g = g0; g < g1; ++g) {
        const int id = __ldcg(selg + p.k_r + g);
        n += id >= 0 && id < C && (id >> 7) % CS == b;
      }
      int tot;
      int pos = nRo + block_scan(n, ms->scan, &tot);
      for (int g = g0; g < g1; ++g) {
        const int id = __ldcg(selg + p.k_r + g);
        if (id >= 0 && id < C && (id >> 7) % CS == b) {
          if (pos < kMaxIdsPerBlock)
            lists[pos] = make_int2(id, max(0, __ldg(p.counts + (size_t)u * Cs + id)));
          ++pos;
        }
      }
      if (tid == 0) ms->own_nE = min(tot, kMaxIdsPerBlock - nRo);
    }
  }
  // the ring was last written by the TMA (async proxy) and by step B: order
  // both before the copies of step C
  fence_proxy_async_smem();
  __syncthreads();

  const int2* rlist = lists;
  const int2* elist_all = lists + ms->own_nR;
  const int nR = ms->own_nR, nE = ms->own_nE;
  const int ns_loc = st1 - st0, st_start = st0;  // steady tokens of this block
  const long long kofs = 0, ntok = (long long)ns_loc + ms->own_tokR;
  const long long rend = ms->own_tokR;  // search key past the last R entry's tokens

  // ---- the state of the two kinds of warps:
  //  token warps (0..7): O^T fragments ot[j][i] (lane holds dims 16 j + gid
  //   (+8), heads 2 tig (+1)), the running maximum tm of head gid (log2
  //   units) and the lane's share tl of head gid's denominator;
  //  estimation warps (8..15): lane (head g, dim group dg) holds its head's
  //   maximum em, denominator el and numerators of its dims.
  // Each kind of warp writes its partial into wo [kWarps][G][128] (the ring,
  // once every warp is done with it) and wm / wl.
  float* wo = reinterpret_cast<float*>(sm);
  RI_STAMP(19, 0);
  if (warp < kTokenWarps) {
    const int gid = lane >> 2, tig = lane & 3;
    float ot[8][4];
    float tm = -INFINITY, tl = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int i = 0; i < 4; ++i) ot[j][i] = 0.f;
    // A fragments of Q (rows = query heads, padded to 16 with zeros):
    // qa[kk][0] = Q[gid][16 kk + 2 tig ..], qa[kk][1] = Q[gid][16 kk + 8 + 2 tig ..]
    uint32_t qa[8][2];
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      if (gid < G) {
        const __nv_bfloat16* qr = p.q + ((size_t)u * G + gid) * kHeadDim + kk * 16 + tig * 2;
        qa[kk][0] = __ldg(reinterpret_cast<const unsigned int*>(qr));
        qa[kk][1] = __ldg(reinterpret_cast<const unsigned int*>(qr + 8));
      } else {
        qa[kk][0] = qa[kk][1] = 0u;
      }
    }
    RI_STAMP(33, 0);
    const __nv_bfloat16* Kr = p.Kr + (size_t)u * lim_rows * kHeadDim;
    const __nv_bfloat16* Vr = p.Vr + (size_t)u * lim_rows * kHeadDim;
    const __nv_bfloat16* Ksu = p.Ks + (size_t)u * n_st * kHeadDim;
    const __nv_bfloat16* Vsu = p.Vs + (size_t)u * n_st * kHeadDim;
    const __nv_bfloat16* safe = n_st > 0 ? Ksu : Kr;  // a readable address for zero fills
    uint8_t* wbuf = sm + warp * kTokenWarpBytes;       // two tiles of 16 rows (K then V)
    int* rowtab = reinterpret_cast<int*>(sm + kOffRuns);
    // 16-byte chunk c of token row t of a tile, XOR-swizzled for ldmatrix
    auto row_chunk = [](int t, int c) { return (uint32_t)(t * 256 + ((c ^ (t & 7)) << 4)); };
    const int tt = tid;  // 0 .. 255 over the token warps
    for (long long wt = 0; wt < ntok; wt += kWindowTokens) {
      // ---- the window's token rows (R rows >= 0, steady rows as -1 - row),
      // written by the 256 threads of the token warps from the local lists
      const int nwt = (int)min((long long)kWindowTokens, ntok - wt);
      // one token per thread: a steady token, or R token j found in its
      // cluster by a binary search over the R list's token prefix
      for (int t = tt; t < nwt; t += kTokenWarps * 32) {
        const long long bt = wt + t;
        if (bt < ns_loc) {
          rowtab[t] = -1 - (st_start + (int)bt);
        } else {
          const int j = (int)(bt - ns_loc + kofs);
          int lo = 0, hi = nR - 1;  // last entry with prefix <= j
          while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (rlist[mid].y <= j) lo = mid; else hi = mid - 1;
          }
          const int2 e = rlist[lo];
          const long long end = lo + 1 < nR ? (long long)rlist[lo + 1].y : rend;
          // an entry without a row (failed checks) or a key outside it: masked
          rowtab[t] = (nR > 0 && e.x >= 0 && j >= e.y && j < end) ? e.x + (j - e.y) : INT_MIN;
        }
      }
      token_bar();
      RI_STAMP(25, 0);
      const int ntile = (nwt + 15) >> 4;
      // ---- tiles warp, warp + kTokenWarps, ...: copies one tile ahead
      // copies of a tile: each instruction moves two whole rows (lanes 0-15
      // row 2 k, lanes 16-31 row 2 k + 1, 16 bytes each), so every 32-byte
      // sector is requested once
      auto issue = [&](int tj, int slot) {
        if (tj < ntile) {
          uint8_t* kb = wbuf + slot * 8192;
          const int tok = tj * 16 + (lane & 15);
          const int code_l = tok < nwt ? rowtab[tok] : INT_MIN;  // lane r < 16: row r
          const int c = lane & 15, h = lane >> 4;
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const int t = 2 * k + h;
            const int code = __shfl_sync(0xffffffffu, code_l, t);
            const __nv_bfloat16 *ks = safe, *vs = safe;
            const bool fill = code != INT_MIN;
            if (code >= 0) {
              ks = Kr + (size_t)code * kHeadDim;
              vs = Vr + (size_t)code * kHeadDim;
            } else if (fill) {
              ks = Ksu + (size_t)(-1 - code) * kHeadDim;
              vs = Vsu + (size_t)(-1 - code) * kHeadDim;
            }
            cp_async16_zfill(kb + row_chunk(t, c), fill ? ks + c * 8 : safe, fill);
            cp_async16_zfill(kb + 4096 + row_chunk(t, c), fill ? vs + c * 8 : safe, fill);
          }
        }
        cp_async_commit();
      };
      constexpr float kQK = kScale * kLog2e;
      int slot = 0;
      issue(warp, 0);
      for (int tj = warp; tj < ntile; tj += kTokenWarps) {
        issue(tj + kTokenWarps, slot ^ 1);
        cp_async_wait<1>();
        __syncwarp();
        const uint32_t kbase = smem_u32(wbuf + slot * 8192);
        const uint32_t vbase = kbase + 4096;
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
            uint32_t bq[4];
            ldmatrix_x4(bq, kbase + row_chunk(tr, ch));
            mma_bf16_16816(sacc[h], qa[2 * kp][0], 0u, qa[2 * kp][1], 0u, bq[0], bq[1]);
            mma_bf16_16816(sacc[h], qa[2 * kp + 1][0], 0u, qa[2 * kp + 1][1], 0u, bq[2], bq[3]);
          }
        }
        // row gid: logits of tokens 8h + 2 tig (+1); padding and rows out of range masked
        float x[4];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int t = tj * 16 + h * 8 + tig * 2 + i;
            const bool ok = t < nwt && rowtab[t] != INT_MIN;
            x[h * 2 + i] = ok ? sacc[h][i] * kQK : -INFINITY;
          }
        float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        float corr = 1.f;
        if (mx > tm + kRescale2) {  // new reference (also the first tile)
          corr = tm == -INFINITY ? 0.f : ex2f(tm - mx);
          tm = mx;
          tl *= corr;
        }
        // O^T columns 2 tig, 2 tig + 1 rescale by the factors of those rows
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
          uint32_t av[4];
          ldmatrix_x4_trans(av, vbase + row_chunk(tr, ch));
          mma_bf16_16816(ot[j], av[0], av[1], av[2], av[3], pb0, pb1);
        }
        __syncwarp();
        slot ^= 1;
      }
      cp_async_wait<0>();
      token_bar();  // the row table is rebuilt for the next window
    }
    RI_STAMP(23, 0);
    __syncthreads();  // every warp done with step C: the ring is free
    tl += __shfl_xor_sync(0xffffffffu, tl, 1);
    tl += __shfl_xor_sync(0xffffffffu, tl, 2);
    if (tig == 0 && gid < G) {
      ms->wm[warp][gid] = tm;
      ms->wl[warp][gid] = tl;
    }
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int g = tig * 2 + k;
        if (g < G) {
          float* rg = wo + ((size_t)warp * G + g) * kHeadDim + j * 16 + gid;
          rg[0] = ot[j][k];
          rg[8] = ot[j][2 + k];
        }
      }
  } else {
    // ---- estimation clusters: the block's E list split over the E warps,
    // folded on the tensor cores in groups of 4 clusters:
    //   O^T[d][g] += sum_k Vsum_k[d] w_k[g],  w_k[g] = 2^(x_k[g] - m_g),
    // one mma.m16n8k4 (TF32 inputs, fp32 sums) per 16 dims.  Lane (gid,
    // tig) supplies cluster tig of the group: the value sums of dims
    // 16 t + 2 gid and + 1 as rows gid and gid + 8 of A (the dims of a
    // 16-dim tile are permuted so both come from one 8-byte load) and the
    // weight of head gid as B[tig][gid]; it accumulates dims 16 t + 2 gid
    // (+1) of heads 2 tig and 2 tig + 1.  The running maximum is per head
    // (the 4 lanes of head gid agree), the denominator summed per lane.
    // Each warp streams its clusters' value sums and scores through its
    // own ring of slots with 16-byte cp.async copies, two groups ahead.
    const int gid = lane >> 2, tig = lane & 3;
    float dacc[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int i = 0; i < 4; ++i) dacc[mt][i] = 0.f;
    float em = -INFINITY, el = 0.f;  // head gid: maximum (log2 units), lane's denominator
    const int ew = warp - kTokenWarps;
    const int e0 = nE * ew / kEWarps, e1 = nE * (ew + 1) / kEWarps;
    const int2* elist = elist_all;
    uint8_t* ering = sm + kOffMeta + ew * kEWarpBytes;
    constexpr int kQuads = kESlots / 4;
    const float* vs_lane = p.vsum + (size_t)u * Cs * kHeadDim + lane * 4;
    const float* sc_lane = p.score + (size_t)u * Cs * Gp + lane * 4;
    const uint32_t ering_lane = smem_u32(ering) + lane * 16;
    const bool sc_lane_on = lane < Gp / 4;
    auto issue = [&](int e, int quad) {
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        if (e + k < e1) {
          const int2 ev = elist[e + k];
          if (ev.y > 0) {
            const uint32_t slot = ering_lane + (uint32_t)(4 * quad + k) * kSlotE;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(slot),
                         "l"(vs_lane + (size_t)ev.x * kHeadDim)
                         : "memory");
            if (sc_lane_on)
              asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(slot + 512u),
                           "l"(sc_lane + (size_t)ev.x * Gp)
                           : "memory");
          }
        }
      }
      cp_async_commit();
    };
    for (int k = 0; k < kQuads - 1; ++k) issue(e0 + 4 * k, k);
#ifdef RI_DEBUG_PHASES
    long long cyc_w = 0, cyc_c = 0, cyc_t = clock64();
#endif
    int qr = 0;  // ring group of item e
#pragma unroll 1
    for (int e = e0; e < e1; e += 4) {
      issue(e + 4 * (kQuads - 1), qr == 0 ? kQuads - 1 : qr - 1);
      cp_async_wait<kQuads - 1>();
      __syncwarp();
#ifdef RI_DEBUG_PHASES
      {
        const long long n_ = clock64();
        cyc_w += n_ - cyc_t;
        cyc_t = n_;
      }
#endif
      const uint8_t* st = ering + (uint32_t)(4 * qr + tig) * kSlotE;  // cluster tig's slot
      const int2 ev = e + tig < e1 ? elist[e + tig] : make_int2(0, 0);
      const bool v = ev.y > 0;  // the slot holds this cluster's sums
      const bool vh = v && gid < G;
      const float x = vh ? reinterpret_cast<const float*>(st + 512)[gid] * kLog2e : -INFINITY;
      float xm = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
      xm = fmaxf(xm, __shfl_xor_sync(0xffffffffu, xm, 2));
      float corr = 1.f;
      if (xm > em + kRescale2) {  // new reference (also the first cluster)
        corr = em == -INFINITY ? 0.f : ex2f(em - xm);
        em = xm;
        el *= corr;
      }
      if (__any_sync(0xffffffffu, corr != 1.f)) {
        // columns 2 tig, 2 tig + 1 rescale by those heads' factors
        const float c0 = __shfl_sync(0xffffffffu, corr, (tig * 2) * 4);
        const float c1 = __shfl_sync(0xffffffffu, corr, (tig * 2 + 1) * 4);
#pragma unroll
        for (int mt = 0; mt < 8; ++mt) {
          dacc[mt][0] *= c0;
          dacc[mt][1] *= c1;
          dacc[mt][2] *= c0;
          dacc[mt][3] *= c1;
        }
      }
      const float w = vh ? ex2f(x - em) : 0.f;
      el = fmaf((float)ev.y, w, el);
      const uint32_t b0 = tf32_rn(w);
      const float* arow = reinterpret_cast<const float*>(st) + 2 * gid;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
        const float2 a = v ? *reinterpret_cast<const float2*>(arow + 16 * mt) : make_float2(0.f, 0.f);
        mma_tf32_1684(dacc[mt], tf32_rn(a.x), tf32_rn(a.y), b0);
      }
      qr = qr + 1 == kQuads ? 0 : qr + 1;
      __syncwarp();
#ifdef RI_DEBUG_PHASES
      {
        const long long n_ = clock64();
        cyc_c += n_ - cyc_t;
        cyc_t = n_;
      }
#endif
    }
#ifdef RI_DEBUG_PHASES
    RI_STAMP_VAL(40, kTokenWarps * 32, cyc_w);
    RI_STAMP_VAL(41, kTokenWarps * 32, cyc_c);
    RI_STAMP_VAL(42, kTokenWarps * 32, e1 - e0);
#endif
    el += __shfl_xor_sync(0xffffffffu, el, 1);
    el += __shfl_xor_sync(0xffffffffu, el, 2);
    cp_async_wait<0>();
    RI_STAMP(24, kTokenWarps * 32);
    __syncthreads();  // every warp done with step C: the ring is free
    if (tig == 0 && gid < G) {
      ms->wm[warp][gid] = em;
      ms->wl[warp][gid] = el;
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int h = tig * 2 + k;
        if (h < G) {
          float* rg = wo + ((size_t)warp * G + h) * kHeadDim + 16 * mt + 2 * gid;
          rg[0] = dacc[mt][k];
          rg[1] = dacc[mt][2 + k];
        }
      }
  }
  __syncthreads();
  RI_STAMP(6, 0);

  // ============================================================ step D
  // warps -> block partial (max in log2 units, denominator, numerator):
  // thread t < 32 G takes head t / 32 and dims 4 (t % 32) .. + 3
  const bool pt = tid < G * 32;
  const int pg = pt ? tid >> 5 : 0, pd = (tid & 31) * 4;
  float4 bo4 = make_float4(0.f, 0.f, 0.f, 0.f);
  float bm = -INFINITY, bl = 0.f;
  if (pt) {
#pragma unroll
    for (int w = 0; w < kWarps; ++w) bm = fmaxf(bm, ms->wm[w][pg]);
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float mw = ms->wm[w][pg];
      const float f = mw == -INFINITY ? 0.f : ex2f(mw - bm);
      bl = fmaf(f, ms->wl[w][pg], bl);
      const float4 o = *reinterpret_cast<const float4*>(wo + ((size_t)w * G + pg) * kHeadDim + pd);
      bo4.x = fmaf(f, o.x, bo4.x);
      bo4.y = fmaf(f, o.y, bo4.y);
      bo4.z = fmaf(f, o.z, bo4.z);
      bo4.w = fmaf(f, o.w, bo4.w);
    }
  }
  // every block's partial into block 0: per block and head 132 floats
  // (numerator[128], max, denominator, 2 unused) at the start of its ring.
  // Block 0 releases the ring with a remote arrive on every other block's
  // `go` (after its own warps' partials are read); the others store theirs
  // with st.async, whose bytes complete block 0's `mrg` (armed at the start
  // for CS - 1 partials).  A block waits only for block 0 and block 0 only
  // for the partials; one last cluster barrier, whose arrivals come early,
  // keeps every block alive until block 0's remote arrive has landed.
  RI_STAMP(7, 0);
  const uint32_t area = sm_base;
  if (b != 0) {
    const bool go = mbar_wait_cl(&ms->go, 0, lim);
    if (!go) {
      record_status(p.status, RI_ERR_TIMEOUT);
    } else if (pt) {
      const uint32_t mrg = mapa(smem_u32(&ms->mrg), 0);
      const uint32_t base = area + (uint32_t)((b * G + pg) * kPartStride);
      st_async_v4(mapa(base + 4u * (uint32_t)pd, 0), bo4, mrg);
      if (pd == 0) st_async_v2(mapa(base + 4u * kHeadDim, 0), bm, bl, mrg);
    }
    cluster_arrive_relaxed();  // 5
    cluster_wait();
    RI_STAMP_DUMP();
    return;
  }
  __syncthreads();  // every warp's partial read: the ring takes the block partials
  if (tid > 0 && tid < CS) mbar_arrive_remote(mapa(smem_u32(&ms->go), (uint32_t)tid));
  if (warp == 0)
    cluster_arrive();  // 5 (release: the remote arrives land before any block exits)
  else
    cluster_arrive_relaxed();
  if (pt) {
    float* base = reinterpret_cast<float*>(sm + pg * kPartStride);
    *reinterpret_cast<float4*>(base + pd) = bo4;
    if (pd == 0) {
      base[kHeadDim] = bm;
      base[kHeadDim + 1] = bl;
    }
  }
  if (!mbar_wait_cl(&ms->mrg, 0, lim)) record_status(p.status, RI_ERR_TIMEOUT);
  __syncthreads();  // block 0's own partial written
  const float* pa = reinterpret_cast<const float*>(sm);
  constexpr int kPS = (int)(kPartStride / 4);
  for (int idx = tid; idx < G * kHeadDim; idx += kThreads) {
    const int g = idx / kHeadDim, d = idx - g * kHeadDim;
    // (loops unrolled over the largest cluster, so the loads are issued together)
    float pm[kMaxCS];
    float mx = -INFINITY;
#pragma unroll
    for (int q = 0; q < kMaxCS; ++q) {
      pm[q] = q < CS ? pa[(q * G + g) * kPS + kHeadDim] : -INFINITY;
      mx = fmaxf(mx, pm[q]);
    }
    float L = 0.f, O = 0.f;
#pragma unroll
    for (int q = 0; q < kMaxCS; ++q) {
      if (q < CS) {
        const float* pq = pa + (q * G + g) * kPS;
        const float f = pm[q] == -INFINITY ? 0.f : ex2f(pm[q] - mx);
        L = fmaf(f, pq[kHeadDim + 1], L);
        O = fmaf(f, pq[d], O);
      }
    }
    // no token and no cluster contributed (empty steady zone and budgets): 0, lse -inf
    const bool any = L > 0.f;
    const size_t hq = (size_t)u * G + g;
    p.out[hq * kHeadDim + d] = __float2bfloat16_rn(any ? O / L : 0.f);
    if (p.lse && d == 0) p.lse[hq] = any ? mx * kLn2 + logf(L) : -INFINITY;
  }
#ifdef RI_DEBUG_PHASES
  __syncthreads();
#endif
  RI_STAMP(8, 0);
  RI_STAMP_DUMP();
  cluster_wait();  // 5
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

// bf16 [rows][128] row-major, boxes of 64 columns x box_rows, 128-byte
// swizzle.  Maps are kept in a small fixed table keyed by (base, rows, box):
// a decode step reuses the maps of its centroid and query buffers.
struct MapSlot {
  const void* base;
  unsigned long long rows;
  unsigned box;
  CUtensorMap map;
};
constexpr int kMapSlots = 64;
std::mutex g_map_mu;
MapSlot g_maps[kMapSlots];
int g_map_next = 0;

cudaError_t encode_rows(CUtensorMap* map, const void* base, unsigned long long rows,
                        unsigned box_rows) {
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    for (int i = 0; i < kMapSlots; ++i)
      if (g_maps[i].base == base && g_maps[i].rows == rows && g_maps[i].box == box_rows) {
        *map = g_maps[i].map;
        return cudaSuccess;
      }
  }
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
  std::lock_guard<std::mutex> lk(g_map_mu);
  MapSlot& s = g_maps[g_map_next];
  g_map_next = (g_map_next + 1) % kMapSlots;
  s.base = base;
  s.rows = rows;
  s.box = box_rows;
  s.map = *map;
  return cudaSuccess;
}

const void* kernel_of(int G) {
  switch (G) {
    case 1: return reinterpret_cast<const void*>(decode_kernel<1>);
    case 2: return reinterpret_cast<const void*>(decode_kernel<2>);
    case 3: return reinterpret_cast<const void*>(decode_kernel<3>);
    case 4: return reinterpret_cast<const void*>(decode_kernel<4>);
    case 5: return reinterpret_cast<const void*>(decode_kernel<5>);
    case 6: return reinterpret_cast<const void*>(decode_kernel<6>);
    case 7: return reinterpret_cast<const void*>(decode_kernel<7>);
    default: return reinterpret_cast<const void*>(decode_kernel<8>);
  }
}

// Per device and group size: kernel attributes set, and how many clusters of
// each size can be resident at once (fixed tables, filled on first use).
constexpr int kMaxDevices = 64;
struct DevState {
  int ready[kMaxGroupHost + 1];
  int n_active[kMaxGroupHost + 1][kMaxClusterBlocks + 1];
};
std::mutex g_dev_mu;
DevState g_dev[kMaxDevices];

cudaError_t device_state(int G, const int** n_active) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevState& s = g_dev[dev];
  if (!s.ready[G]) {
    const void* fn = kernel_of(G);
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    for (int cs = 1; cs <= kMaxClusterBlocks; ++cs) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)cs);
      cfg.blockDim = dim3(kThreads);
      cfg.dynamicSmemBytes = kSmemBytes;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = (unsigned)cs;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) n = 0;
      s.n_active[G][cs] = n;
    }
    cudaGetLastError();
    s.ready[G] = 1;
  }
  *n_active = s.n_active[G];
  return cudaSuccess;
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
  p.sel = reinterpret_cast<int32_t*>(a.ws + L.off_sel);
  p.rpre = reinterpret_cast<int32_t*>(a.ws + L.off_rpre);
  p.status = reinterpret_cast<int*>(a.ws);
  p.wait_ns = a.wait_ns;
  p.fault = a.fault;
  p.BH = (int)g.BH();
  p.C = g.C;
  p.Cs = g.Cs;
  p.Ms = g.Ms;
  p.n_steady = g.n_steady;
  p.k_r = L.k_r;
  p.k_e = L.k_e;
  p.kr = L.kr;
  p.ke = L.ke;
  p.tiles = (g.C + kTileC - 1) / kTileC;
  p.exec_rows = exec ? a.exec_rows : 0;
  p.mode = mode;

  CUtensorMap map_c, map_q;
  memset(&map_c, 0, sizeof(map_c));
  memset(&map_q, 0, sizeof(map_q));
  if (g.C > 0 && mode != kModeAttend) {
    cudaError_t e = encode_rows(&map_c, a.centroid, (unsigned long long)g.BH() * g.Cs, kTileC);
    if (e == cudaSuccess) e = encode_rows(&map_q, a.q, (unsigned long long)g.BH() * G, kQRows);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(g.BH() * L.CS));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)L.CS;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent launch: the set-up of this launch (barriers,
  // tensor memory) may overlap the end of the kernel before it on the stream
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
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

// Launch shape: one cluster of CS blocks per unit, CS between the smallest
// size whose blocks hold the unit's clusters (at most kMaxIdsPerBlock ids per
// block) and kMaxClusterBlocks.  Each size is scored by the waves it needs
// (units over the clusters of that size the device holds at once) times the
// share of a unit one block carries, plus a small per-block term for the
// cluster barriers; the cheapest size wins.
bool decode_plan(const Geometry& g, DecodeLayout* L) {
  const int* n_active = nullptr;
  if (device_state(g.G, &n_active) != cudaSuccess) {
    cudaGetLastError();
    set_error("decode kernel cannot be configured on this device");
    return false;
  }
  const long long units = g.BH();
  const int tiles = (g.C + kTileC - 1) / kTileC;
  const int cs_min = tiles > 0 ? (tiles + kMaxTilesPerBlock - 1) / kMaxTilesPerBlock : 1;
  if (cs_min > kMaxClusterBlocks) {
    set_error("%d clusters per (sequence, KV head) exceed the decode kernel's limit of %d", g.C,
              kMaxClusterBlocks * kMaxIdsPerBlock);
    return false;
  }
  int best = -1;
  double best_cost = 1e30;
  for (int cs = cs_min; cs <= kMaxClusterBlocks; ++cs) {
    const int n = n_active[cs];
    if (n < 1) continue;
    const long long waves = (units + n - 1) / n;
    const double cost = (double)waves * (1.0 / cs + 0.02);
    if (cost < best_cost - 1e-12) {
      best_cost = cost;
      best = cs;
    }
  }
  if (best < 0) {
    set_error("decode kernel cannot be resident on this device (cluster of %d blocks)", cs_min);
    return false;
  }
  L->CS = best;
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

#ifdef RI_DEBUG_PHASES
// Profiling builds only: copies the phase timestamps of the last launch.
extern "C" int ri_debug_phase_times(unsigned long long* host, int blocks) {
  if (blocks > ri::kStampBlocks) blocks = ri::kStampBlocks;
  return (int)cudaMemcpyFromSymbol(host, ri::g_phase_ns,
                                   sizeof(unsigned long long) * ri::kStamps * blocks);
}
#endif
