// Tripartite decode attention over the wave index (sm_100a): one kernel
// launch per decode step, one thread-block cluster per (sequence, KV head).
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
// The P blocks of a unit form one cluster (P <= 16).  Block j
//   A) scores 128-centroid tiles [T j / P, T (j+1) / P) on the tensor cores:
//      TMA brings a tile (128-byte swizzle), one thread issues tcgen05.mma
//      with the unit's G query rows (padded to N = 16) as the B operand, four
//      warps read the fp32 scores from TMEM; the block keeps its keys r_c;
//   B) selects R and E together with the other blocks of the cluster through
//      distributed shared memory: the key range, a 2048-bucket value
//      histogram and the boundary buckets' members are gathered in block 0,
//      every block ranks the few boundary keys exactly, then scatters its R
//      and E members to their positions (R ids to block 0, each E id to the
//      block that attends it).  If a boundary bucket is crowded (heavy ties),
//      every block instead runs the exact selection over all C keys;
//   C) attends its share of the steady + retrieval tokens and of the
//      estimation clusters (16-byte cp.async copies into shared memory, three
//      buffers in flight; 16-lane groups with shuffle reductions);
//   D) leaves its partial (m, l, o) in shared memory; block 0 merges the P
//      partials through distributed shared memory.
// Cluster barriers are hardware barriers; every block executes the same
// sequence of them (no block leaves early), and the mbarrier waits of step A
// are bounded.
#include <cooperative_groups.h>
#include <map>
#include <mutex>
#include <tuple>
#include <float.h>
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace cg = cooperative_groups;

namespace ri {

namespace {

constexpr float kScale = 0.08838834764831845f;  // 1/sqrt(128)
constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr int kTileC = 128;          // centroids per MMA tile (M)
constexpr int kQRows = 16;           // MMA N: query rows padded to 16
constexpr int kStagesA = 2;
constexpr int kNB = 2048;            // value buckets of the selection
constexpr int kBoundaryCap = 256;    // keys ranked exactly in a boundary bucket
constexpr int kPer = 32;             // fallback: keys per thread and round
constexpr int kRound = kThreads * kPer;
constexpr int kTokChunk = 64;        // tokens per copy chunk (K and V rows: 32 KB)
constexpr int kEChunk = 56;          // estimation clusters per chunk (value sum + scores)
constexpr uint32_t kChunkBytes = 32768;
constexpr int kChunkBufs = 2;        // copy buffers of the attention step
static_assert(kTokChunk * 512 <= (int)kChunkBytes && kEChunk * 544 <= (int)kChunkBytes, "chunk");
constexpr int kMaxClusterBlocks = 16;  // blocks per unit (cluster size)
constexpr uint32_t kTileBytes = kTileC * kHeadDim * 2;  // 32 KB
constexpr uint32_t kStageBytes = 65536;  // A: 2 TMA stages; C: 2 copy buffers; D: partials
static_assert(kStagesA * kTileBytes <= kStageBytes && kChunkBufs * kChunkBytes <= kStageBytes, "stage");
constexpr uint32_t kPartOff = 40960;  // own partial [G][132] inside the stage region
constexpr uint32_t kMiscBytes = 512;

// Shared memory map of one launch (byte offsets from a 1024-byte aligned base),
// sized from the configuration so that small problems fit two blocks per SM.
struct SmemLayout {
  uint32_t q, lkeys, hist, gslice, cand, rpre, rbase, rtrip, ecnt, eslice, misc, total;
  int lkeys_cap;   // keys (floats) the lkeys region holds
  int eslice_cap;  // estimation clusters one block handles
};

enum Mode { kModeFull = 0, kModeSelect = 1, kModeAttend = 2 };

struct FusedParams {
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
  int* status;
  int G, C, M, n_steady, k_r, k_e, kr, ke, P, exec_rows, mode;
  SmemLayout L;
};

struct Misc {
  uint64_t full[kStagesA], empty[kStagesA], tfull[2], tempty[2], drain;
  uint32_t tmem;
  int abort_flag;
  int bucket[2], above[2], ncand[2];
  uint32_t Tu[2];
  int Tid[2];
  int wtot[2][kWarps];
  float red[2][kWarps];
  int scan[kWarps + 4];
  float rlo, rhi;      // this block's key range (finite keys)
  int rninf;           // this block's -inf keys
  int cntR, cntE;      // this block's R / E members
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

// Block-wide inclusive prefix of one int per thread (thread order); returns
// the exclusive prefix and writes the block total to *total.
__device__ __forceinline__ int block_excl_scan(int v, int* scratch /* [kWarps] */, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += t;
  }
  if (lane == 31) scratch[warp] = incl;
  __syncthreads();
  int excl = incl - v, tot = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    if (w < warp) excl += scratch[w];
    tot += scratch[w];
  }
  __syncthreads();
  *total = tot;
  return excl;
}

__device__ void kth_in_bucket_slow(const float* keys, bool cached, int C, int b, float lo,
                                   float scale, int k, Misc* ms, int* hist, uint32_t* Tu,
                                   int* Tid) {
  auto key = [&](int c) { return cached ? keys[c] : __ldcg(keys + c); };
  uint32_t prefix = 0, mask = 0;
  int remaining = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += kThreads) hist[i] = 0;
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += kThreads) {
      const float r = key(c);
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
  for (int base = 0; base < C; base += kThreads) {
    const int c = base + threadIdx.x;
    const float r = c < C ? key(c) : 0.f;
    const bool eq = c < C && bucket_of(r, lo, scale) == b && float_order_key(r) == prefix;
    const unsigned mk = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) ms->wtot[0][warp] = __popc(mk);
    __syncthreads();
    int before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
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

// ------------------------------------------------------------------ kernel
template <int G>
__global__ void __launch_bounds__(kThreads, G <= 4 ? 2 : 1)
    fused_decode_kernel(const __grid_constant__ CUtensorMap tm_cent, const FusedParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  cg::cluster_group cluster = cg::this_cluster();
  Misc* ms = reinterpret_cast<Misc*>(sm + p.L.misc);
  float* keys = reinterpret_cast<float*>(sm + p.L.lkeys);   // fallback key cache
  float* lkeys = keys;                                        // own chunk's keys (fast path)
  int* hist = reinterpret_cast<int*>(sm + p.L.hist);
  int* gslice = reinterpret_cast<int*>(sm + p.L.gslice);
  unsigned long long* cand = reinterpret_cast<unsigned long long*>(sm + p.L.cand);
  int32_t* rpre_sm = reinterpret_cast<int32_t*>(sm + p.L.rpre);
  int32_t* rbase_sm = reinterpret_cast<int32_t*>(sm + p.L.rbase);
  int32_t* rtrip = reinterpret_cast<int32_t*>(sm + p.L.rtrip);  // [3][kr]: id, size, row
  int32_t* eslice = reinterpret_cast<int32_t*>(sm + p.L.eslice);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x / p.P;
  const int j = blockIdx.x - bh * p.P;  // rank in the cluster
  const int C = p.C;
  const int tiles = C > 0 ? (C + kTileC - 1) / kTileC : 0;
  const int t_begin = (int)((long long)tiles * j / p.P);
  const int t_end = (int)((long long)tiles * (j + 1) / p.P);
  const int c_begin = t_begin * kTileC;
  const int c_end = min(t_end * kTileC, C);
  const int n_loc = max(0, c_end - c_begin);
  const int kr = p.kr, ke = p.ke;
  auto e_first = [&](int r) { return (int)((long long)ke * r / p.P); };
  const int e0 = e_first(j), e1 = e_first(j + 1);

  if (threadIdx.x == 0) ms->abort_flag = 0;
  __syncthreads();

  // ============================================================ phase A
  if (p.mode != kModeAttend && C > 0) {
    const int nt = t_end - t_begin;
    uint8_t* qsm = sm + p.L.q;
    if (threadIdx.x == 0) {
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
    // B operand: the unit's G query rows, zero rows up to 16, in the 128-byte
    // swizzle layout (row n, 16-byte chunk c stored at chunk c ^ (n & 7)).
    for (int i = threadIdx.x; i < 2 * kQRows * 8; i += kThreads) {
      const int kh = i / (kQRows * 8), n = (i / 8) % kQRows, c = i % 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (n < G) v = ldg_nc_v4(p.q + ((size_t)bh * G + n) * kHeadDim + kh * 64 + c * 8);
      *reinterpret_cast<uint4*>(qsm + kh * (kQRows * 128) + n * 128 + ((c ^ (n & 7)) << 4)) = v;
    }
    fence_proxy_async_smem();
    if (warp == 1) {
      tmem_alloc(&ms->tmem, 32);
      tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ms->tmem;
    if (warp == 0 && lane == 0) {
      // TMA producer
      tma_prefetch_desc(&tm_cent);
      int issued[kStagesA] = {0, 0};
      for (int it = 0; it < nt; ++it) {
        if (ms->abort_flag) break;
        const int st = it % kStagesA;
        if (it >= kStagesA && !mbar_wait(&ms->empty[st], ((it / kStagesA) - 1) & 1)) {
          record_status(p.status, RI_ERR_TIMEOUT);
          ms->abort_flag = 1;
          break;
        }
        mbar_arrive_expect_tx(&ms->full[st], kTileBytes);
        const int row = bh * C + (t_begin + it) * kTileC;
        for (int kh = 0; kh < 2; ++kh)
          tma_load_2d(sm + st * kTileBytes + kh * (kTileC * 128), &tm_cent, kh * 64,
                      row, &ms->full[st]);
        ++issued[st];
      }
      for (int st = 0; st < kStagesA; ++st)
        if (issued[st]) mbar_wait(&ms->full[st], (uint32_t)((issued[st] - 1) & 1));
    } else if (warp == 1 && lane == 0) {
      // MMA issuer: D[128 x 16] = tile[128 x 128] . Q[16 x 128]^T
      constexpr uint32_t idesc = umma_idesc_bf16_f32(kTileC, kQRows);
      const uint32_t st_addr = smem_u32(sm);
      const uint32_t q_addr = smem_u32(qsm);
      for (int it = 0; it < nt; ++it) {
        if (ms->abort_flag) break;
        const int st = it % kStagesA, buf = it & 1;
        if (!mbar_wait(&ms->full[st], (uint32_t)((it / kStagesA) & 1)) ||
            (it >= 2 && !mbar_wait(&ms->tempty[buf], (uint32_t)(((it >> 1) - 1) & 1)))) {
          record_status(p.status, RI_ERR_TIMEOUT);
          ms->abort_flag = 1;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t aoff = st * kTileBytes + (kk >> 2) * (kTileC * 128) + (kk & 3) * 32;
          const uint32_t boff = (kk >> 2) * (kQRows * 128) + (kk & 3) * 32;
          umma_bf16(tmem + buf * kQRows, umma_desc_sw128(st_addr + aoff),
                    umma_desc_sw128(q_addr + boff), idesc, kk > 0 ? 1u : 0u);
        }
        umma_commit(&ms->empty[st]);
        umma_commit(&ms->tfull[buf]);
      }
      umma_commit(&ms->drain);
      mbar_wait(&ms->drain, 0);
    } else if (warp >= 4) {
      // epilogue: one centroid per thread
      const int quad = warp & 3;
      const int r = quad * 32 + lane;
      for (int it = 0; it < nt; ++it) {
        if (ms->abort_flag) break;
        const int buf = it & 1;
        const int c = (t_begin + it) * kTileC + r;
        // issued before the wait so the load overlaps the MMA
        const int cnt = c < C ? __ldg(p.counts + (size_t)bh * C + c) : 0;
        if (!mbar_wait(&ms->tfull[buf], (uint32_t)((it >> 1) & 1))) {
          record_status(p.status, RI_ERR_TIMEOUT);
          ms->abort_flag = 1;
          break;
        }
        tc_fence_after();
        float v[16];
        tmem_ld16(tmem + ((uint32_t)(quad * 32) << 16) + buf * kQRows, v);
        tc_fence_before();
        mbar_arrive(&ms->tempty[buf]);
        if (c < C) {
          float s[8];
          float rs = 0.f;
#pragma unroll
          for (int g = 0; g < 8; ++g) {
            s[g] = g < G ? v[g] * kScale : 0.f;
            if (g < G) rs += s[g];
          }
          float4* dst = reinterpret_cast<float4*>(p.score + ((size_t)bh * C + c) * 8);
          dst[0] = make_float4(s[0], s[1], s[2], s[3]);
          dst[1] = make_float4(s[4], s[5], s[6], s[7]);
          const float key = cnt > 0 ? rs : -INFINITY;
          p.rkey[(size_t)bh * C + c] = key;
          lkeys[c - c_begin] = key;
        }
      }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 32);

  }

  // ============================================================ phase B
  // Exact selection over all C keys of the unit by every block (the
  // fallback for crowded boundary buckets): keys from the rkey workspace.
  auto select_all_keys = [&]() {
    // Thread t of round rd owns the keys of ids [rd kRound + 32 t, +32): every
    // pass below works on 32 keys held in registers (independent, unrolled).
    const float* rk = p.rkey + (size_t)bh * C;
    const bool cached = C <= p.L.lkeys_cap;
    const bool vec = (C & 3) == 0;
    if (cached) {
      if (vec) {
        for (int i = threadIdx.x; i < C / 4; i += kThreads) cp_async16(keys + 4 * i, rk + 4 * i);
      } else {
        for (int i = threadIdx.x; i < C; i += kThreads) cp_async4(keys + i, rk + i);
      }
      cp_async_commit();
      cp_async_wait<0>();
      __syncthreads();
    }
    const float* K = cached ? keys : rk;
    const int rounds = (C + kRound - 1) / kRound;
    auto load32 = [&](int rd, float (&kk)[kPer]) {
      const int c0 = rd * kRound + threadIdx.x * kPer;
      if (vec && c0 + kPer <= C) {
#pragma unroll
        for (int i = 0; i < kPer; i += 4) {
          const float4 v = cached ? *reinterpret_cast<const float4*>(K + c0 + i)
                                  : __ldcg(reinterpret_cast<const float4*>(K + c0 + i));
          kk[i] = v.x;
          kk[i + 1] = v.y;
          kk[i + 2] = v.z;
          kk[i + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
          const int c = c0 + i;
          kk[i] = c < C ? (cached ? K[c] : __ldcg(K + c)) : 0.f;
        }
      }
    };
    // 1) range of the finite keys, number of -inf keys (empty clusters)
    float lo = FLT_MAX, hi = -FLT_MAX;
    int ninf = 0;
    for (int rd = 0; rd < rounds; ++rd) {
      float kk[kPer];
      load32(rd, kk);
      const int c0 = rd * kRound + threadIdx.x * kPer;
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        if (c0 + i < C) {
          if (kk[i] == -INFINITY) {
            ++ninf;
          } else {
            lo = fminf(lo, kk[i]);
            hi = fmaxf(hi, kk[i]);
          }
        }
      }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) {
      lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
      hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
      ninf += __shfl_xor_sync(0xffffffffu, ninf, off);
    }
    if (lane == 0) {
      ms->red[0][warp] = lo;
      ms->red[1][warp] = hi;
      ms->wtot[0][warp] = ninf;
    }
    for (int i = threadIdx.x; i < kNB; i += kThreads) hist[i] = 0;
    __syncthreads();
    lo = FLT_MAX;
    hi = -FLT_MAX;
    ninf = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      lo = fminf(lo, ms->red[0][w]);
      hi = fmaxf(hi, ms->red[1][w]);
      ninf += ms->wtot[0][w];
    }
    const int nfin = C - ninf;
    const float scale = (nfin > 0 && hi > lo) ? (float)kNB / (hi - lo) : 0.f;
    // 2) histogram over value buckets (monotone in the key)
    for (int rd = 0; rd < rounds; ++rd) {
      float kk[kPer];
      load32(rd, kk);
      const int c0 = rd * kRound + threadIdx.x * kPer;
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int b = bucket_of(kk[i], lo, scale);
        if (c0 + i < C && b >= 0) atomicAdd(&hist[b], 1);
      }
    }
    __syncthreads();
    // 3) boundary buckets of ranks kA = kr and kB = kr + ke from the top:
    //    thread t owns buckets kNB-1-8t .. kNB-8-8t (descending)
    {
      int hc[kNB / kThreads];
      int sum = 0;
#pragma unroll
      for (int i = 0; i < kNB / kThreads; ++i) {
        hc[i] = hist[kNB - 1 - (kNB / kThreads) * threadIdx.x - i];
        sum += hc[i];
      }
      int incl = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
      }
      if (lane == 31) ms->scan[warp] = incl;
      if (threadIdx.x < 2) {
        const int k = threadIdx.x == 0 ? kr : kr + ke;
        ms->bucket[threadIdx.x] = k <= 0 ? -2 : (k > nfin ? -1 : -3);
        ms->above[threadIdx.x] = k > nfin ? nfin : 0;
      }
      __syncthreads();
      int excl = incl - sum;
      for (int w = 0; w < warp; ++w) excl += ms->scan[w];
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const int k = w == 0 ? kr : kr + ke;
        if (k > 0 && k <= nfin && excl < k && excl + sum >= k) {
          int cum = excl;
#pragma unroll
          for (int i = 0; i < kNB / kThreads; ++i) {
            if (cum + hc[i] >= k) {
              ms->bucket[w] = kNB - 1 - (kNB / kThreads) * threadIdx.x - i;
              ms->above[w] = cum;
              break;
            }
            cum += hc[i];
          }
        }
      }
      __syncthreads();
    }
    // 4) exact order inside each boundary bucket
    for (int w = 0; w < 2; ++w) {
      const int b = ms->bucket[w];
      if (b == -2) continue;
      const int k = (w == 0 ? kr : kr + ke) - ms->above[w];  // 1-based rank in the bucket
      const int nb = b >= 0 ? hist[b] : ninf;
      if (nb <= kBoundaryCap) {
        if (threadIdx.x == 0) ms->ncand[w] = 0;
        __syncthreads();
        for (int rd = 0; rd < rounds; ++rd) {
          float kk[kPer];
          load32(rd, kk);
          const int c0 = rd * kRound + threadIdx.x * kPer;
#pragma unroll
          for (int i = 0; i < kPer; ++i) {
            if (c0 + i < C && bucket_of(kk[i], lo, scale) == b) {
              const int slot = atomicAdd(&ms->ncand[w], 1);
              cand[w * kBoundaryCap + slot] = ord64(float_order_key(kk[i]), c0 + i);
            }
          }
        }
        __syncthreads();
        const int n = ms->ncand[w];
        for (int i = threadIdx.x; i < n; i += kThreads) {
          const unsigned long long me = cand[w * kBoundaryCap + i];
          int rank = 0;
          for (int t = 0; t < n; ++t) rank += cand[w * kBoundaryCap + t] > me;
          if (rank == k - 1) {
            ms->Tu[w] = (uint32_t)(me >> 32);
            ms->Tid[w] = (int)(0xFFFFFFFFu - (uint32_t)(me & 0xFFFFFFFFull));
          }
        }
        __syncthreads();
      } else {
        uint32_t Tu;
        int Tid;
        kth_in_bucket_slow(K, cached, C, b, lo, scale, k, ms, hist, &Tu, &Tid);
        if (threadIdx.x == 0) {
          ms->Tu[w] = Tu;
          ms->Tid[w] = Tid;
        }
        __syncthreads();
      }
    }
    const bool selA = ms->bucket[0] != -2, selB = ms->bucket[1] != -2;
    const unsigned long long TA = selA ? ord64(ms->Tu[0], ms->Tid[0]) : ~0ull;
    const unsigned long long TB = selB ? ord64(ms->Tu[1], ms->Tid[1]) : ~0ull;
    // 5) membership and compaction in id order
    const bool write_global = p.mode == kModeSelect && j == 0;
    const bool report = p.mode == kModeFull && p.sel_user != nullptr;
    int32_t* selg = p.sel + (size_t)bh * (p.k_r + p.k_e);
    int32_t* selu = p.sel_user ? p.sel_user + (size_t)bh * (p.k_r + p.k_e) : nullptr;
    int baseR = 0, baseE = 0;
    for (int rd = 0; rd < rounds; ++rd) {
      float kk[kPer];
      load32(rd, kk);
      const int c0 = rd * kRound + threadIdx.x * kPer;
      uint32_t mR = 0, mE = 0;
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        if (c0 + i < C) {
          const unsigned long long o = ord64(float_order_key(kk[i]), c0 + i);
          const bool inR = selA && o >= TA;
          const bool inE = !inR && selB && o >= TB;
          mR |= (uint32_t)inR << i;
          mE |= (uint32_t)inE << i;
        }
      }
      // block exclusive scan of (count R, count E) packed in one int
      const int v = (__popc(mR) << 16) | __popc(mE);
      int incl = v;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
      }
      if (lane == 31) ms->scan[warp] = incl;
      __syncthreads();
      int excl = incl - v, tot = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        if (w < warp) excl += ms->scan[w];
        tot += ms->scan[w];
      }
      __syncthreads();
      int pr = baseR + (excl >> 16), pe = baseE + (excl & 0xFFFF);
      while (mR) {
        const int c = c0 + __ffs(mR) - 1;
        mR &= mR - 1;
        rbase_sm[pr] = c;  // cluster ids for now; row offsets below
        if (write_global) selg[pr] = c;
        if (report && j == 0) selu[pr] = c;
        ++pr;
      }
      while (mE) {
        const int c = c0 + __ffs(mE) - 1;
        mE &= mE - 1;
        if (pe >= e0 && pe < e1) {
          eslice[pe - e0] = c;
          if (report) selu[p.k_r + pe] = c;
        }
        if (write_global) selg[p.k_r + pe] = c;
        ++pe;
      }
      baseR += tot >> 16;
      baseE += tot & 0xFFFF;
    }
    __syncthreads();
    // 6) sizes of the R clusters (prefix = execution-buffer rows) and their
    //    first rows in Kp/Vp; loads issued together, then one block scan
    {
      constexpr int kPerR = kMaxRetrieval / kThreads;  // 16
      const int per = (kr + kThreads - 1) / kThreads;
      const int i0 = min(kr, (int)threadIdx.x * per), i1 = min(kr, i0 + per);
      int cn[kPerR], of[kPerR];
#pragma unroll
      for (int u = 0; u < kPerR; ++u) {
        const int i = i0 + u;
        const bool in = i < i1;
        const int c = in ? rbase_sm[i] : 0;
        cn[u] = in ? __ldg(p.counts + (size_t)bh * C + c) : 0;
        of[u] = (in && !p.exec_rows) ? __ldg(p.offsets + (size_t)bh * (C + 1) + c) : 0;
      }
      int loc = 0;
#pragma unroll
      for (int u = 0; u < kPerR; ++u) loc += cn[u];
      int incl = loc;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += t;
      }
      if (lane == 31) ms->scan[warp] = incl;
      __syncthreads();
      int run = incl - loc, total = 0;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        if (w < warp) run += ms->scan[w];
        total += ms->scan[w];
      }
#pragma unroll
      for (int u = 0; u < kPerR; ++u) {
        const int i = i0 + u;
        if (i < i1) {
          rpre_sm[i] = run;
          rbase_sm[i] = of[u];
          run += cn[u];
        }
      }
      if (threadIdx.x == 0) rpre_sm[kr] = total;
      __syncthreads();
    }
    if (write_global) {
      for (int i = kr + threadIdx.x; i < p.k_r; i += kThreads) selg[i] = -1;
      for (int i = ke + threadIdx.x; i < p.k_e; i += kThreads) selg[p.k_r + i] = -1;
      for (int i = threadIdx.x; i <= p.k_r; i += kThreads)
        p.rpre[(size_t)bh * (p.k_r + 1) + i] = rpre_sm[i < kr ? i : kr];
      if (p.rpre_user)
        for (int i = threadIdx.x; i <= p.k_r; i += kThreads)
          p.rpre_user[(size_t)bh * (p.k_r + 1) + i] = rpre_sm[i < kr ? i : kr];
      __syncthreads();
      if (p.sel_user)
        for (int i = threadIdx.x; i < p.k_r + p.k_e; i += kThreads) selu[i] = __ldcg(selg + i);
    }
    if (report) {
      if (j == 0)
        for (int i = kr + threadIdx.x; i < p.k_r; i += kThreads) selu[i] = -1;
      if (j == p.P - 1)
        for (int i = ke + threadIdx.x; i < p.k_e; i += kThreads) selu[p.k_r + i] = -1;
    }
    __syncthreads();
  };

  if (p.mode == kModeAttend) {
    // selection left in the workspace by a select call
    const int32_t* selb = p.sel + (size_t)bh * (p.k_r + p.k_e);
    for (int i = threadIdx.x; i <= kr; i += kThreads)
      rpre_sm[i] = p.rpre[(size_t)bh * (p.k_r + 1) + i];
    for (int i = threadIdx.x; i < kr; i += kThreads)
      rbase_sm[i] = p.exec_rows ? 0 : p.offsets[(size_t)bh * (C + 1) + selb[i]];
    for (int i = e0 + threadIdx.x; i < e1; i += kThreads) eslice[i - e0] = selb[p.k_r + i];
    __syncthreads();
  } else if (C > 0) {
    // ---- B1: key range of the unit (finite keys), -inf count
    {
      float lo = FLT_MAX, hi = -FLT_MAX;
      int ninf = 0;
      for (int i = threadIdx.x; i < n_loc; i += kThreads) {
        const float r = lkeys[i];
        if (r == -INFINITY) {
          ++ninf;
        } else {
          lo = fminf(lo, r);
          hi = fmaxf(hi, r);
        }
      }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) {
        lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, off));
        hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, off));
        ninf += __shfl_xor_sync(0xffffffffu, ninf, off);
      }
      if (lane == 0) {
        ms->red[0][warp] = lo;
        ms->red[1][warp] = hi;
        ms->wtot[0][warp] = ninf;
      }
      for (int i = threadIdx.x; i < kNB; i += kThreads) hist[i] = 0;
      if (threadIdx.x < 2) ms->ncand[threadIdx.x] = 0;
      __syncthreads();
      if (threadIdx.x == 0) {
        float l2 = FLT_MAX, h2 = -FLT_MAX;
        int n2 = 0;
        for (int w = 0; w < kWarps; ++w) {
          l2 = fminf(l2, ms->red[0][w]);
          h2 = fmaxf(h2, ms->red[1][w]);
          n2 += ms->wtot[0][w];
        }
        ms->rlo = l2;
        ms->rhi = h2;
        ms->rninf = n2;
      }
    }
    cluster.sync();  // S1: every block's range; histograms and counters zeroed
    float lo = FLT_MAX, hi = -FLT_MAX;
    int ninf = 0;
    for (int r = 0; r < p.P; ++r) {
      const Misc* mr = cluster.map_shared_rank(ms, r);
      lo = fminf(lo, mr->rlo);
      hi = fmaxf(hi, mr->rhi);
      ninf += mr->rninf;
    }
    const int nfin = C - ninf;
    const float scale = (nfin > 0 && hi > lo) ? (float)kNB / (hi - lo) : 0.f;
    // ---- B2: value histogram of the unit: local histograms, then a
    //      reduce-scatter (block r sums bucket slice r over the cluster) and an
    //      all-gather of the slices, both through distributed shared memory
    for (int i = threadIdx.x; i < n_loc; i += kThreads) {
      const int b = bucket_of(lkeys[i], lo, scale);
      if (b >= 0) atomicAdd(hist + b, 1);
    }
    cluster.sync();  // S2: local histograms complete
    {
      const int b0 = kNB * j / p.P, b1 = kNB * (j + 1) / p.P;
      for (int b = b0 + threadIdx.x; b < b1; b += kThreads) {
        int sum = 0;
        for (int r = 0; r < p.P; ++r) sum += cluster.map_shared_rank(hist, r)[b];
        gslice[b - b0] = sum;
      }
    }
    cluster.sync();  // S2b: reduced slices complete; local histograms no longer read
    for (int b = threadIdx.x; b < kNB; b += kThreads) {
      int r = (int)(((long long)(b + 1) * p.P + kNB - 1) / kNB) - 1;  // slice owning b
      hist[b] = cluster.map_shared_rank(gslice, r)[b - kNB * r / p.P];
    }
    __syncthreads();
    // ---- B3: boundary buckets of ranks kA = kr and kB = kr + ke from the
    //      top; thread t owns buckets kNB-1-8t .. kNB-8-8t (descending)
    {
      int hc[kNB / kThreads];
      int sum = 0;
#pragma unroll
      for (int i = 0; i < kNB / kThreads; ++i) {
        hc[i] = hist[kNB - 1 - (kNB / kThreads) * threadIdx.x - i];
        sum += hc[i];
      }
      if (threadIdx.x < 2) {
        const int k = threadIdx.x == 0 ? kr : kr + ke;
        ms->bucket[threadIdx.x] = k <= 0 ? -2 : (k > nfin ? -1 : -3);
        ms->above[threadIdx.x] = k > nfin ? nfin : 0;
      }
      int tot;
      const int excl = block_excl_scan(sum, ms->scan, &tot);
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const int k = w == 0 ? kr : kr + ke;
        if (k > 0 && k <= nfin && excl < k && excl + sum >= k) {
          int cum = excl;
#pragma unroll
          for (int i = 0; i < kNB / kThreads; ++i) {
            if (cum + hc[i] >= k) {
              ms->bucket[w] = kNB - 1 - (kNB / kThreads) * threadIdx.x - i;
              ms->above[w] = cum;
              break;
            }
            cum += hc[i];
          }
        }
      }
      __syncthreads();
    }
    bool crowded = false;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const int b = ms->bucket[w];
      const int nb = b >= 0 ? hist[b] : (b == -1 ? ninf : 0);
      crowded |= nb > kBoundaryCap;
    }
    if (crowded) {
      cluster.sync();  // every block has gathered the slices
      select_all_keys();
    } else {
      // ---- B4: members of the boundary buckets, gathered in block 0
      unsigned long long* cand0 = cluster.map_shared_rank(cand, 0);
      int* ncand0 = cluster.map_shared_rank(&ms->ncand[0], 0);
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const int b = ms->bucket[w];
        if (b == -2) continue;
        for (int i = threadIdx.x; i < n_loc; i += kThreads) {
          const float r = lkeys[i];
          if (bucket_of(r, lo, scale) == b) {
            const int slot = atomicAdd(ncand0 + w, 1);
            cand0[w * kBoundaryCap + slot] = ord64(float_order_key(r), c_begin + i);
          }
        }
      }
      cluster.sync();  // S3
      // thresholds: the k-th member of each boundary bucket in exact order
#pragma unroll
      for (int w = 0; w < 2; ++w) {
        const int b = ms->bucket[w];
        if (b == -2) continue;
        const int n = ncand0[w];
        const int k = (w == 0 ? kr : kr + ke) - ms->above[w];
        if (j != 0)
          for (int i = threadIdx.x; i < n; i += kThreads)
            cand[w * kBoundaryCap + i] = cand0[w * kBoundaryCap + i];
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += kThreads) {
          const unsigned long long me = cand[w * kBoundaryCap + i];
          int rank = 0;
          for (int t = 0; t < n; ++t) rank += cand[w * kBoundaryCap + t] > me;
          if (rank == k - 1) {
            ms->Tu[w] = (uint32_t)(me >> 32);
            ms->Tid[w] = (int)(0xFFFFFFFFu - (uint32_t)(me & 0xFFFFFFFFull));
          }
        }
        __syncthreads();
      }
      const bool selA = ms->bucket[0] != -2, selB = ms->bucket[1] != -2;
      const unsigned long long TA = selA ? ord64(ms->Tu[0], ms->Tid[0]) : ~0ull;
      const unsigned long long TB = selB ? ord64(ms->Tu[1], ms->Tid[1]) : ~0ull;
      // ---- B5: this block's members, in id order: thread t owns the local
      //      keys [t kk, t kk + kk); positions from a block scan and the
      //      cluster prefix of the blocks' member counts
      const int kk = (n_loc + kThreads - 1) / kThreads;  // <= 32 (n_loc <= 8192)
      const int l0 = min(n_loc, (int)threadIdx.x * kk), l1 = min(n_loc, l0 + kk);
      uint32_t mR = 0, mE = 0;
      for (int i = l0; i < l1; ++i) {
        const unsigned long long o = ord64(float_order_key(lkeys[i]), c_begin + i);
        const bool inR = selA && o >= TA;
        const bool inE = !inR && selB && o >= TB;
        mR |= (uint32_t)inR << (i - l0);
        mE |= (uint32_t)inE << (i - l0);
      }
      int tot;
      const int x = block_excl_scan((__popc(mR) << 16) | __popc(mE), ms->scan, &tot);
      if (threadIdx.x == 0) {
        ms->cntR = tot >> 16;
        ms->cntE = tot & 0xFFFF;
      }
      cluster.sync();  // S4
      int baseR = 0, baseE = 0;
      for (int r = 0; r < j; ++r) {
        const Misc* mr = cluster.map_shared_rank(ms, r);
        baseR += mr->cntR;
        baseE += mr->cntE;
      }
      const bool write_global = p.mode == kModeSelect;
      const bool report = p.mode == kModeFull && p.sel_user != nullptr;
      int32_t* selg = p.sel + (size_t)bh * (p.k_r + p.k_e);
      int32_t* selu = p.sel_user ? p.sel_user + (size_t)bh * (p.k_r + p.k_e) : nullptr;
      // R members: (id, size, first row) to block 0
      int32_t* rtrip0 = cluster.map_shared_rank(rtrip, 0);
      int pr = baseR + (x >> 16), pe = baseE + (x & 0xFFFF);
      while (mR) {
        const int c = c_begin + l0 + __ffs(mR) - 1;
        mR &= mR - 1;
        rtrip0[pr] = c;
        rtrip0[kr + pr] = __ldg(p.counts + (size_t)bh * C + c);
        rtrip0[2 * kr + pr] = p.exec_rows ? 0 : __ldg(p.offsets + (size_t)bh * (C + 1) + c);
        if (write_global) selg[pr] = c;
        if (report) selu[pr] = c;
        ++pr;
      }
      // E members: each id to the block that attends it
      while (mE) {
        const int c = c_begin + l0 + __ffs(mE) - 1;
        mE &= mE - 1;
        const int owner = (int)(((long long)(pe + 1) * p.P + ke - 1) / ke) - 1;
        cluster.map_shared_rank(eslice, owner)[pe - e_first(owner)] = c;
        if (write_global) selg[p.k_r + pe] = c;
        if (report) selu[p.k_r + pe] = c;
        ++pe;
      }
      cluster.sync();  // S5: R triples complete in block 0, E slices in their blocks
      // ---- B6: prefix of the R clusters' sizes (execution-buffer rows)
      constexpr int kPerR = kMaxRetrieval / kThreads;  // 16
      const int per = (kr + kThreads - 1) / kThreads;
      const int i0 = min(kr, (int)threadIdx.x * per), i1 = min(kr, i0 + per);
      int cn[kPerR], of[kPerR];
#pragma unroll
      for (int u = 0; u < kPerR; ++u) {
        const bool in = i0 + u < i1;
        cn[u] = in ? rtrip0[kr + i0 + u] : 0;
        of[u] = in ? rtrip0[2 * kr + i0 + u] : 0;
      }
      int loc = 0;
#pragma unroll
      for (int u = 0; u < kPerR; ++u) loc += cn[u];
      int total;
      int run = block_excl_scan(loc, ms->scan, &total);
#pragma unroll
      for (int u = 0; u < kPerR; ++u) {
        const int i = i0 + u;
        if (i < i1) {
          rpre_sm[i] = run;
          rbase_sm[i] = of[u];
          run += cn[u];
        }
      }
      if (threadIdx.x == 0) rpre_sm[kr] = total;
      __syncthreads();
      if (j == 0 && (write_global || report)) {
        // tails of the id lists and the execution-buffer prefix
        int32_t* dst = write_global ? selg : selu;
        for (int i = kr + threadIdx.x; i < p.k_r; i += kThreads) {
          if (write_global) selg[i] = -1;
          if (p.sel_user) p.sel_user[(size_t)bh * (p.k_r + p.k_e) + i] = -1;
        }
        for (int i = ke + threadIdx.x; i < p.k_e; i += kThreads) {
          if (write_global) selg[p.k_r + i] = -1;
          if (p.sel_user) p.sel_user[(size_t)bh * (p.k_r + p.k_e) + p.k_r + i] = -1;
        }
        (void)dst;
        if (write_global) {
          for (int i = threadIdx.x; i <= p.k_r; i += kThreads)
            p.rpre[(size_t)bh * (p.k_r + 1) + i] = rpre_sm[i < kr ? i : kr];
          if (p.rpre_user)
            for (int i = threadIdx.x; i <= p.k_r; i += kThreads)
              p.rpre_user[(size_t)bh * (p.k_r + 1) + i] = rpre_sm[i < kr ? i : kr];
        }
      }
      if (write_global && p.sel_user)
        for (int i = threadIdx.x; i < kr; i += kThreads)
          p.sel_user[(size_t)bh * (p.k_r + p.k_e) + i] = rtrip0[i];
      if (write_global && p.sel_user)
        for (int i = e0 + threadIdx.x; i < e1; i += kThreads)
          p.sel_user[(size_t)bh * (p.k_r + p.k_e) + p.k_r + i] = eslice[i - e0];
    }
  } else {
    if (threadIdx.x == 0) rpre_sm[0] = 0;
    if (p.mode != kModeAttend && p.sel_user && j == 0)
      for (int i = threadIdx.x; i < p.k_r + p.k_e; i += kThreads)
        p.sel_user[(size_t)bh * (p.k_r + p.k_e) + i] = -1;
    if (p.mode == kModeSelect && j == 0) {
      int32_t* selg = p.sel + (size_t)bh * (p.k_r + p.k_e);
      for (int i = threadIdx.x; i < p.k_r + p.k_e; i += kThreads) selg[i] = -1;
      for (int i = threadIdx.x; i <= p.k_r; i += kThreads) {
        p.rpre[(size_t)bh * (p.k_r + 1) + i] = 0;
        if (p.rpre_user) p.rpre_user[(size_t)bh * (p.k_r + 1) + i] = 0;
      }
    }
    __syncthreads();
  }

  if (p.mode == kModeSelect) {
    cluster.sync();  // block 0's R triples were read by every block
    return;
  }

  // ============================================================ phase C
  // Work items of this block: tokens [t0, t1) of steady + retrieval, then
  // estimation clusters [e0, e1).  They are brought into shared memory in
  // chunks by 16-byte cp.async copies (double buffered: the next chunk is in
  // flight while the current one is consumed); a 16-lane group handles one
  // token or cluster at a time, lane l16 owning dims 8 l16 .. 8 l16 + 7.
  const int l16 = threadIdx.x & 15;
  const int hw = threadIdx.x >> 4;  // 16 half-warps
  float qv[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const uint4 raw = ldg_nc_v4(p.q + ((size_t)bh * G + g) * kHeadDim + l16 * 8);
    bf16x8_to_float(raw, qv[g]);
  }
  float m[G], l[G], o[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    m[g] = -INFINITY;
    l[g] = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) o[g][i] = 0.f;
  }
  const long long T_R = C > 0 ? rpre_sm[kr] : 0;
  const long long T = p.n_steady + T_R;
  const long long t0 = T * j / p.P, t1 = T * (j + 1) / p.P;
  const size_t steady_base = (size_t)bh * p.n_steady * kHeadDim;
  const size_t rbase_rows = p.exec_rows ? (size_t)bh * p.exec_rows : (size_t)bh * p.M;
  const long long lim_rows = p.exec_rows ? p.exec_rows : p.M;
  // Everything this block reads below is first requested into L2 in bulk,
  // so the chunked copies wait on L2 rather than on a round trip to HBM each.
  {
    const long long s_end = min(t1, (long long)p.n_steady);
    if (threadIdx.x == 0 && t0 < s_end) {
      const uint32_t bytes = (uint32_t)((s_end - t0) * kHeadDim * 2);
      prefetch_l2_bulk(p.Ks + steady_base + (size_t)t0 * kHeadDim, bytes);
      prefetch_l2_bulk(p.Vs + steady_base + (size_t)t0 * kHeadDim, bytes);
    }
    const long long r0 = max(t0, (long long)p.n_steady) - p.n_steady;
    const long long r1 = t1 - p.n_steady;
    if (r1 > r0) {
      if (p.exec_rows) {
        if (threadIdx.x == 0 && r1 <= p.exec_rows) {
          const uint32_t bytes = (uint32_t)((r1 - r0) * kHeadDim * 2);
          prefetch_l2_bulk(p.Kr + (rbase_rows + (size_t)r0) * kHeadDim, bytes);
          prefetch_l2_bulk(p.Vr + (rbase_rows + (size_t)r0) * kHeadDim, bytes);
        }
      } else {
        int first = 0, hi = kr - 1;  // last cluster with rpre <= r0
        while (first < hi) {
          const int mid = (first + hi + 1) >> 1;
          if (rpre_sm[mid] <= r0) first = mid; else hi = mid - 1;
        }
        for (int i = first + threadIdx.x; i < kr && rpre_sm[i] < r1; i += kThreads) {
          const long long a = max((long long)rpre_sm[i], r0);
          const long long b = min((long long)rpre_sm[i + 1], r1);
          const long long row = (long long)rbase_sm[i] + (a - rpre_sm[i]);
          if (b > a && row >= 0 && row + (b - a) <= lim_rows) {
            const uint32_t bytes = (uint32_t)((b - a) * kHeadDim * 2);
            prefetch_l2_bulk(p.Kr + (rbase_rows + (size_t)row) * kHeadDim, bytes);
            prefetch_l2_bulk(p.Vr + (rbase_rows + (size_t)row) * kHeadDim, bytes);
          }
        }
      }
    }
    for (int e = e0 + threadIdx.x; e < e1; e += kThreads) {
      const int c = eslice[e - e0];
      prefetch_l2_bulk(p.vsum + ((size_t)bh * C + c) * kHeadDim, kHeadDim * 4);
      prefetch_l2_bulk(p.score + ((size_t)bh * C + c) * 8, 32);
      prefetch_l2(p.counts + (size_t)bh * C + c);
    }
  }
  const int n_tok_chunks = (int)((t1 - t0 + kTokChunk - 1) / kTokChunk);
  const int n_e_chunks = (e1 - e0 + kEChunk - 1) / kEChunk;
  const int n_chunks = n_tok_chunks + n_e_chunks;
  uint8_t* cbuf = sm;                                      // [kChunkBufs][kChunkBytes]
  int* ecnt = reinterpret_cast<int*>(sm + p.L.ecnt);       // [kChunkBufs][kEChunk]

  // issue the copies of chunk k into buffer k % 3 (4 threads per item)
  auto issue = [&](int k) {
    uint8_t* buf = cbuf + (k % kChunkBufs) * kChunkBytes;
    const int slot = threadIdx.x >> 2, part = threadIdx.x & 3;
    if (k < n_tok_chunks) {
      const long long tok = t0 + (long long)k * kTokChunk + slot;
      if (slot < kTokChunk && tok < t1) {
        const __nv_bfloat16* kp = nullptr;
        const __nv_bfloat16* vp = nullptr;
        if (tok < p.n_steady) {
          kp = p.Ks + steady_base + (size_t)tok * kHeadDim;
          vp = p.Vs + steady_base + (size_t)tok * kHeadDim;
        } else {
          const int tt = (int)(tok - p.n_steady);
          long long row;
          if (p.exec_rows) {
            row = tt;
          } else {
            int lo = 0, hi = kr - 1;
            while (lo < hi) {
              const int mid = (lo + hi + 1) >> 1;
              if (rpre_sm[mid] <= tt) lo = mid; else hi = mid - 1;
            }
            row = (long long)rbase_sm[lo] + (tt - rpre_sm[lo]);
          }
          // rows outside the source buffer (an inconsistent index, or an
          // execution buffer smaller than the selection) are zero, flagged
          if (row >= 0 && row < lim_rows) {
            kp = p.Kr + (rbase_rows + (size_t)row) * kHeadDim;
            vp = p.Vr + (rbase_rows + (size_t)row) * kHeadDim;
          } else if (part == 0) {
            record_status(p.status, RI_ERR_INVALID_ARG);
          }
        }
        uint8_t* dst = buf + slot * 512;
        if (kp) {
          // parts 0-1: K row halves, parts 2-3: V row halves (128 bytes each)
          const uint8_t* src = reinterpret_cast<const uint8_t*>(part < 2 ? kp : vp) + (part & 1) * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) cp_async16(dst + part * 128 + c * 16, src + c * 16);
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(dst + part * 128 + c * 16) = make_uint4(0, 0, 0, 0);
        }
      }
    } else {
      const int e = e0 + (k - n_tok_chunks) * kEChunk + slot;
      if (slot < kEChunk && e < e1) {
        const int c = eslice[e - e0];
        uint8_t* dst = buf + slot * 544;
        const uint8_t* vs = reinterpret_cast<const uint8_t*>(p.vsum + ((size_t)bh * C + c) * kHeadDim);
#pragma unroll
        for (int q = 0; q < 8; ++q) cp_async16(dst + part * 128 + q * 16, vs + part * 128 + q * 16);
        if (part == 0) {
          const uint8_t* sc = reinterpret_cast<const uint8_t*>(p.score + ((size_t)bh * C + c) * 8);
          cp_async16(dst + 512, sc);
          cp_async16(dst + 528, sc + 16);
        } else if (part == 1) {
          cp_async4(&ecnt[(k % kChunkBufs) * kEChunk + slot], p.counts + (size_t)bh * C + c);
        }
      }
    }
  };

  for (int k = 0; k < kChunkBufs - 1; ++k) {
    if (k < n_chunks) issue(k);
    cp_async_commit();
  }
  for (int k = 0; k < n_chunks; ++k) {
    if (k + kChunkBufs - 1 < n_chunks) issue(k + kChunkBufs - 1);
    cp_async_commit();
    cp_async_wait<kChunkBufs - 1>();
    __syncthreads();
    const uint8_t* buf = cbuf + (k % kChunkBufs) * kChunkBytes;
    if (k < n_tok_chunks) {
      const long long base = t0 + (long long)k * kTokChunk;
      const int nitems = (int)min((long long)kTokChunk, t1 - base);
      // every 16-lane group runs the same trip count (the shuffles are warp-wide)
#pragma unroll
      for (int u = 0; u < kTokChunk / 16; ++u) {
        const int slot = u * 16 + hw;
        const bool live = slot < nitems;
        const uint8_t* row = buf + (live ? slot : 0) * 512;
        float kf[8], vf[8];
        bf16x8_to_float(*reinterpret_cast<const uint4*>(row + l16 * 16), kf);
        bf16x8_to_float(*reinterpret_cast<const uint4*>(row + 256 + l16 * 16), vf);
        float x[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float a = 0.f;
#pragma unroll
          for (int i = 0; i < 8; ++i) a = fmaf(qv[g][i], kf[i], a);
          x[g] = a;
        }
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1)
#pragma unroll
          for (int g = 0; g < G; ++g) x[g] += __shfl_xor_sync(0xffffffffu, x[g], off);
        if (live) {
#pragma unroll
          for (int g = 0; g < G; ++g) {
            const float s = x[g] * kScale;
            const float mn = fmaxf(m[g], s);
            const float corr = __expf(m[g] - mn);
            const float pw = __expf(s - mn);
            l[g] = l[g] * corr + pw;
#pragma unroll
            for (int i = 0; i < 8; ++i) o[g][i] = fmaf(o[g][i], corr, pw * vf[i]);
            m[g] = mn;
          }
        }
      }
    } else {
      const int base = e0 + (k - n_tok_chunks) * kEChunk;
      const int nitems = min(kEChunk, e1 - base);
      for (int slot = hw; slot < nitems; slot += 16) {
        const int n = ecnt[(k % kChunkBufs) * kEChunk + slot];
        if (n <= 0) continue;
        const uint8_t* row = buf + slot * 544;
        const float4 v0 = *reinterpret_cast<const float4*>(row + l16 * 32);
        const float4 v1 = *reinterpret_cast<const float4*>(row + l16 * 32 + 16);
        const float vv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        const float* sc = reinterpret_cast<const float*>(row + 512);
        const float nf = (float)n;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float s = sc[g];
          const float mn = fmaxf(m[g], s);
          const float corr = __expf(m[g] - mn);
          const float pw = __expf(s - mn);
          l[g] = l[g] * corr + nf * pw;
#pragma unroll
          for (int i = 0; i < 8; ++i) o[g][i] = fmaf(o[g][i], corr, pw * vv[i]);
          m[g] = mn;
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  // merge the two half-warps of each warp (lanes l and l + 16 hold the same dims)
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float mo = __shfl_xor_sync(0xffffffffu, m[g], 16);
    const float lo2 = __shfl_xor_sync(0xffffffffu, l[g], 16);
    const float mn = fmaxf(m[g], mo);
    const float fa = mn == -INFINITY ? 0.f : __expf(m[g] - mn);
    const float fb = mn == -INFINITY ? 0.f : __expf(mo - mn);
    l[g] = l[g] * fa + lo2 * fb;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float oo = __shfl_xor_sync(0xffffffffu, o[g][i], 16);
      o[g][i] = o[g][i] * fa + oo * fb;
    }
    m[g] = mn;
  }
  // block merge over the 8 warps, then this block's partial into shared memory
  float* wst = reinterpret_cast<float*>(sm);  // [8 warps][G][132]
  float* mypart = reinterpret_cast<float*>(sm + kPartOff);  // [G][132]
  __syncthreads();
  if (lane < 16) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float* row = wst + ((size_t)warp * G + g) * kPartStride;
      if (lane == 0) {
        row[0] = m[g];
        row[1] = l[g];
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) row[4 + l16 * 8 + i] = o[g][i];
    }
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < G * kHeadDim; idx += kThreads) {
    const int g = idx / kHeadDim, dd = idx % kHeadDim;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) mx = fmaxf(mx, wst[((size_t)w * G + g) * kPartStride]);
    float ls = 0.f, os = 0.f;
    if (mx != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float* row = wst + ((size_t)w * G + g) * kPartStride;
        const float f = __expf(row[0] - mx);
        ls += row[1] * f;
        os += row[4 + dd] * f;
      }
    }
    mypart[(size_t)g * kPartStride + 4 + dd] = os;
    if (dd == 0) {
      mypart[(size_t)g * kPartStride + 0] = mx;
      mypart[(size_t)g * kPartStride + 1] = ls;
    }
  }
  // ============================================================ phase D
  cluster.sync();  // S6: every block's partial is in its shared memory
  if (j == 0) {
    for (int idx = threadIdx.x; idx < G * kHeadDim; idx += kThreads) {
      const int g = idx / kHeadDim, dd = idx % kHeadDim;
      float mr[kMaxClusterBlocks], lr[kMaxClusterBlocks], orr[kMaxClusterBlocks];
      float mx = -INFINITY;
#pragma unroll
      for (int r = 0; r < kMaxClusterBlocks; ++r) {
        if (r < p.P) {
          const float* rp = cluster.map_shared_rank(mypart, r) + (size_t)g * kPartStride;
          mr[r] = rp[0];
          lr[r] = rp[1];
          orr[r] = rp[4 + dd];
          mx = fmaxf(mx, mr[r]);
        }
      }
      float ls = 0.f, os = 0.f;
      if (mx != -INFINITY) {
#pragma unroll
        for (int r = 0; r < kMaxClusterBlocks; ++r) {
          if (r < p.P) {
            const float f = __expf(mr[r] - mx);
            ls += lr[r] * f;
            os += orr[r] * f;
          }
        }
      }
      // no token and no cluster contributed (empty steady zone and budgets): 0, lse -inf
      const bool any = ls > 0.f;
      const size_t hq = (size_t)bh * G + g;
      p.out[hq * kHeadDim + dd] = __float2bfloat16_rn(any ? os / ls : 0.f);
      if (p.lse && dd == 0) p.lse[hq] = any ? mx + logf(ls) : -INFINITY;
    }
  }
  cluster.sync();  // S7: block 0 is done reading the other blocks' partials
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

template <int G>
cudaError_t prepare_kernel() {
  auto kern = fused_decode_kernel<G>;
  cudaError_t e = set_smem_once(reinterpret_cast<const void*>(kern), 232448);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
}

SmemLayout make_smem_layout(const Geometry& g, int kr, int ke, int P) {
  SmemLayout s;
  uint32_t off = kStageBytes;
  auto take = [&](uint32_t bytes) {
    const uint32_t o = off;
    off = (off + bytes + 15u) & ~15u;
    return o;
  };
  s.q = take(2 * kQRows * 128);  // 1024-aligned: right after the 64 KB stage region
  const int tiles = g.C > 0 ? (g.C + kTileC - 1) / kTileC : 1;
  const int per = (tiles + P - 1) / P;
  s.lkeys_cap = per * kTileC;
  s.lkeys = take((uint32_t)s.lkeys_cap * 4);
  s.hist = take(kNB * 4);
  s.gslice = take((kNB / P + 8) * 4);
  s.cand = take(2 * kBoundaryCap * 8);
  s.rpre = take((uint32_t)(kr + 4) * 4);
  s.rbase = take((uint32_t)(kr + 4) * 4);
  s.rtrip = take((uint32_t)(3 * kr + 4) * 4);
  s.ecnt = take(kChunkBufs * kEChunk * 4);
  s.eslice_cap = (ke + P - 1) / P + 1;
  s.eslice = take((uint32_t)s.eslice_cap * 4);
  s.misc = take(kMiscBytes);
  s.total = off + 1024;  // alignment slack of the dynamic shared memory base
  return s;
}

template <int G>
int active_clusters(int P, uint32_t smem) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)P);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)P;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (prepare_kernel<G>() != cudaSuccess ||
      cudaOccupancyMaxActiveClusters(&n, fused_decode_kernel<G>, &cfg) != cudaSuccess)
    n = 0;
  cudaGetLastError();
  return n;
}

int active_clusters_g(int G, int P, uint32_t smem) {
  switch (G) {
    case 1: return active_clusters<1>(P, smem);
    case 2: return active_clusters<2>(P, smem);
    case 3: return active_clusters<3>(P, smem);
    case 4: return active_clusters<4>(P, smem);
    case 5: return active_clusters<5>(P, smem);
    case 6: return active_clusters<6>(P, smem);
    case 7: return active_clusters<7>(P, smem);
    default: return active_clusters<8>(P, smem);
  }
}

template <int G>
cudaError_t launch_fused_g(const Geometry& g, const DecodeLayout& L, const DecodeArgs& a,
                           int mode, cudaStream_t s) {
  FusedParams p;
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
  p.status = reinterpret_cast<int*>(a.ws);
  p.G = G;
  p.C = g.C;
  p.M = g.M;
  p.n_steady = g.n_steady;
  p.k_r = L.k_r;
  p.k_e = L.k_e;
  p.kr = L.kr;
  p.ke = L.ke;
  p.P = L.P;
  p.exec_rows = exec ? a.exec_rows : 0;
  p.mode = mode;
  p.L = make_smem_layout(g, L.kr, L.ke, L.P);

  CUtensorMap map;
  memset(&map, 0, sizeof(map));
  if (g.C > 0) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cudaErrorNotSupported;
    cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)g.BH() * g.C};
    cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)kTileC};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.centroid), dims,
           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  cudaError_t e = prepare_kernel<G>();
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(g.BH() * L.P));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = p.L.total;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)L.P;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fused_decode_kernel<G>, map, p);
}

cudaError_t launch_fused(const Geometry& g, const DecodeLayout& L, const DecodeArgs& a, int mode,
                         cudaStream_t s) {
  switch (g.G) {
    case 1: return launch_fused_g<1>(g, L, a, mode, s);
    case 2: return launch_fused_g<2>(g, L, a, mode, s);
    case 3: return launch_fused_g<3>(g, L, a, mode, s);
    case 4: return launch_fused_g<4>(g, L, a, mode, s);
    case 5: return launch_fused_g<5>(g, L, a, mode, s);
    case 6: return launch_fused_g<6>(g, L, a, mode, s);
    case 7: return launch_fused_g<7>(g, L, a, mode, s);
    default: return launch_fused_g<8>(g, L, a, mode, s);
  }
}

}  // namespace

// Blocks per unit of the decode kernel (one thread-block cluster, <= 16):
// the largest P whose clusters all fit on the device at once (one wave),
// with at least ceil(C / 8192) blocks so a block's keys fit its local mask.
// Without a device the plan is P = 16 capped by the tiles.
bool decode_plan(const Geometry& g, DecodeLayout* L) {
  const int tiles = g.C > 0 ? (g.C + kTileC - 1) / kTileC : 1;
  const int pmin = g.C > 0 ? (g.C + 8191) / 8192 : 1;
  const int pmax = tiles < kMaxClusterBlocks ? tiles : kMaxClusterBlocks;
  if (pmin > kMaxClusterBlocks) {
    set_error("%d clusters per head: more than %d blocks per head needed", g.C,
              kMaxClusterBlocks);
    return false;
  }
  int dev = -1;
  const bool have_dev = cudaGetDevice(&dev) == cudaSuccess;
  cudaGetLastError();
  const long long units = g.BH();
  int chosen = -1, fallback = -1;
  for (int P = pmax; P >= pmin && P >= 1; --P) {
    // balance: the same critical path with fewer blocks
    const int per = (tiles + P - 1) / P;
    const int Pb = (tiles + per - 1) / per;
    if (Pb != P) continue;
    const SmemLayout s = make_smem_layout(g, L->kr, L->ke, P);
    if (s.total > 232448) continue;
    if (!have_dev) {
      chosen = P;
      break;
    }
    static std::mutex mu;
    static std::map<std::tuple<int, int, int, uint32_t>, int> cache;
    int n;
    {
      std::lock_guard<std::mutex> lk(mu);
      auto key = std::make_tuple(dev, g.G, P, s.total);
      auto it = cache.find(key);
      if (it == cache.end()) it = cache.emplace(key, active_clusters_g(g.G, P, s.total)).first;
      n = it->second;
    }
    if (n <= 0) continue;
    if (fallback < 0) fallback = P;
    if (n >= units) {
      chosen = P;
      break;
    }
  }
  if (chosen < 0) chosen = fallback;
  if (chosen < 0) {
    set_error("no launchable decode configuration (C = %d, k_r = %d, k_e = %d)", g.C, L->kr,
              L->ke);
    return false;
  }
  L->P = chosen;
  return true;
}

cudaError_t launch_select(const Geometry& g, const DecodeLayout& L, const DecodeArgs& a,
                          cudaStream_t s) {
  return launch_fused(g, L, a, kModeSelect, s);
}

cudaError_t launch_attend(const Geometry& g, const DecodeLayout& L, const DecodeArgs& a,
                          cudaStream_t s) {
  return launch_fused(g, L, a, kModeAttend, s);
}

cudaError_t launch_decode(const Geometry& g, const DecodeLayout& L, const DecodeArgs& a,
                          cudaStream_t s) {
  return launch_fused(g, L, a, kModeFull, s);
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
    __nanosleep(1000);
  }
}

cudaError_t launch_wait_timeout_selftest(int* status, unsigned long long limit_ns,
                                         cudaStream_t s) {
  wait_timeout_kernel<<<1, 1, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace ri
