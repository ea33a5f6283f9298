// Tripartite decode attention over the wave index (sm_100a).
//
// Steps (RetroInfer; "KV缓存技术与RetroInfer系统在长上下文推理中的优化实践",
// framerc.cn, §2.1 zones, §2.2 step 1 index query, §3.3 attention over the
// zones and merge of the partial results):
//   S1 centroid scoring   s[g][c] = q_g . centroid_c / sqrt(d), key r_c = sum_g s
//   S2 cluster selection  R = top k_r by (r desc, id asc), E = the next k_e
//   S4 exact partials     split-K flash decode over steady + R tokens
//   S5 estimation term    each c in E adds n_c e^{s} / e^{s} Vsum_c
//   S6 merge              log-sum-exp over the split partials
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace ri {

namespace {

constexpr float kScale = 0.08838834764831845f;  // 1/sqrt(128)
constexpr int kScoreCentroidsPerBlock = 256;
constexpr int kMaxRetrievalInSmem = 8192;

// ------------------------------------------------------------------- S1
// Half-warp per centroid: lane l16 holds dims [8 l16, 8 l16 + 8).  Four
// centroids in flight per half-warp.
template <int G>
__global__ void __launch_bounds__(256) score_kernel(const __nv_bfloat16* __restrict__ q,
                                                    const __nv_bfloat16* __restrict__ centroid,
                                                    const int32_t* __restrict__ counts,
                                                    float* __restrict__ score,
                                                    float* __restrict__ rkey, int C) {
  const int bh = blockIdx.y;
  const int l16 = threadIdx.x & 15;
  const int hw = threadIdx.x >> 4;  // 0..15
  float qv[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    uint4 raw = ldg_nc_v4(q + ((size_t)bh * G + g) * kHeadDim + l16 * 8);
    bf16x8_to_float(raw, qv[g]);
  }
  const int c_begin = blockIdx.x * kScoreCentroidsPerBlock;
  const int c_end = min(c_begin + kScoreCentroidsPerBlock, C);
  const __nv_bfloat16* cbase = centroid + (size_t)bh * C * kHeadDim + l16 * 8;
  // The loop bound uses the warp's even half so both halves of a warp run
  // the same trip count (the shuffles below are warp-wide).
  for (int c0 = c_begin + hw; c0 - (hw & 1) < c_end; c0 += 16 * 4) {
    uint4 raw[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = c0 + u * 16;
      raw[u] = c < c_end ? ldg_nc_v4(cbase + (size_t)c * kHeadDim) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int c = c0 + u * 16;
      float k[8];
      bf16x8_to_float(raw[u], k);
      float acc[G];
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float a = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) a = fmaf(qv[g][i], k[i], a);
        acc[g] = a;
      }
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1)
#pragma unroll
        for (int g = 0; g < G; ++g) acc[g] += __shfl_xor_sync(0xffffffffu, acc[g], off);
      if (l16 == 0 && c < c_end) {
        float r = 0.f;
#pragma unroll
        for (int g = 0; g < G; ++g) {
          const float s = acc[g] * kScale;
          score[((size_t)bh * G + g) * C + c] = s;
          r += s;
        }
        rkey[(size_t)bh * C + c] = counts[(size_t)bh * C + c] > 0 ? r : -INFINITY;
      }
    }
  }
}

// ------------------------------------------------------------------- S2
// Block-wide exclusive prefix of two predicates (1024 threads, id order).
struct Scan2 {
  int ex_a, ex_b, tot_a, tot_b;
};

__device__ __forceinline__ Scan2 block_scan2(bool a, bool b, int* sm /* [2][32] */) {
  const unsigned lane = lane_id();
  const unsigned warp = threadIdx.x >> 5;
  const unsigned lt = (1u << lane) - 1u;
  const unsigned ma = __ballot_sync(0xffffffffu, a);
  const unsigned mb = __ballot_sync(0xffffffffu, b);
  if (lane == 0) {
    sm[warp] = __popc(ma);
    sm[32 + warp] = __popc(mb);
  }
  __syncthreads();
  if (warp == 0) {
    int va = sm[lane], vb = sm[32 + lane];
    int ia = va, ib = vb;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      int ta = __shfl_up_sync(0xffffffffu, ia, off);
      int tb = __shfl_up_sync(0xffffffffu, ib, off);
      if ((int)lane >= off) {
        ia += ta;
        ib += tb;
      }
    }
    sm[lane] = ia - va;  // exclusive
    sm[32 + lane] = ib - vb;
    if (lane == 31) {
      sm[64] = ia;
      sm[65] = ib;
    }
  }
  __syncthreads();
  Scan2 r;
  r.ex_a = sm[warp] + __popc(ma & lt);
  r.ex_b = sm[32 + warp] + __popc(mb & lt);
  r.tot_a = sm[64];
  r.tot_b = sm[65];
  __syncthreads();
  return r;
}

// Radix select of the k-th largest key (k >= 1): returns the key T and the
// number of keys strictly greater than T.
__device__ void radix_threshold(const float* __restrict__ r, int C, int k, uint32_t* T_out,
                                int* ngt_out, uint32_t* hist /*[256]*/, int* sm) {
  uint32_t prefix = 0, mask = 0;
  int remaining = k;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += blockDim.x) {
      const uint32_t u = float_order_key(r[c]);
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      // lane l owns digits 255-8l .. 248-8l (descending)
      const unsigned lane = threadIdx.x;
      int cnt[8];
      int sum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        cnt[i] = hist[255 - 8 * lane - i];
        sum += cnt[i];
      }
      int incl = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, incl, off);
        if ((int)lane >= off) incl += t;
      }
      const int excl = incl - sum;
      const bool here = excl < remaining && incl >= remaining;
      if (here) {
        int cum = excl;
        for (int i = 0; i < 8; ++i) {
          if (cum + cnt[i] >= remaining) {
            sm[0] = 255 - 8 * lane - i;
            sm[1] = remaining - cum;
            break;
          }
          cum += cnt[i];
        }
      }
    }
    __syncthreads();
    const uint32_t digit = (uint32_t)sm[0];
    remaining = sm[1];
    prefix |= digit << shift;
    mask |= 255u << shift;
    __syncthreads();
  }
  *T_out = prefix;
  *ngt_out = k - remaining;
}

__global__ void __launch_bounds__(1024) select_kernel(const float* __restrict__ rkey,
                                                      const int32_t* __restrict__ counts,
                                                      const int32_t* __restrict__ offsets,
                                                      int32_t* __restrict__ sel,
                                                      int32_t* __restrict__ rpre,
                                                      int32_t* __restrict__ sel_user,
                                                      int32_t* __restrict__ rpre_user, int C,
                                                      int k_r, int k_e, int kr, int ke) {
  __shared__ uint32_t hist[256];
  __shared__ int sm[72];
  const int bh = blockIdx.x;
  const float* r = rkey + (size_t)bh * C;
  const int kA = kr, kB = kr + ke;
  uint32_t TA = 0, TB = 0;
  int ngtA = 0, ngtB = 0;
  if (kA > 0) radix_threshold(r, C, kA, &TA, &ngtA, hist, sm);
  if (kB > 0) {
    if (kB == kA) {
      TB = TA;
      ngtB = ngtA;
    } else {
      radix_threshold(r, C, kB, &TB, &ngtB, hist, sm);
    }
  }
  const int tieA = kA - ngtA, tieB = kB - ngtB;
  int32_t* selb = sel + (size_t)bh * (k_r + k_e);
  int runEqA = 0, runEqB = 0, runR = 0, runE = 0;
  for (int base = 0; base < C; base += blockDim.x) {
    const int c = base + threadIdx.x;
    const bool valid = c < C;
    const uint32_t u = valid ? float_order_key(r[c]) : 0u;
    const bool eqA = valid && kA > 0 && u == TA;
    const bool eqB = valid && kB > 0 && u == TB;
    Scan2 s1 = block_scan2(eqA, eqB, sm);
    const bool inA = valid && kA > 0 && (u > TA || (eqA && runEqA + s1.ex_a < tieA));
    const bool inB = valid && kB > 0 && (u > TB || (eqB && runEqB + s1.ex_b < tieB));
    const bool inE = inB && !inA;
    Scan2 s2 = block_scan2(inA, inE, sm);
    if (inA) selb[runR + s2.ex_a] = c;
    if (inE) selb[k_r + runE + s2.ex_b] = c;
    runEqA += s1.tot_a;
    runEqB += s1.tot_b;
    runR += s2.tot_a;
    runE += s2.tot_b;
  }
  __syncthreads();
  // unused slots
  for (int i = kr + threadIdx.x; i < k_r; i += blockDim.x) selb[i] = -1;
  for (int i = ke + threadIdx.x; i < k_e; i += blockDim.x) selb[k_r + i] = -1;
  __syncthreads();
  // exclusive prefix of the R clusters' sizes (execution-buffer rows)
  int32_t* rp = rpre + (size_t)bh * (k_r + 1);
  const int32_t* cnt = counts + (size_t)bh * C;
  int run = 0;
  for (int base = 0; base < kr; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const int v = i < kr ? cnt[selb[i]] : 0;
    // block inclusive scan of v
    const unsigned lane = lane_id(), warp = threadIdx.x >> 5;
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      int t = __shfl_up_sync(0xffffffffu, incl, off);
      if ((int)lane >= off) incl += t;
    }
    if (lane == 31) sm[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int w = sm[lane];
      int wi = w;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, wi, off);
        if ((int)lane >= off) wi += t;
      }
      sm[lane] = wi - w;
      if (lane == 31) sm[64] = wi;
    }
    __syncthreads();
    const int excl = run + sm[warp] + incl - v;
    if (i < kr) rp[i] = excl;
    run += sm[64];
    __syncthreads();
  }
  if (threadIdx.x == 0) rp[kr] = run;
  for (int i = kr + 1 + threadIdx.x; i <= k_r; i += blockDim.x) rp[i] = run;
  if (sel_user || rpre_user) {
    __syncthreads();
    if (sel_user)
      for (int i = threadIdx.x; i < k_r + k_e; i += blockDim.x)
        sel_user[(size_t)bh * (k_r + k_e) + i] = selb[i];
    if (rpre_user)
      for (int i = threadIdx.x; i <= k_r; i += blockDim.x)
        rpre_user[(size_t)bh * (k_r + 1) + i] = rp[i];
  }
  (void)offsets;
}

// ------------------------------------------------------------------- S4+S5
struct OnlineState {
  float m, l;
  float o[8];
};

template <int G>
__device__ __forceinline__ void online_token(OnlineState (&st)[G], const float (&qv)[G][8],
                                             const uint4& kraw, const uint4& vraw,
                                             bool live) {
  float k[8], v[8];
  bf16x8_to_float(kraw, k);
  bf16x8_to_float(vraw, v);
  float x[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaf(qv[g][i], k[i], a);
    x[g] = a;
  }
#pragma unroll
  for (int off = 8; off >= 1; off >>= 1)
#pragma unroll
    for (int g = 0; g < G; ++g) x[g] += __shfl_xor_sync(0xffffffffu, x[g], off);
  if (!live) return;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float s = x[g] * kScale;
    const float mn = fmaxf(st[g].m, s);
    const float corr = __expf(st[g].m - mn);
    const float p = __expf(s - mn);
    st[g].l = st[g].l * corr + p;
#pragma unroll
    for (int i = 0; i < 8; ++i) st[g].o[i] = fmaf(st[g].o[i], corr, p * v[i]);
    st[g].m = mn;
  }
}

template <int G>
__global__ void __launch_bounds__(256) attend_kernel(
    const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ Ks,
    const __nv_bfloat16* __restrict__ Vs, const __nv_bfloat16* __restrict__ Kr,
    const __nv_bfloat16* __restrict__ Vr, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ counts, const float* __restrict__ vsum,
    const float* __restrict__ score, const int32_t* __restrict__ sel,
    const int32_t* __restrict__ rpre, float* __restrict__ part, int n_steady, int M, int C,
    int k_r, int k_e, int kr, int ke, int P, int exec_rows /* 0: in place */, int* status) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  // [16 hw][G][132] states, then rpre [kr+1], rbase [kr]
  float* st_sm = reinterpret_cast<float*>(smem_raw);
  int32_t* rp_sm = reinterpret_cast<int32_t*>(st_sm + 16 * G * kPartStride);
  int32_t* rb_sm = rp_sm + (kr + 1);

  const int bh = blockIdx.y;
  const int j = blockIdx.x;
  const int l16 = threadIdx.x & 15;
  const int hw = threadIdx.x >> 4;
  const int32_t* selb = sel + (size_t)bh * (k_r + k_e);
  const int32_t* rpb = rpre + (size_t)bh * (k_r + 1);
  const bool smem_tab = kr <= kMaxRetrievalInSmem;
  if (smem_tab) {
    for (int i = threadIdx.x; i <= kr; i += blockDim.x) rp_sm[i] = rpb[i];
    if (exec_rows == 0)
      for (int i = threadIdx.x; i < kr; i += blockDim.x)
        rb_sm[i] = offsets[(size_t)bh * (C + 1) + selb[i]];
  }
  float qv[G][8];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    uint4 raw = ldg_nc_v4(q + ((size_t)bh * G + g) * kHeadDim + l16 * 8);
    bf16x8_to_float(raw, qv[g]);
  }
  OnlineState st[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    st[g].m = -INFINITY;
    st[g].l = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) st[g].o[i] = 0.f;
  }
  __syncthreads();
  const int32_t* rp = smem_tab ? rp_sm : rpb;
  const long long T_R = rp[kr];
  const long long T = n_steady + T_R;
  const long long t0 = T * j / P, t1 = T * (j + 1) / P;
  const size_t steady_base = (size_t)bh * n_steady * kHeadDim;
  const size_t rbase_rows = exec_rows ? (size_t)bh * exec_rows : (size_t)bh * M;

  // Warp-uniform trip count (shuffles inside online_token are warp-wide);
  // a half-warp past the end runs on zeros and discards the result.
  for (long long t = t0 + hw; t - (hw & 1) < t1; t += 16) {
    bool live = t < t1;
    const __nv_bfloat16 *kp = Ks, *vp = Vs;
    if (!live) {
    } else if (t < n_steady) {
      kp = Ks + steady_base + (size_t)t * kHeadDim;
      vp = Vs + steady_base + (size_t)t * kHeadDim;
    } else {
      const int tt = (int)(t - n_steady);
      long long row;
      if (exec_rows) {
        row = tt;
      } else {
        // cluster i with rp[i] <= tt < rp[i+1]
        int lo = 0, hi = kr - 1;
        while (lo < hi) {
          const int mid = (lo + hi + 1) >> 1;
          if (rp[mid] <= tt) lo = mid; else hi = mid - 1;
        }
        const int rb = smem_tab ? rb_sm[lo] : offsets[(size_t)bh * (C + 1) + selb[lo]];
        row = (long long)rb + (tt - rp[lo]);
      }
      // rows outside the source buffer (an inconsistent index, or an
      // execution buffer smaller than the selection) are skipped and flagged
      if (row < 0 || row >= (exec_rows ? exec_rows : M)) {
        if (l16 == 0) record_status(status, RI_ERR_INVALID_ARG);
        live = false;
      } else {
        kp = Kr + (rbase_rows + (size_t)row) * kHeadDim;
        vp = Vr + (rbase_rows + (size_t)row) * kHeadDim;
      }
    }
    const uint4 kraw = live ? ldg_nc_v4(kp + l16 * 8) : make_uint4(0, 0, 0, 0);
    const uint4 vraw = live ? ldg_nc_v4(vp + l16 * 8) : make_uint4(0, 0, 0, 0);
    online_token<G>(st, qv, kraw, vraw, live);
  }

  // estimation clusters [e0, e1) of E
  const int e0 = (int)((long long)ke * j / P), e1 = (int)((long long)ke * (j + 1) / P);
  for (int e = e0 + hw; e < e1; e += 16) {
    const int c = selb[k_r + e];
    const int n = counts[(size_t)bh * C + c];
    if (n <= 0) continue;
    const float* vs = vsum + ((size_t)bh * C + c) * kHeadDim + l16 * 8;
    const float4 v0 = *reinterpret_cast<const float4*>(vs);
    const float4 v1 = *reinterpret_cast<const float4*>(vs + 4);
    const float vv[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    const float nf = (float)n;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float s = score[((size_t)bh * G + g) * C + c];
      const float mn = fmaxf(st[g].m, s);
      const float corr = __expf(st[g].m - mn);
      const float p = __expf(s - mn);
      st[g].l = st[g].l * corr + nf * p;
#pragma unroll
      for (int i = 0; i < 8; ++i) st[g].o[i] = fmaf(st[g].o[i], corr, p * vv[i]);
      st[g].m = mn;
    }
  }

  // merge the 16 half-warp states of this block
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float* row = st_sm + ((size_t)hw * G + g) * kPartStride;
    if (l16 == 0) {
      row[0] = st[g].m;
      row[1] = st[g].l;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) row[4 + l16 * 8 + i] = st[g].o[i];
  }
  __syncthreads();
  float* pout = part + ((size_t)bh * P + j) * G * kPartStride;
  for (int idx = threadIdx.x; idx < G * kHeadDim; idx += blockDim.x) {
    const int g = idx / kHeadDim, dd = idx % kHeadDim;
    float mx = -INFINITY;
    for (int w = 0; w < 16; ++w) mx = fmaxf(mx, st_sm[((size_t)w * G + g) * kPartStride]);
    float l = 0.f, o = 0.f;
    if (mx != -INFINITY) {
      for (int w = 0; w < 16; ++w) {
        const float* row = st_sm + ((size_t)w * G + g) * kPartStride;
        const float f = __expf(row[0] - mx);
        l += row[1] * f;
        o += row[4 + dd] * f;
      }
    }
    pout[(size_t)g * kPartStride + 4 + dd] = o;
    if (dd == 0) {
      pout[(size_t)g * kPartStride + 0] = mx;
      pout[(size_t)g * kPartStride + 1] = l;
    }
  }
}

// ------------------------------------------------------------------- S6
__global__ void __launch_bounds__(128) merge_kernel(const float* __restrict__ part,
                                                    __nv_bfloat16* __restrict__ out,
                                                    float* __restrict__ lse, int G, int P) {
  const int hq = blockIdx.x;  // (b*H + h)*G + g
  const int bh = hq / G, g = hq % G;
  const int dd = threadIdx.x;
  float mx = -INFINITY;
  for (int p = 0; p < P; ++p)
    mx = fmaxf(mx, part[(((size_t)bh * P + p) * G + g) * kPartStride]);
  float l = 0.f, o = 0.f;
  if (mx != -INFINITY) {
    for (int p = 0; p < P; ++p) {
      const float* row = part + (((size_t)bh * P + p) * G + g) * kPartStride;
      const float f = __expf(row[0] - mx);
      l += row[1] * f;
      o += row[4 + dd] * f;
    }
  }
  // no token and no cluster contributed (empty steady zone and budgets): 0, lse -inf
  const bool any = l > 0.f;
  out[(size_t)hq * kHeadDim + dd] = __float2bfloat16_rn(any ? o / l : 0.f);
  if (lse && dd == 0) lse[hq] = any ? mx + logf(l) : -INFINITY;
}

template <int G>
cudaError_t launch_attend_g(const Geometry& g, const DecodeLayout& L, const DecodeArgs& a,
                            cudaStream_t s) {
  char* ws = a.ws;
  const float* score = reinterpret_cast<const float*>(ws + L.off_score);
  const int32_t* sel = reinterpret_cast<const int32_t*>(ws + L.off_sel);
  const int32_t* rpre = reinterpret_cast<const int32_t*>(ws + L.off_rpre);
  float* part = reinterpret_cast<float*>(ws + L.off_part);
  const bool exec = a.exec_K != nullptr;
  size_t smem = (size_t)16 * G * kPartStride * sizeof(float);
  if (L.kr <= kMaxRetrievalInSmem) smem += (size_t)(2 * L.kr + 1) * sizeof(int32_t);
  auto kern = attend_kernel<G>;
  constexpr int kMaxSmem = 16 * G * kPartStride * 4 + (2 * kMaxRetrievalInSmem + 1) * 4;
  cudaError_t e = set_smem_once(reinterpret_cast<const void*>(kern), kMaxSmem);
  if (e != cudaSuccess) return e;
  dim3 grid(L.P, (unsigned)g.BH());
  kern<<<grid, 256, smem, s>>>(
      reinterpret_cast<const __nv_bfloat16*>(a.q), reinterpret_cast<const __nv_bfloat16*>(a.Ks),
      reinterpret_cast<const __nv_bfloat16*>(a.Vs),
      reinterpret_cast<const __nv_bfloat16*>(exec ? a.exec_K : a.Kp),
      reinterpret_cast<const __nv_bfloat16*>(exec ? a.exec_V : a.Vp), a.offsets, a.counts,
      a.vsum, score, sel, rpre, part, g.n_steady, g.M, g.C, L.k_r, L.k_e, L.kr, L.ke, L.P,
      exec ? a.exec_rows : 0, reinterpret_cast<int*>(ws));
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  merge_kernel<<<(unsigned)(g.BH() * G), 128, 0, s>>>(
      part, reinterpret_cast<__nv_bfloat16*>(a.out), a.lse, G, L.P);
  return cudaGetLastError();
}

template <int G>
cudaError_t launch_score_g(const Geometry& g, const DecodeLayout& L, const DecodeArgs& a,
                           cudaStream_t s) {
  float* rkey = reinterpret_cast<float*>(a.ws + L.off_rkey);
  float* score = reinterpret_cast<float*>(a.ws + L.off_score);
  dim3 grid((g.C + kScoreCentroidsPerBlock - 1) / kScoreCentroidsPerBlock, (unsigned)g.BH());
  score_kernel<G><<<grid, 256, 0, s>>>(reinterpret_cast<const __nv_bfloat16*>(a.q),
                                       reinterpret_cast<const __nv_bfloat16*>(a.centroid),
                                       a.counts, score, rkey, g.C);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_select(const Geometry& g, const DecodeLayout& L, const DecodeArgs& a,
                          cudaStream_t s) {
  if (g.C == 0) {
    // no index: selection is empty
    int32_t* sel = reinterpret_cast<int32_t*>(a.ws + L.off_sel);
    int32_t* rpre = reinterpret_cast<int32_t*>(a.ws + L.off_rpre);
    cudaError_t e;
    if (L.k_r + L.k_e > 0) {
      e = cudaMemsetAsync(sel, 0xFF, g.BH() * (L.k_r + L.k_e) * sizeof(int32_t), s);
      if (e != cudaSuccess) return e;
      if (a.sel_user) {
        e = cudaMemsetAsync(a.sel_user, 0xFF, g.BH() * (L.k_r + L.k_e) * sizeof(int32_t), s);
        if (e != cudaSuccess) return e;
      }
    }
    e = cudaMemsetAsync(rpre, 0, g.BH() * (L.k_r + 1) * sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
    if (a.rpre_user) e = cudaMemsetAsync(a.rpre_user, 0, g.BH() * (L.k_r + 1) * sizeof(int32_t), s);
    return e;
  }
  cudaError_t e;
  switch (g.G) {
    case 1: e = launch_score_g<1>(g, L, a, s); break;
    case 2: e = launch_score_g<2>(g, L, a, s); break;
    case 3: e = launch_score_g<3>(g, L, a, s); break;
    case 4: e = launch_score_g<4>(g, L, a, s); break;
    case 5: e = launch_score_g<5>(g, L, a, s); break;
    case 6: e = launch_score_g<6>(g, L, a, s); break;
    case 7: e = launch_score_g<7>(g, L, a, s); break;
    default: e = launch_score_g<8>(g, L, a, s); break;
  }
  if (e != cudaSuccess) return e;
  select_kernel<<<(unsigned)g.BH(), 1024, 0, s>>>(
      reinterpret_cast<const float*>(a.ws + L.off_rkey), a.counts, a.offsets,
      reinterpret_cast<int32_t*>(a.ws + L.off_sel), reinterpret_cast<int32_t*>(a.ws + L.off_rpre),
      a.sel_user, a.rpre_user, g.C, L.k_r, L.k_e, L.kr, L.ke);
  return cudaGetLastError();
}

cudaError_t launch_attend(const Geometry& g, const DecodeLayout& L, const DecodeArgs& a,
                          cudaStream_t s) {
  switch (g.G) {
    case 1: return launch_attend_g<1>(g, L, a, s);
    case 2: return launch_attend_g<2>(g, L, a, s);
    case 3: return launch_attend_g<3>(g, L, a, s);
    case 4: return launch_attend_g<4>(g, L, a, s);
    case 5: return launch_attend_g<5>(g, L, a, s);
    case 6: return launch_attend_g<6>(g, L, a, s);
    case 7: return launch_attend_g<7>(g, L, a, s);
    default: return launch_attend_g<8>(g, L, a, s);
  }
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
