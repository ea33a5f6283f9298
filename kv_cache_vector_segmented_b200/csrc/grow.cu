// Index maintenance during decode (sm_100a): the wave index of every
// (sequence, KV head) kept up to date while the sequence grows by one token
// per step.
//
// "KV缓存技术与RetroInfer系统在长上下文推理中的优化实践" (framerc.cn) §2.1 item 1
// (the steady zone holds the first 4 and the most recent 64 tokens, so one
// token leaves the recent window per decode step) and the §2.1 pseudocode
// (k-means per 8K-token segment).  The pages give no mechanism; the reading:
// the token that leaves the window joins the *open segment*, in the open
// cluster of its nearest centroid (squared Euclidean distance to the stored
// bf16 centroids, lower id on ties) among the last closed segment's
// clusters that still have a free slot; each open cluster has
// ceil(2 seg_len / K_last) slots and is scored with that centroid; when the
// open segment holds seg_len tokens, k-means over them (position order,
// seeds floor(j L / K)) turns it into a closed segment and a new, empty open
// segment follows.
//
// Layout of a growing index, per unit: closed segments cluster-contiguous
// from row 0 (the prefill's, then the appended ones), the open clusters'
// slots from row R0 (open cluster j at R0 + j cap, its members in arrival
// order), cluster ids closed first, then the K open ones; the recent window
// is a ring in Ks/Vs (slot s0 + ((p - base_len) mod s1) holds position p).
#include "common.cuh"
#include "internal.h"

namespace ri {

namespace {

constexpr int kGrowThreads = 256;

struct OpenParams {
  int Cs, Ms, open_id, K_full, tgt_id, K_tgt, cap, R0;
};

// Records of the open segment: open cluster j takes the centroid of target
// j (zero past K_tgt), no members, its slots at R0 + j cap; every id after
// the open ones is empty; offsets[Cs] = Ms.
__global__ void __launch_bounds__(kGrowThreads)
    open_init_kernel(ri_index idx, OpenParams o) {
  const int u = blockIdx.x, tid = threadIdx.x;
  __nv_bfloat16* cent = static_cast<__nv_bfloat16*>(idx.centroid) + (size_t)u * o.Cs * kHeadDim;
  float* vsum = idx.vsum + (size_t)u * o.Cs * kHeadDim;
  for (int e = tid; e < o.K_full * kHeadDim; e += kGrowThreads) {
    const int j = e / kHeadDim, c = e % kHeadDim;
    const __nv_bfloat16 z = __float2bfloat16_rn(0.f);
    cent[(size_t)(o.open_id + j) * kHeadDim + c] =
        j < o.K_tgt ? cent[(size_t)(o.tgt_id + j) * kHeadDim + c] : z;
    vsum[(size_t)(o.open_id + j) * kHeadDim + c] = 0.f;
  }
  int32_t* counts = idx.counts + (size_t)u * o.Cs;
  int32_t* offsets = idx.offsets + (size_t)u * (o.Cs + 1);
  for (int j = tid; j < o.Cs - o.open_id; j += kGrowThreads) {
    counts[o.open_id + j] = 0;
    offsets[o.open_id + j] = j < o.K_tgt ? o.R0 + j * o.cap : o.R0;
  }
  if (tid == 0) offsets[o.Cs] = o.Ms;
}

struct AppendParams {
  int Cs, Ms, open_id, tgt_id, K_tgt, cap;
  int slot;      // ring slot of the leaving token (and of the new one)
  int pos;       // position of the leaving token
  int n_steady;  // rows of Ks / Vs per unit
};

// One block per unit: the leaving token's open cluster (nearest target with
// a free slot), its row, size and value sum; then the new token in its ring
// slot.  `assigned` (optional) gets the open cluster chosen per unit.
__global__ void __launch_bounds__(kGrowThreads)
    append_kernel(ri_index idx, AppendParams a, const __nv_bfloat16* __restrict__ k_new,
                  const __nv_bfloat16* __restrict__ v_new, int32_t* assigned, int* status) {
  __shared__ float key[kHeadDim];
  __shared__ float bd[kGrowThreads / 32];
  __shared__ int bj[kGrowThreads / 32];
  __shared__ int choice;
  const int u = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  __nv_bfloat16* Ks = static_cast<__nv_bfloat16*>(idx.Ks) + (size_t)u * a.n_steady * kHeadDim;
  __nv_bfloat16* Vs = static_cast<__nv_bfloat16*>(idx.Vs) + (size_t)u * a.n_steady * kHeadDim;
  const __nv_bfloat16* kl = Ks + (size_t)a.slot * kHeadDim;
  const __nv_bfloat16* vl = Vs + (size_t)a.slot * kHeadDim;
  if (tid < kHeadDim) key[tid] = __bfloat162float(kl[tid]);
  __syncthreads();
  // squared distances in the direct difference form, lane = 4 dims
  const __nv_bfloat16* cent =
      static_cast<const __nv_bfloat16*>(idx.centroid) + (size_t)u * a.Cs * kHeadDim;
  const int32_t* counts = idx.counts + (size_t)u * a.Cs;
  float best = INFINITY;
  int bestj = 0x7fffffff;
  for (int j = warp; j < a.K_tgt; j += kGrowThreads / 32) {
    const __nv_bfloat16* c = cent + (size_t)(a.tgt_id + j) * kHeadDim + lane * 4;
    const uint2 raw = *reinterpret_cast<const uint2*>(c);
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
    const float2 c01 = __bfloat1622float2(h[0]), c23 = __bfloat1622float2(h[1]);
    const float d0 = key[lane * 4] - c01.x, d1 = key[lane * 4 + 1] - c01.y;
    const float d2 = key[lane * 4 + 2] - c23.x, d3 = key[lane * 4 + 3] - c23.y;
    float dist = d0 * d0 + d1 * d1 + d2 * d2 + d3 * d3;
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) dist += __shfl_xor_sync(0xffffffffu, dist, off);
    const bool room = counts[a.open_id + j] < a.cap;
    if (room && (dist < best || (dist == best && j < bestj))) {
      best = dist;
      bestj = j;
    }
  }
  if (lane == 0) {
    bd[warp] = best;
    bj[warp] = bestj;
  }
  __syncthreads();
  if (tid == 0) {
    float b = INFINITY;
    int jj = 0x7fffffff;
    for (int w = 0; w < kGrowThreads / 32; ++w)
      if (bj[w] != 0x7fffffff && (bd[w] < b || (bd[w] == b && bj[w] < jj))) {
        b = bd[w];
        jj = bj[w];
      }
    choice = jj;
    if (jj == 0x7fffffff) record_status(status, RI_ERR_CAPACITY);  // no slot anywhere
    if (assigned) assigned[u] = jj == 0x7fffffff ? -1 : jj;
  }
  __syncthreads();
  const int j = choice;
  if (j != 0x7fffffff) {
    const int id = a.open_id + j;
    const int row = idx.offsets[(size_t)u * (a.Cs + 1) + id] + counts[id];
    if (row < 0 || row >= a.Ms) {
      if (tid == 0) record_status(status, RI_ERR_INVALID_ARG);
    } else {
      __nv_bfloat16* Kp = static_cast<__nv_bfloat16*>(idx.Kp) + ((size_t)u * a.Ms + row) * kHeadDim;
      __nv_bfloat16* Vp = static_cast<__nv_bfloat16*>(idx.Vp) + ((size_t)u * a.Ms + row) * kHeadDim;
      if (tid < kHeadDim) {
        Kp[tid] = kl[tid];
        const __nv_bfloat16 v = vl[tid];
        Vp[tid] = v;
        float* vs = idx.vsum + ((size_t)u * a.Cs + id) * kHeadDim;
        vs[tid] += __bfloat162float(v);
      }
      if (tid == 0) {
        idx.perm[(size_t)u * a.Ms + row] = a.pos;
        idx.counts[(size_t)u * a.Cs + id] = counts[id] + 1;
      }
    }
  }
  __syncthreads();  // the leaving token is read before its slot is reused
  if (tid < kHeadDim) {
    Ks[(size_t)a.slot * kHeadDim + tid] = k_new[(size_t)u * kHeadDim + tid];
    Vs[(size_t)a.slot * kHeadDim + tid] = v_new[(size_t)u * kHeadDim + tid];
  }
}

// The open segment's tokens in position order: one warp per open cluster,
// lanes 0-15 move 16-byte chunks of the K row, 16-31 of the V row.
__global__ void __launch_bounds__(kGrowThreads)
    close_gather_kernel(ri_index idx, int Cs, int Ms, int open_id, int K_tgt, int first_pos,
                        int seg_len, __nv_bfloat16* sK, __nv_bfloat16* sV, int* status) {
  const int u = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.y * (kGrowThreads / 32) + warp;
  if (j >= K_tgt) return;
  const int id = open_id + j;
  const int n = idx.counts[(size_t)u * Cs + id];
  const int r0 = idx.offsets[(size_t)u * (Cs + 1) + id];
  const bool v_half = lane >= 16;
  const int chunk = lane & 15;
  const uint4* src = reinterpret_cast<const uint4*>(v_half ? idx.Vp : idx.Kp);
  uint4* dst = reinterpret_cast<uint4*>(v_half ? sV : sK);
  for (int i = 0; i < n; ++i) {
    const int row = r0 + i;
    const int p = row >= 0 && row < Ms ? idx.perm[(size_t)u * Ms + row] - first_pos : -1;
    if (p < 0 || p >= seg_len) {
      if (lane == 0) record_status(status, RI_ERR_INVALID_ARG);
      continue;
    }
    dst[((size_t)u * seg_len + p) * (kHeadDim / 8) + chunk] =
        src[((size_t)u * Ms + row) * (kHeadDim / 8) + chunk];
  }
}

// The closed segment built from the open tokens into its place: rows from
// `closed_rows`, ids from `first_id` (the former open ids), positions from
// first_pos.
__global__ void __launch_bounds__(kGrowThreads)
    close_scatter_kernel(ri_index idx, ri_index seg, int Cs, int Ms, int first_id, int K,
                         int closed_rows, int first_pos, int seg_len) {
  const int u = blockIdx.x;
  const int t0 = blockIdx.y * kGrowThreads + threadIdx.x, stride = gridDim.y * kGrowThreads;
  const uint4* sK = reinterpret_cast<const uint4*>(seg.Kp) + (size_t)u * seg_len * (kHeadDim / 8);
  const uint4* sV = reinterpret_cast<const uint4*>(seg.Vp) + (size_t)u * seg_len * (kHeadDim / 8);
  uint4* dK = reinterpret_cast<uint4*>(idx.Kp) + ((size_t)u * Ms + closed_rows) * (kHeadDim / 8);
  uint4* dV = reinterpret_cast<uint4*>(idx.Vp) + ((size_t)u * Ms + closed_rows) * (kHeadDim / 8);
  for (int e = t0; e < seg_len * (kHeadDim / 8); e += stride) {
    dK[e] = sK[e];
    dV[e] = sV[e];
  }
  for (int i = t0; i < seg_len; i += stride)
    idx.perm[(size_t)u * Ms + closed_rows + i] = seg.perm[(size_t)u * seg_len + i] + first_pos;
  const __nv_bfloat16* sc = static_cast<const __nv_bfloat16*>(seg.centroid) + (size_t)u * K * kHeadDim;
  __nv_bfloat16* dc = static_cast<__nv_bfloat16*>(idx.centroid) + ((size_t)u * Cs + first_id) * kHeadDim;
  const float* sv = seg.vsum + (size_t)u * K * kHeadDim;
  float* dv = idx.vsum + ((size_t)u * Cs + first_id) * kHeadDim;
  for (int e = t0; e < K * kHeadDim; e += stride) {
    dc[e] = sc[e];
    dv[e] = sv[e];
  }
  for (int j = t0; j < K; j += stride) {
    idx.counts[(size_t)u * Cs + first_id + j] = seg.counts[(size_t)u * K + j];
    idx.offsets[(size_t)u * (Cs + 1) + first_id + j] =
        seg.offsets[(size_t)u * (K + 1) + j] + closed_rows;
  }
}

OpenParams open_params(const Geometry& g) {
  OpenParams o;
  o.Cs = g.Cs;
  o.Ms = g.Ms;
  o.open_id = g.open_id;
  o.K_full = g.K_full;
  o.tgt_id = g.tgt_id;
  o.K_tgt = g.K_tgt;
  o.cap = g.cap;
  o.R0 = g.R0;
  return o;
}

}  // namespace

cudaError_t launch_open_init(const Geometry& g, const ri_index& idx, cudaStream_t s) {
  open_init_kernel<<<(unsigned)g.BH(), kGrowThreads, 0, s>>>(idx, open_params(g));
  return cudaGetLastError();
}

cudaError_t launch_append(const Geometry& g, const ri_index& idx, const void* k_new,
                          const void* v_new, int32_t* assigned, int* status, cudaStream_t s) {
  AppendParams a;
  a.Cs = g.Cs;
  a.Ms = g.Ms;
  a.open_id = g.open_id;
  a.tgt_id = g.tgt_id;
  a.K_tgt = g.K_tgt;
  a.cap = g.cap;
  a.slot = g.s0 + (g.N - g.base_len) % g.s1;
  a.pos = g.N - g.s1;
  a.n_steady = g.n_steady;
  append_kernel<<<(unsigned)g.BH(), kGrowThreads, 0, s>>>(
      idx, a, static_cast<const __nv_bfloat16*>(k_new), static_cast<const __nv_bfloat16*>(v_new),
      assigned, status);
  return cudaGetLastError();
}

cudaError_t launch_close_gather(const Geometry& g, const ri_index& idx, void* sK, void* sV,
                                int* status, cudaStream_t s) {
  const int first_pos = g.base_len - g.s1 + g.F * g.seg_len;
  dim3 grid((unsigned)g.BH(), (unsigned)((g.K_tgt + kGrowThreads / 32 - 1) / (kGrowThreads / 32)));
  close_gather_kernel<<<grid, kGrowThreads, 0, s>>>(idx, g.Cs, g.Ms, g.open_id, g.K_tgt,
                                                   first_pos, g.seg_len,
                                                   static_cast<__nv_bfloat16*>(sK),
                                                   static_cast<__nv_bfloat16*>(sV), status);
  return cudaGetLastError();
}

cudaError_t launch_close_scatter(const Geometry& g, const ri_index& idx, const ri_index& seg,
                                 cudaStream_t s) {
  const int first_pos = g.base_len - g.s1 + g.F * g.seg_len;
  dim3 grid((unsigned)g.BH(), 16);
  close_scatter_kernel<<<grid, kGrowThreads, 0, s>>>(idx, seg, g.Cs, g.Ms, g.open_id, g.K_full,
                                                     g.closed_rows, first_pos, g.seg_len);
  return cudaGetLastError();
}

}  // namespace ri
