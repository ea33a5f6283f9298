// Execution-buffer gather of the wave buffer (RetroInfer,
// "KV缓存技术与RetroInfer系统在长上下文推理中的优化实践" (framerc.cn) §3.2
// execution buffer assembly): copies of K and V rows between the host copy
// of the index (pinned memory, read through unified addressing), the GPU
// block cache pool and the execution buffer.  One warp per copy descriptor
// (at most 16 rows): lane l moves 16-byte chunk l & 15 of the K (l < 16) or
// V (l >= 16) row, all of a descriptor's loads issued before its stores so
// the host-link reads overlap.
#include "common.cuh"
#include "internal.h"

namespace ri {

namespace {

constexpr int kMaxGatherThreads = 512;
constexpr int kMaxRows = 16;  // rows per descriptor (the plan's chunk size)

__global__ void __launch_bounds__(kMaxGatherThreads)
    gather_kernel(GatherArgs a, const ri_copy_desc* __restrict__ desc, int n_desc, int* status) {
  const int lane = threadIdx.x & 31;
  const int wpb = blockDim.x >> 5;  // warps per block (the launch shape)
  const int warps = gridDim.x * wpb;
  for (int w = blockIdx.x * wpb + (threadIdx.x >> 5); w < n_desc; w += warps) {
    const ri_copy_desc d = desc[w];
    const bool v_half = lane >= 16;
    const int chunk = lane & 15;
    const __nv_bfloat16* src_base = nullptr;
    long long src_lim = 0;
    switch (d.src_kind) {
      case RI_SRC_HOST:
        src_base = static_cast<const __nv_bfloat16*>(v_half ? a.host_V : a.host_K);
        src_lim = a.M;
        break;
      case RI_SRC_CACHE:
        src_base = static_cast<const __nv_bfloat16*>(v_half ? a.cache_V : a.cache_K);
        src_lim = a.pool_rows;
        break;
      case RI_SRC_EXEC:
        src_base = static_cast<const __nv_bfloat16*>(v_half ? a.exec_V : a.exec_K);
        src_lim = a.exec_rows;
        break;
      default:
        break;
    }
    __nv_bfloat16* dst_base = nullptr;
    long long dst_lim = 0;
    if (d.dst_kind == RI_DST_EXEC) {
      dst_base = static_cast<__nv_bfloat16*>(v_half ? a.exec_V : a.exec_K);
      dst_lim = a.exec_rows;
    } else if (d.dst_kind == RI_DST_CACHE) {
      dst_base = static_cast<__nv_bfloat16*>(v_half ? a.cache_V : a.cache_K);
      dst_lim = a.pool_rows;
    }
    const bool ok = src_base && dst_base && d.unit >= 0 && d.unit < a.units && d.n_rows >= 0 &&
                    d.n_rows <= kMaxRows && d.src_row >= 0 &&
                    (long long)d.src_row + d.n_rows <= src_lim && d.dst_row >= 0 &&
                    (long long)d.dst_row + d.n_rows <= dst_lim;
    if (!ok) {
      if (lane == 0) record_status(status, RI_ERR_INVALID_ARG);
      continue;
    }
    const uint4* src = reinterpret_cast<const uint4*>(
        src_base + ((size_t)d.unit * src_lim + d.src_row) * kHeadDim) + chunk;
    uint4* dst = reinterpret_cast<uint4*>(dst_base + ((size_t)d.unit * dst_lim + d.dst_row) *
                                                         kHeadDim) + chunk;
    uint4 v[kMaxRows];
#pragma unroll
    for (int r = 0; r < kMaxRows; ++r)
      if (r < d.n_rows) v[r] = ldg_nc_v4(src + r * (kHeadDim / 8));
#pragma unroll
    for (int r = 0; r < kMaxRows; ++r)
      if (r < d.n_rows) dst[r * (kHeadDim / 8)] = v[r];
  }
}

}  // namespace

cudaError_t launch_gather(const GatherArgs& a, const ri_copy_desc* desc, int n_desc, int* status,
                          cudaStream_t s, int threads, int blocks_per_sm) {
  if (n_desc <= 0) return cudaSuccess;
  if (threads <= 0) threads = kGatherDefaultThreads;
  if (blocks_per_sm <= 0) blocks_per_sm = kGatherDefaultBlocksPerSM;
  const int per_block = threads / 32;
  int blocks = (n_desc + per_block - 1) / per_block;
  const int cap = blocks_per_sm * num_sms();
  if (blocks > cap) blocks = cap;
  gather_kernel<<<blocks, threads, 0, s>>>(a, desc, n_desc, status);
  return cudaGetLastError();
}

}  // namespace ri
