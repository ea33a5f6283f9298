// Fixed device scratch for ri_decode_attention_static: a file-scope
// __device__ array, so that entry point needs no caller workspace and
// allocates nothing.  Its address is looked up once per device (with that
// device current) and cached; the lookup is the call's only setup cost.
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"

namespace ri {

namespace {

static __device__ __align__(256) unsigned char g_decode_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

}  // namespace

cudaError_t static_decode_scratch(void** addr) {
  *addr = nullptr;
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = p;
  }
  *addr = g_addr[dev];
  return cudaSuccess;
}

}  // namespace ri
