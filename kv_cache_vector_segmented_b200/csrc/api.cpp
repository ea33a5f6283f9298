// C ABI of the wave-index path: argument validation, derived geometry,
// workspace layouts and the launch sequence of each call.  Every check runs
// on the host before the first launch; nothing here allocates device memory.
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <cmath>
#include <mutex>

#include "internal.h"
#include "retroinfer.h"

namespace ri {

namespace {
thread_local char g_last_error[512] = "";
}

void set_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_last_error, sizeof(g_last_error), fmt, ap);
  va_end(ap);
}

int num_sms() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0)
      n = v;
  }
  return n;
}

namespace {
constexpr int kMaxDevicesHost = 64;
std::mutex g_smem_mu;
bool g_smem_done[kMaxDevicesHost][kSmemSlots];
}  // namespace

cudaError_t set_smem_once(int slot, const void* func, int bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevicesHost || slot < 0 || slot >= kSmemSlots)
    return cudaErrorInvalidValue;
  std::lock_guard<std::mutex> lk(g_smem_mu);
  if (g_smem_done[dev][slot]) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) g_smem_done[dev][slot] = true;
  return e;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool make_geometry(const ri_index_config* cfg, Geometry* g) {
  if (!cfg) {
    set_error("config is NULL");
    return false;
  }
  const ri_index_config& c = *cfg;
  if (c.batch < 1 || c.num_kv_heads < 1 || c.seq_len < 1) {
    set_error("batch, num_kv_heads and seq_len must be >= 1 (got %d, %d, %d)", c.batch,
              c.num_kv_heads, c.seq_len);
    return false;
  }
  if (c.group_size < 1 || c.group_size > kMaxGroupHost) {
    set_error("group_size must be in [1, %d] (got %d)", kMaxGroupHost, c.group_size);
    return false;
  }
  if (c.head_dim != 128) {
    set_error("head_dim must be 128 (got %d)", c.head_dim);
    return false;
  }
  if (c.seg_len < 1 || c.seg_len > kMaxSegLen) {
    set_error("seg_len must be in [1, %d] (got %d)", kMaxSegLen, c.seg_len);
    return false;
  }
  if (c.clusters_per_seg < 1 || c.clusters_per_seg > 512) {
    set_error("clusters_per_seg must be in [1, 512] (got %d)", c.clusters_per_seg);
    return false;
  }
  if (c.iters < 0 || c.iters > 1000) {
    set_error("iters must be in [0, 1000] (got %d)", c.iters);
    return false;
  }
  if (c.steady_initial < 0 || c.steady_recent < 0) {
    set_error("steady_initial and steady_recent must be >= 0");
    return false;
  }
  const long long bhn = (long long)c.batch * c.num_kv_heads * c.seq_len;
  if (bhn > (1ll << 31) - 1) {
    set_error("batch * num_kv_heads * seq_len must be < 2^31 (got %lld)", bhn);
    return false;
  }
  g->B = c.batch;
  g->H = c.num_kv_heads;
  g->G = c.group_size;
  g->d = c.head_dim;
  g->N = c.seq_len;
  g->seg_len = c.seg_len;
  g->K = c.clusters_per_seg;
  g->iters = c.iters;
  g->s0 = c.steady_initial;
  g->s1 = c.steady_recent;
  const long long steady = (long long)c.steady_initial + c.steady_recent;
  g->M = (int)(c.seq_len > steady ? c.seq_len - steady : 0);
  g->n_steady = (int)(c.seq_len < steady ? c.seq_len : steady);
  g->m0 = g->M > 0 ? c.steady_initial : 0;
  g->S = (g->M + c.seg_len - 1) / c.seg_len;
  g->K_full = c.clusters_per_seg < c.seg_len ? c.clusters_per_seg : c.seg_len;
  if (g->S > 0) {
    g->L_last = g->M - (g->S - 1) * c.seg_len;
    g->K_last = c.clusters_per_seg < g->L_last ? c.clusters_per_seg : g->L_last;
    g->C = (g->S - 1) * g->K_full + g->K_last;
    g->tiles_full = (c.seg_len + 127) / 128;
    g->tiles_last = (g->L_last + 127) / 128;
    g->tiles_bh = (g->S - 1) * g->tiles_full + g->tiles_last;
  } else {
    g->L_last = g->K_last = g->C = 0;
    g->tiles_full = g->tiles_last = g->tiles_bh = 0;
  }
  g->Cs = g->C;
  g->Ms = g->M;
  g->growing = false;
  g->base_len = g->capacity = g->C0 = g->K_last0 = g->F = g->Fmax = g->L_open = 0;
  g->open_id = g->tgt_id = g->K_tgt = g->cap = g->R0 = 0;
  g->closed_rows = g->M;
  const int base = c.base_len > 0 ? c.base_len : c.seq_len;
  const int capa = c.capacity > 0 ? c.capacity : c.seq_len;
  if (c.base_len < 0 || c.capacity < 0) {
    set_error("base_len and capacity must be >= 0");
    return false;
  }
  if (base == c.seq_len && capa == c.seq_len) return true;  // compact
  // growing index: the prefill's segments, then whole appended segments,
  // then one open segment of K_full clusters
  if (!(base <= c.seq_len && c.seq_len <= capa) || base <= steady || c.steady_recent < 1) {
    set_error("growing index needs steady_initial + steady_recent < base_len <= seq_len <= "
              "capacity and steady_recent >= 1 (got %d, %d, %d)", base, c.seq_len, capa);
    return false;
  }
  if ((long long)c.batch * c.num_kv_heads * capa > (1ll << 31) - 1) {
    set_error("batch * num_kv_heads * capacity must be < 2^31");
    return false;
  }
  g->growing = true;
  g->base_len = base;
  g->capacity = capa;
  const int M0 = base - (int)steady;
  const int S0 = (M0 + c.seg_len - 1) / c.seg_len;
  const int L0 = M0 - (S0 - 1) * c.seg_len;
  g->K_last0 = c.clusters_per_seg < L0 ? c.clusters_per_seg : L0;
  g->C0 = (S0 - 1) * g->K_full + g->K_last0;
  const int A = c.seq_len - base;
  g->F = A / c.seg_len;
  g->L_open = A % c.seg_len;
  g->Fmax = (capa - base) / c.seg_len;
  g->open_id = g->C0 + g->F * g->K_full;
  g->C = g->open_id + g->K_full;
  g->Cs = g->C0 + g->Fmax * g->K_full + g->K_full;
  g->tgt_id = g->F == 0 ? g->C0 - g->K_last0 : g->C0 + (g->F - 1) * g->K_full;
  g->K_tgt = g->F == 0 ? g->K_last0 : g->K_full;
  g->cap = (2 * c.seg_len + g->K_tgt - 1) / g->K_tgt;
  g->closed_rows = M0 + g->F * c.seg_len;
  g->R0 = M0 + g->Fmax * c.seg_len;
  g->Ms = g->R0 + 2 * c.seg_len + g->K_full;
  g->S = S0 + g->F + 1;  // closed segments and the open one
  // the k-means build geometry fields describe the prefill only
  return true;
}

ri_status make_decode_layout(const Geometry& g, const ri_decode_config* dcfg, DecodeLayout* L) {
  if (!dcfg) {
    set_error("decode config is NULL");
    return RI_ERR_INVALID_ARG;
  }
  if (dcfg->k_retrieval < 0 || dcfg->k_estimation < 0) {
    set_error("k_retrieval and k_estimation must be >= 0");
    return RI_ERR_INVALID_ARG;
  }
  if (dcfg->k_retrieval > kMaxRetrieval) {
    set_error("k_retrieval must be <= %d (got %d)", kMaxRetrieval, dcfg->k_retrieval);
    return RI_ERR_INVALID_ARG;
  }
  if ((long long)dcfg->k_retrieval + dcfg->k_estimation > (1 << 24)) {
    set_error("k_retrieval + k_estimation too large");
    return RI_ERR_INVALID_ARG;
  }
  L->k_r = dcfg->k_retrieval;
  L->k_e = dcfg->k_estimation;
  L->kr = L->k_r < g.C ? L->k_r : g.C;
  L->ke = L->k_e < g.C - L->kr ? L->k_e : g.C - L->kr;
  L->Gp = g.G <= 4 ? 4 : 8;
  L->CS = 0;  // chosen per device by decode_plan
  if ((long long)g.C > (long long)kMaxClusterBlocks * kMaxIdsPerBlock) {
    set_error("%d clusters per (sequence, KV head): the decode kernel handles at most %d", g.C,
              kMaxClusterBlocks * kMaxIdsPerBlock);
    return RI_ERR_UNSUPPORTED;
  }
  const long long BH = g.BH();
  size_t off = kStatusBytesHost;
  L->off_score = off;
  off = align_up(off + (size_t)BH * g.Cs * L->Gp * 4, 256);  // room for every live C
  L->off_sel = off;
  off = align_up(off + (size_t)BH * (L->k_r + L->k_e) * 4, 256);
  L->off_rpre = off;
  off = align_up(off + (size_t)BH * (L->k_r + 1) * 4, 256);
  L->total = off;
  return RI_OK;
}

bool make_build_layout(const Geometry& g, BuildLayout* L) {
  const size_t BH = (size_t)g.BH();
  size_t off = kStatusBytesHost;
  L->off_mu = off;
  off = align_up(off + BH * g.C * 128 * 4, 1024);
  L->off_mu_bf16 = off;
  off = align_up(off + BH * g.C * 128 * 2, 1024);
  L->off_nsplit = off;
  off = align_up(off + BH * g.S * 512 * 16 * 2, 1024);
  L->off_ust = off;
  off = align_up(off + BH * g.S * 2 * 4, 256);
  L->off_counts = off;
  off = align_up(off + BH * g.C * 4, 256);
  L->off_labels = off;
  off = align_up(off + BH * g.M * 4, 256);
  L->off_knorm = off;
  off = align_up(off + BH * g.M * 4, 256);
  L->off_queue = off;
  off = align_up(off + build_queue_bytes((long long)BH * g.M), 256);
  L->off_members = off;
  off = align_up(off + BH * g.M * 4, 256);
  L->off_mstart = off;
  off = align_up(off + BH * g.S * 513 * 4, 256);
  L->off_ecs = off;
  off = align_up(off + BH * g.S * 512 * 8, 256);
  L->total = off;
  return true;
}

bool make_append_layout(const Geometry& g, const ri_index_config* cfg, AppendLayout* L) {
  ri_index_config c = *cfg;
  c.seq_len = c.seg_len;  // one segment per unit, no steady zone
  c.steady_initial = c.steady_recent = 0;
  c.base_len = c.capacity = 0;
  if (!make_geometry(&c, &L->gb)) return false;
  make_build_layout(L->gb, &L->bl);
  const size_t BH = (size_t)g.BH(), n = (size_t)g.seg_len, K = (size_t)g.K_full;
  size_t off = align_up(L->bl.total, 1024);
  L->off_sK = off;
  off = align_up(off + BH * n * 256, 1024);
  L->off_sV = off;
  off = align_up(off + BH * n * 256, 1024);
  L->off_Kp = off;
  off = align_up(off + BH * n * 256, 1024);
  L->off_Vp = off;
  off = align_up(off + BH * n * 256, 1024);
  L->off_perm = off;
  off = align_up(off + BH * n * 4, 256);
  L->off_cent = off;
  off = align_up(off + BH * K * 256, 256);
  L->off_counts = off;
  off = align_up(off + BH * K * 4, 256);
  L->off_offsets = off;
  off = align_up(off + BH * (K + 1) * 4, 256);
  L->off_vsum = off;
  off = align_up(off + BH * K * 512, 256);
  L->total = off;
  return true;
}

}  // namespace ri

using namespace ri;

#define RI_CHECK(cond, code, ...) \
  do {                            \
    if (!(cond)) {                \
      set_error(__VA_ARGS__);     \
      return code;                \
    }                             \
  } while (0)

static ri_status cuda_fail(cudaError_t e, const char* what) {
  set_error("%s: %s", what, cudaGetErrorString(e));
  return RI_ERR_CUDA;
}

namespace ri {
ri_status check_gather_buffers(const ri_gather_buffers* bufs) {
  RI_CHECK(bufs, RI_ERR_INVALID_ARG, "gather buffers are NULL");
  RI_CHECK(bufs->units >= 1 && bufs->M >= 0 && bufs->pool_rows >= 0 && bufs->exec_rows >= 0,
           RI_ERR_INVALID_ARG, "bad gather buffer sizes");
  const void* ptrs[] = {bufs->host_K, bufs->host_V, bufs->cache_K, bufs->cache_V, bufs->exec_K,
                        bufs->exec_V};
  for (const void* q : ptrs)
    RI_CHECK(!q || aligned16(q), RI_ERR_INVALID_ARG, "gather buffers must be 16-byte aligned");
  RI_CHECK((bufs->host_K == nullptr) == (bufs->host_V == nullptr) &&
               (bufs->cache_K == nullptr) == (bufs->cache_V == nullptr) &&
               (bufs->exec_K == nullptr) == (bufs->exec_V == nullptr),
           RI_ERR_INVALID_ARG, "K and V buffers must be given together");
  return RI_OK;
}
}  // namespace ri

extern "C" {

const char* ri_status_string(ri_status s) {
  switch (s) {
    case RI_OK: return "ok";
    case RI_ERR_INVALID_ARG: return "invalid argument";
    case RI_ERR_UNSUPPORTED: return "unsupported";
    case RI_ERR_WORKSPACE: return "workspace too small";
    case RI_ERR_CAPACITY: return "capacity exceeded";
    case RI_ERR_CUDA: return "CUDA error";
    case RI_ERR_TIMEOUT: return "device wait timed out";
    case RI_ERR_HOST: return "host failure";
  }
  return "unknown status";
}

const char* ri_last_error(void) { return ri::g_last_error; }

ri_status ri_index_geometry(const ri_index_config* cfg, ri_geometry* out) {
  Geometry g;
  if (!make_geometry(cfg, &g)) return RI_ERR_INVALID_ARG;
  RI_CHECK(out, RI_ERR_INVALID_ARG, "out is NULL");
  out->middle = g.M;
  out->num_segments = g.S;
  out->clusters = g.C;
  out->cluster_stride = g.Cs;
  out->row_stride = g.Ms;
  out->steady = g.n_steady;
  return RI_OK;
}

ri_status ri_default_budgets(int32_t clusters, ri_decode_config* out) {
  RI_CHECK(out, RI_ERR_INVALID_ARG, "out is NULL");
  RI_CHECK(clusters >= 0, RI_ERR_INVALID_ARG, "clusters must be >= 0");
  // round half up of 1.8 % and 23 % of C, in exact integer arithmetic
  out->k_retrieval = (int32_t)((18LL * clusters + 500) / 1000);
  out->k_estimation = (int32_t)((23LL * clusters + 50) / 100);
  return RI_OK;
}

size_t ri_build_index_workspace(const ri_index_config* cfg) {
  Geometry g;
  if (!make_geometry(cfg, &g) || g.growing) return 0;
  BuildLayout L;
  make_build_layout(g, &L);
  return L.total;
}

size_t ri_decode_workspace(const ri_index_config* cfg, const ri_decode_config* dcfg) {
  Geometry g;
  if (!make_geometry(cfg, &g)) return 0;
  DecodeLayout L;
  if (make_decode_layout(g, dcfg, &L) != RI_OK) return 0;
  return L.total;
}

static ri_status check_index_pointers(const Geometry& g, const ri_index* idx, bool for_build) {
  RI_CHECK(idx, RI_ERR_INVALID_ARG, "index is NULL");
  if (g.n_steady > 0) {
    RI_CHECK(idx->Ks && idx->Vs, RI_ERR_INVALID_ARG, "index Ks/Vs is NULL");
    RI_CHECK(aligned16(idx->Ks) && aligned16(idx->Vs), RI_ERR_INVALID_ARG,
             "index Ks/Vs must be 16-byte aligned");
  }
  RI_CHECK(idx->offsets && aligned16(idx->offsets), RI_ERR_INVALID_ARG,
           "index offsets must be non-NULL and 16-byte aligned");
  if (g.M > 0) {
    const void* ptrs[] = {idx->Kp, idx->Vp, idx->perm, idx->centroid, idx->counts, idx->vsum};
    const char* names[] = {"Kp", "Vp", "perm", "centroid", "counts", "vsum"};
    for (int i = 0; i < 6; ++i) {
      RI_CHECK(ptrs[i], RI_ERR_INVALID_ARG, "index %s is NULL", names[i]);
      RI_CHECK(aligned16(ptrs[i]), RI_ERR_INVALID_ARG, "index %s must be 16-byte aligned",
               names[i]);
    }
  }
  if (for_build) {
    RI_CHECK(!idx->labels || aligned16(idx->labels), RI_ERR_INVALID_ARG,
             "labels must be 16-byte aligned");
    RI_CHECK(!idx->objective || aligned16(idx->objective), RI_ERR_INVALID_ARG,
             "objective must be 16-byte aligned");
  }
  return RI_OK;
}

ri_status ri_build_index(const ri_index_config* cfg, const void* K, const void* V,
                         const int32_t* init_pos, const ri_index* out, void* workspace,
                         size_t workspace_bytes, ri_stream_t stream) {
  Geometry g;
  if (!make_geometry(cfg, &g)) return RI_ERR_INVALID_ARG;
  RI_CHECK(!g.growing, RI_ERR_UNSUPPORTED,
           "the build makes a compact index (base_len and capacity 0 or seq_len); open it "
           "with ri_index_open to let it grow");
  RI_CHECK(K && V, RI_ERR_INVALID_ARG, "K and V must be non-NULL");
  RI_CHECK(aligned16(K) && aligned16(V), RI_ERR_INVALID_ARG, "K and V must be 16-byte aligned");
  RI_CHECK(!init_pos || aligned16(init_pos), RI_ERR_INVALID_ARG,
           "init_pos must be 16-byte aligned");
  ri_status st = check_index_pointers(g, out, true);
  if (st != RI_OK) return st;
  BuildLayout L;
  make_build_layout(g, &L);
  RI_CHECK(workspace, RI_ERR_INVALID_ARG, "workspace is NULL");
  RI_CHECK((reinterpret_cast<uintptr_t>(workspace) & 1023u) == 0, RI_ERR_INVALID_ARG,
           "workspace must be 1024-byte aligned");
  RI_CHECK(workspace_bytes >= L.total, RI_ERR_WORKSPACE,
           "workspace has %zu bytes, build needs %zu", workspace_bytes, L.total);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytesHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status)");
  BuildArgs a;
  a.K = K;
  a.V = V;
  a.init_pos = init_pos;
  a.out = *out;
  a.ws = static_cast<char*>(workspace);
  return launch_build(g, L, a, s);
}

static ri_status prepare_decode(const ri_index_config* cfg, const ri_decode_config* dcfg,
                                const void* q, const ri_index* idx, void* workspace,
                                size_t workspace_bytes, Geometry* g, DecodeLayout* L) {
  if (!make_geometry(cfg, g)) return RI_ERR_INVALID_ARG;
  const ri_status ls = make_decode_layout(*g, dcfg, L);
  if (ls != RI_OK) return ls;
  RI_CHECK(q && aligned16(q), RI_ERR_INVALID_ARG, "q must be non-NULL and 16-byte aligned");
  ri_status st = check_index_pointers(*g, idx, false);
  if (st != RI_OK) return st;
  RI_CHECK(workspace && aligned16(workspace), RI_ERR_INVALID_ARG,
           "workspace must be non-NULL and 16-byte aligned");
  RI_CHECK(workspace_bytes >= L->total, RI_ERR_WORKSPACE,
           "workspace has %zu bytes, decode needs %zu", workspace_bytes, L->total);
  return RI_OK;
}

static DecodeArgs decode_args(const void* q, const ri_index* idx, void* out, float* lse,
                              int32_t* sel, int32_t* rpre, void* ws) {
  DecodeArgs a0;
  a0.wait_ns = kWaitLimitNsHost;
  a0.fault = RI_FAULT_NONE;
  DecodeArgs a;
  a.q = q;
  a.centroid = idx->centroid;
  a.counts = idx->counts;
  a.offsets = idx->offsets;
  a.vsum = idx->vsum;
  a.Kp = idx->Kp;
  a.Vp = idx->Vp;
  a.Ks = idx->Ks;
  a.Vs = idx->Vs;
  a.exec_K = nullptr;
  a.exec_V = nullptr;
  a.exec_rows = 0;
  a.out = out;
  a.lse = lse;
  a.sel_user = sel;
  a.rpre_user = rpre;
  a.ws = static_cast<char*>(ws);
  a.wait_ns = a0.wait_ns;
  a.fault = a0.fault;
  return a;
}

ri_status ri_decode_attention(const ri_index_config* cfg, const ri_decode_config* dcfg,
                              const void* q, const ri_index* idx, void* out, float* lse,
                              int32_t* sel_ids, void* workspace, size_t workspace_bytes,
                              ri_stream_t stream) {
  Geometry g;
  DecodeLayout L;
  ri_status st = prepare_decode(cfg, dcfg, q, idx, workspace, workspace_bytes, &g, &L);
  if (st != RI_OK) return st;
  RI_CHECK(out && aligned16(out), RI_ERR_INVALID_ARG, "out must be non-NULL and 16-byte aligned");
  RI_CHECK(!sel_ids || aligned16(sel_ids), RI_ERR_INVALID_ARG, "sel_ids must be 16-byte aligned");
  if (!decode_plan(g, &L)) return RI_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DecodeArgs a = decode_args(q, idx, out, lse, sel_ids, nullptr, workspace);
  cudaError_t e = launch_decode(g, L, a, s);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return RI_OK;
}

ri_status ri_decode_attention_host(const ri_index_config* cfg, const ri_decode_config* dcfg,
                                   const void* q_host, void* q_dev, const ri_index* idx,
                                   void* out_dev, void* out_host, float* lse, void* workspace,
                                   size_t workspace_bytes, ri_stream_t stream) {
  Geometry g;
  DecodeLayout L;
  ri_status st = prepare_decode(cfg, dcfg, q_dev, idx, workspace, workspace_bytes, &g, &L);
  if (st != RI_OK) return st;
  RI_CHECK(q_host && out_host, RI_ERR_INVALID_ARG, "q_host and out_host must be non-NULL");
  RI_CHECK(out_dev && aligned16(out_dev), RI_ERR_INVALID_ARG,
           "out_dev must be non-NULL and 16-byte aligned");
  if (!decode_plan(g, &L)) return RI_ERR_UNSUPPORTED;
  const size_t bytes = (size_t)g.BH() * g.G * g.d * 2;  // q and out: bf16 [B][H G][d]
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(q_dev, q_host, bytes, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return cuda_fail(e, "query copy to the device");
  DecodeArgs a = decode_args(q_dev, idx, out_dev, lse, nullptr, nullptr, workspace);
  e = launch_decode(g, L, a, s);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  e = cudaMemcpyAsync(out_host, out_dev, bytes, cudaMemcpyDeviceToHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "output copy to the host");
  e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronisation");
  return RI_OK;
}

ri_status ri_selftest_decode_timeout(const ri_index_config* cfg, const ri_decode_config* dcfg,
                                     const void* q, const ri_index* idx, void* out,
                                     void* workspace, size_t workspace_bytes, int32_t hand_off,
                                     uint64_t limit_ns, ri_stream_t stream) {
  Geometry g;
  DecodeLayout L;
  ri_status st = prepare_decode(cfg, dcfg, q, idx, workspace, workspace_bytes, &g, &L);
  if (st != RI_OK) return st;
  RI_CHECK(out && aligned16(out), RI_ERR_INVALID_ARG, "out must be non-NULL and 16-byte aligned");
  RI_CHECK(hand_off >= RI_FAULT_SCORE_COPY && hand_off <= RI_FAULT_SCORE_SIZES,
           RI_ERR_INVALID_ARG, "hand_off must be 1, 2 or 3 (got %d)", hand_off);
  RI_CHECK(limit_ns > 0 && limit_ns <= 10ull * 1000000000ull, RI_ERR_INVALID_ARG,
           "limit_ns must be in (0, 10 s]");
  if (!decode_plan(g, &L)) return RI_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DecodeArgs a = decode_args(q, idx, out, nullptr, nullptr, nullptr, workspace);
  a.wait_ns = limit_ns;
  a.fault = hand_off;
  cudaError_t e = launch_decode(g, L, a, s);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  return RI_OK;
}

ri_status ri_decode_attention_static(const ri_index_config* cfg, const ri_decode_config* dcfg,
                                     const void* q, const ri_index* idx, void* out, float* lse,
                                     int32_t* sel_ids, int32_t* device_status,
                                     ri_stream_t stream) {
  Geometry g;
  DecodeLayout L;
  if (!make_geometry(cfg, &g)) return RI_ERR_INVALID_ARG;
  const ri_status ls = make_decode_layout(g, dcfg, &L);
  if (ls != RI_OK) return ls;
  RI_CHECK(L.total <= kStaticScratchBytes, RI_ERR_CAPACITY,
           "decode needs %zu bytes of scratch, the static array holds %zu", L.total,
           kStaticScratchBytes);
  RI_CHECK(!device_status || aligned4(device_status), RI_ERR_INVALID_ARG,
           "device_status must be 4-byte aligned");
  void* ws = nullptr;
  cudaError_t e = static_decode_scratch(&ws);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(static decode scratch)");
  ri_status st = prepare_decode(cfg, dcfg, q, idx, ws, kStaticScratchBytes, &g, &L);
  if (st != RI_OK) return st;
  RI_CHECK(out && aligned16(out), RI_ERR_INVALID_ARG, "out must be non-NULL and 16-byte aligned");
  RI_CHECK(!sel_ids || aligned16(sel_ids), RI_ERR_INVALID_ARG, "sel_ids must be 16-byte aligned");
  if (!decode_plan(g, &L)) return RI_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  e = cudaMemsetAsync(ws, 0, kStatusBytesHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status)");
  DecodeArgs a = decode_args(q, idx, out, lse, sel_ids, nullptr, ws);
  e = launch_decode(g, L, a, s);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  if (device_status) {
    e = cudaMemcpyAsync(device_status, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "copying the device status");
  }
  return RI_OK;
}

ri_status ri_select_clusters(const ri_index_config* cfg, const ri_decode_config* dcfg,
                             const void* q, const ri_index* idx, int32_t* sel_ids,
                             int32_t* retr_rows, void* workspace, size_t workspace_bytes,
                             ri_stream_t stream) {
  Geometry g;
  DecodeLayout L;
  ri_status st = prepare_decode(cfg, dcfg, q, idx, workspace, workspace_bytes, &g, &L);
  if (st != RI_OK) return st;
  RI_CHECK(sel_ids && aligned16(sel_ids), RI_ERR_INVALID_ARG,
           "sel_ids must be non-NULL and 16-byte aligned");
  if (!decode_plan(g, &L)) return RI_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DecodeArgs a = decode_args(q, idx, nullptr, nullptr, sel_ids, retr_rows, workspace);
  cudaError_t e = launch_select(g, L, a, s);
  if (e != cudaSuccess) return cuda_fail(e, "select launch");
  return RI_OK;
}

ri_status ri_attend_selected(const ri_index_config* cfg, const ri_decode_config* dcfg,
                             const void* q, const ri_index* idx, const void* exec_K,
                             const void* exec_V, int32_t exec_rows, void* out, float* lse,
                             void* workspace, size_t workspace_bytes, ri_stream_t stream) {
  Geometry g;
  DecodeLayout L;
  ri_status st = prepare_decode(cfg, dcfg, q, idx, workspace, workspace_bytes, &g, &L);
  if (st != RI_OK) return st;
  RI_CHECK(out && aligned16(out), RI_ERR_INVALID_ARG, "out must be non-NULL and 16-byte aligned");
  RI_CHECK((exec_K == nullptr) == (exec_V == nullptr), RI_ERR_INVALID_ARG,
           "exec_K and exec_V must be both NULL or both non-NULL");
  if (exec_K) {
    RI_CHECK(aligned16(exec_K) && aligned16(exec_V), RI_ERR_INVALID_ARG,
             "exec buffers must be 16-byte aligned");
    RI_CHECK(exec_rows >= 1, RI_ERR_INVALID_ARG, "exec_rows must be >= 1");
  }
  if (!decode_plan(g, &L)) return RI_ERR_UNSUPPORTED;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DecodeArgs a = decode_args(q, idx, out, lse, nullptr, nullptr, workspace);
  a.exec_K = exec_K;
  a.exec_V = exec_V;
  a.exec_rows = exec_rows;
  cudaError_t e = launch_attend(g, L, a, s);
  if (e != cudaSuccess) return cuda_fail(e, "attend launch");
  return RI_OK;
}

ri_status ri_gather_blocks(const ri_gather_buffers* bufs, const ri_copy_desc* desc,
                           int32_t n_desc, void* workspace, ri_stream_t stream) {
  return ri_gather_blocks_shaped(bufs, desc, n_desc, 0, 0, workspace, stream);
}

ri_status ri_gather_shape(int64_t host_copies, int64_t total_copies, int32_t* threads,
                          int32_t* blocks_per_sm) {
  RI_CHECK(threads && blocks_per_sm, RI_ERR_INVALID_ARG, "gather shape: NULL output");
  RI_CHECK(host_copies >= 0 && total_copies >= host_copies, RI_ERR_INVALID_ARG,
           "gather shape: bad copy counts (%lld host of %lld)", (long long)host_copies,
           (long long)total_copies);
  // a list with any copy from host memory waits on the host link: the most
  // warps in flight (2048 threads per SM) keep the device copies from
  // queueing behind the slow ones; lists served from the device's own
  // memory stream at fewer, larger blocks
  if (host_copies > 0) {
    *threads = kGatherHostThreads;
    *blocks_per_sm = kGatherHostBlocksPerSM;
  } else {
    *threads = kGatherDeviceThreads;
    *blocks_per_sm = kGatherDeviceBlocksPerSM;
  }
  return RI_OK;
}

ri_status ri_gather_blocks_shaped(const ri_gather_buffers* bufs, const ri_copy_desc* desc,
                                  int32_t n_desc, int32_t threads, int32_t blocks_per_sm,
                                  void* workspace, ri_stream_t stream) {
  RI_CHECK(threads == 0 || (threads >= 32 && threads <= 512 && threads % 32 == 0),
           RI_ERR_INVALID_ARG, "threads per block must be 0 or a multiple of 32 in [32, 512]");
  RI_CHECK(blocks_per_sm >= 0 && blocks_per_sm <= 64, RI_ERR_INVALID_ARG,
           "blocks per SM must be in [0, 64]");
  RI_CHECK(n_desc >= 0, RI_ERR_INVALID_ARG, "n_desc must be >= 0");
  RI_CHECK(n_desc == 0 || desc, RI_ERR_INVALID_ARG, "descriptors are NULL");
  RI_CHECK(workspace && aligned16(workspace), RI_ERR_INVALID_ARG,
           "workspace must be non-NULL and 16-byte aligned");
  const ri_status bs = check_gather_buffers(bufs);
  if (bs != RI_OK) return bs;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytesHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status)");
  GatherArgs a;
  a.host_K = bufs->host_K;
  a.host_V = bufs->host_V;
  a.cache_K = bufs->cache_K;
  a.cache_V = bufs->cache_V;
  a.exec_K = bufs->exec_K;
  a.exec_V = bufs->exec_V;
  a.units = bufs->units;
  a.M = bufs->M;
  a.pool_rows = bufs->pool_rows;
  a.exec_rows = bufs->exec_rows;
  e = launch_gather(a, desc, n_desc, static_cast<int*>(workspace), s, threads, blocks_per_sm);
  if (e != cudaSuccess) return cuda_fail(e, "gather launch");
  return RI_OK;
}

ri_status ri_index_open(const ri_index_config* cfg, const ri_index* compact, const ri_index* out,
                        ri_stream_t stream) {
  Geometry g;
  if (!make_geometry(cfg, &g)) return RI_ERR_INVALID_ARG;
  RI_CHECK(g.growing && cfg->seq_len == g.base_len, RI_ERR_INVALID_ARG,
           "index open: cfg must describe a growing index at its prefill (seq_len == base_len "
           "< capacity)");
  ri_index_config cc = *cfg;
  cc.base_len = cc.capacity = 0;
  Geometry gc;
  if (!make_geometry(&cc, &gc)) return RI_ERR_INVALID_ARG;
  ri_status st = check_index_pointers(gc, compact, false);
  if (st != RI_OK) return st;
  if ((st = check_index_pointers(g, out, false)) != RI_OK) return st;
  RI_CHECK(out->perm && compact->perm, RI_ERR_INVALID_ARG, "index open: perm is NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t BH = (size_t)g.BH();
  struct Copy {
    void* dst;
    const void* src;
    size_t elem, dst_n, src_n;
  } copies[] = {
      {out->Kp, compact->Kp, 256, (size_t)g.Ms, (size_t)gc.M},
      {out->Vp, compact->Vp, 256, (size_t)g.Ms, (size_t)gc.M},
      {out->perm, compact->perm, 4, (size_t)g.Ms, (size_t)gc.M},
      {out->centroid, compact->centroid, 256, (size_t)g.Cs, (size_t)gc.C},
      {out->counts, compact->counts, 4, (size_t)g.Cs, (size_t)gc.C},
      {out->offsets, compact->offsets, 4, (size_t)g.Cs + 1, (size_t)gc.C + 1},
      {out->vsum, compact->vsum, 512, (size_t)g.Cs, (size_t)gc.C},
  };
  for (const Copy& c : copies) {
    cudaError_t e = cudaMemcpy2DAsync(c.dst, c.dst_n * c.elem, c.src, c.src_n * c.elem,
                                      c.src_n * c.elem, BH, cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e, "index open: cudaMemcpy2DAsync");
  }
  const size_t steady_bytes = BH * (size_t)g.n_steady * 256;
  cudaError_t e = cudaMemcpyAsync(out->Ks, compact->Ks, steady_bytes, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(out->Vs, compact->Vs, steady_bytes, cudaMemcpyDeviceToDevice, s);
  if (e == cudaSuccess) e = launch_open_init(g, *out, s);
  if (e != cudaSuccess) return cuda_fail(e, "index open");
  return RI_OK;
}

size_t ri_index_append_workspace(const ri_index_config* cfg) {
  Geometry g;
  if (!make_geometry(cfg, &g) || !g.growing) return 0;
  AppendLayout L;
  if (!make_append_layout(g, cfg, &L)) return 0;
  return L.total;
}

ri_status ri_index_append(const ri_index_config* cfg, const void* k_new, const void* v_new,
                          const ri_index* idx, int32_t* assigned, void* workspace,
                          size_t workspace_bytes, ri_stream_t stream) {
  Geometry g;
  if (!make_geometry(cfg, &g)) return RI_ERR_INVALID_ARG;
  RI_CHECK(g.growing, RI_ERR_INVALID_ARG, "index append: cfg is not a growing index");
  RI_CHECK(cfg->seq_len < g.capacity, RI_ERR_CAPACITY,
           "index append: the layout is full (%d tokens)", g.capacity);
  RI_CHECK(k_new && v_new && aligned16(k_new) && aligned16(v_new), RI_ERR_INVALID_ARG,
           "k_new and v_new must be non-NULL and 16-byte aligned");
  RI_CHECK(!assigned || aligned4(assigned), RI_ERR_INVALID_ARG, "assigned must be aligned");
  ri_status st = check_index_pointers(g, idx, false);
  if (st != RI_OK) return st;
  RI_CHECK(idx->perm, RI_ERR_INVALID_ARG, "index append: perm is NULL");
  AppendLayout L;
  if (!make_append_layout(g, cfg, &L)) return RI_ERR_INVALID_ARG;
  RI_CHECK(workspace && (reinterpret_cast<uintptr_t>(workspace) & 1023u) == 0,
           RI_ERR_INVALID_ARG, "workspace must be non-NULL and 1024-byte aligned");
  RI_CHECK(workspace_bytes >= L.total, RI_ERR_WORKSPACE,
           "workspace has %zu bytes, append needs %zu", workspace_bytes, L.total);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  int* status = reinterpret_cast<int*>(ws);
  cudaError_t e = launch_append(g, *idx, k_new, v_new, assigned, status, s);
  if (e != cudaSuccess) return cuda_fail(e, "index append");
  if ((g.L_open + 1) % g.seg_len != 0) return RI_OK;
  // the open segment is full: k-means turns it into a closed segment
  e = launch_close_gather(g, *idx, ws + L.off_sK, ws + L.off_sV, status, s);
  if (e != cudaSuccess) return cuda_fail(e, "index append: close gather");
  ri_index seg = {};
  seg.Kp = ws + L.off_Kp;
  seg.Vp = ws + L.off_Vp;
  seg.perm = reinterpret_cast<int32_t*>(ws + L.off_perm);
  seg.centroid = ws + L.off_cent;
  seg.counts = reinterpret_cast<int32_t*>(ws + L.off_counts);
  seg.offsets = reinterpret_cast<int32_t*>(ws + L.off_offsets);
  seg.vsum = reinterpret_cast<float*>(ws + L.off_vsum);
  BuildArgs a;
  a.K = ws + L.off_sK;
  a.V = ws + L.off_sV;
  a.init_pos = nullptr;
  a.out = seg;
  a.ws = ws;
  st = launch_build(L.gb, L.bl, a, s);
  if (st != RI_OK) return st;
  e = launch_close_scatter(g, *idx, seg, s);
  if (e != cudaSuccess) return cuda_fail(e, "index append: close scatter");
  ri_index_config next = *cfg;
  next.seq_len += 1;
  Geometry gn;
  if (!make_geometry(&next, &gn)) return RI_ERR_INVALID_ARG;
  e = launch_open_init(gn, *idx, s);
  if (e != cudaSuccess) return cuda_fail(e, "index append: open segment");
  return RI_OK;
}

ri_status ri_read_device_status(void* workspace, ri_stream_t stream) {
  RI_CHECK(workspace, RI_ERR_INVALID_ARG, "workspace is NULL");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device status");
  if (v != RI_OK) {
    set_error("device reported: %s", ri_status_string((ri_status)v));
    e = cudaMemsetAsync(workspace, 0, sizeof(int), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device status");
  }
  return (ri_status)v;
}

ri_status ri_selftest_wait_timeout(void* workspace, uint64_t limit_ns, ri_stream_t stream) {
  RI_CHECK(workspace && aligned16(workspace), RI_ERR_INVALID_ARG,
           "workspace must be non-NULL and 16-byte aligned");
  RI_CHECK(limit_ns > 0 && limit_ns <= 10ull * 1000000000ull, RI_ERR_INVALID_ARG,
           "limit_ns must be in (0, 10 s]");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytesHost, s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status)");
  e = launch_wait_timeout_selftest(static_cast<int*>(workspace), limit_ns, s);
  if (e != cudaSuccess) return cuda_fail(e, "self-test launch");
  return RI_OK;
}

}  // extern "C"
