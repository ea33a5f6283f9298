// Host-side shapes, workspace layouts and kernel launchers shared by the
// C ABI (api.cpp) and the CUDA translation units.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "retroinfer.h"

namespace ri {

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr int kMaxGroupHost = 8;          // query heads per KV head
constexpr size_t kStatusBytesHost = 256;  // status word region at workspace start
constexpr unsigned long long kWaitLimitNsHost = 2000000000ull;  // bounded device waits: 2 s

// Everything derived from an ri_index_config.
struct Geometry {
  int B, H, G, d, N;
  int seg_len, K;          // tokens per segment, clusters per full segment
  int iters;
  int s0, s1;              // steady initial / recent
  int M;                   // middle tokens
  int S;                   // segments
  int C;                   // clusters per (b, h)
  int n_steady;            // steady tokens per (b, h)
  int m0;                  // first middle position
  int K_full;              // clusters of a full segment = min(K, seg_len)
  int L_last, K_last;      // length / clusters of the last segment
  int tiles_full, tiles_last, tiles_bh;  // 128-row assignment tiles
  // Layout strides per unit: Cs clusters, Ms rows (= C, M for a compact
  // index; the capacity layout of a growing index otherwise).
  int Cs, Ms;
  // Growing index (index maintenance during decode; all 0 / false when
  // compact): prefill of base_len tokens, room for `capacity` tokens.
  bool growing;
  int base_len, capacity;
  int C0, K_last0;   // clusters of the prefill's segments, of its last segment
  int F, Fmax;       // closed appended segments (now / at capacity)
  int L_open;        // tokens in the open segment
  int open_id;       // first open cluster id (K_full open clusters follow)
  int tgt_id, K_tgt; // the last closed segment's clusters (assignment targets)
  int cap;           // member slots of one open cluster
  int R0;            // first row of the open region
  int closed_rows;   // rows of the closed segments (cluster-contiguous from row 0)
  long long BH() const { return (long long)B * H; }
};

// Returns false (and sets the thread's last error) for an invalid config.
bool make_geometry(const ri_index_config* cfg, Geometry* g);

// --------------------------------------------------------------- decode
constexpr int kMaxIdsPerBlock = 4096;  // clusters of a unit one decode block scores
constexpr int kMaxClusterBlocks = 16;  // blocks of the thread-block cluster of one unit
constexpr int kMaxRetrieval = 4096;    // k_retrieval limit (retrieval-row prefix)

struct DecodeLayout {
  int k_r, k_e;  // requested budgets (sizes of the sel regions)
  int kr, ke;    // clamped to C
  int CS;        // blocks per unit (thread-block cluster size)
  int Gp;        // scores stored per cluster: 4 (G <= 4) or 8
  // status region [0, 256); score fp32 [BH][C][Gp]; sel int32 [BH][k_r + k_e];
  // rpre int32 [BH][k_r + 1] (the last two hold a selection between
  // ri_select_clusters and ri_attend_selected)
  size_t off_score, off_sel, off_rpre, total;
};

// RI_OK, or the status of the first failed check (the thread's last error
// says which).
ri_status make_decode_layout(const Geometry& g, const ri_decode_config* dcfg, DecodeLayout* L);

// Test hook of the decode kernel's bounded waits: which hand-off is left
// unreleased (0 in every public call).
enum {
  RI_FAULT_NONE = 0,
  RI_FAULT_SCORE_COPY = 1,    // the first centroid tile's copy is never issued
  RI_FAULT_SCORE_COMMIT = 2,  // the first tile's MMA completion is never signalled
  RI_FAULT_SCORE_SIZES = 3    // the cluster sizes loaded for scoring are never signalled
};

struct DecodeArgs {
  const void* q;
  const void* centroid;
  const int32_t* counts;
  const int32_t* offsets;
  const float* vsum;
  const void* Kp;
  const void* Vp;
  const void* Ks;
  const void* Vs;
  const void* exec_K;  // NULL: read Kp/Vp in place
  const void* exec_V;
  int exec_rows;
  void* out;
  float* lse;
  int32_t* sel_user;
  int32_t* rpre_user;
  char* ws;
  unsigned long long wait_ns;  // limit of every bounded wait
  int fault;                   // RI_FAULT_* (test hook)
};

cudaError_t launch_decode(const Geometry& g, const DecodeLayout& L, const DecodeArgs& a,
                          cudaStream_t s);
cudaError_t launch_select(const Geometry& g, const DecodeLayout& L, const DecodeArgs& a,
                          cudaStream_t s);
// Chooses the launch shape of the decode kernel (blocks per unit).
bool decode_plan(const Geometry& g, DecodeLayout* L);
cudaError_t launch_attend(const Geometry& g, const DecodeLayout& L, const DecodeArgs& a,
                          cudaStream_t s);

// Fixed scratch of ri_decode_attention_static (static_scratch.cu): the
// current device's copy, looked up once per device.
constexpr size_t kStaticScratchBytes = RI_STATIC_SCRATCH_BYTES;
cudaError_t static_decode_scratch(void** addr);

// --------------------------------------------------------------- gather
struct GatherArgs {
  const void* host_K;
  const void* host_V;
  void* cache_K;
  void* cache_V;
  void* exec_K;
  void* exec_V;
  int units, M, pool_rows, exec_rows;
};
// Launch shape of the gather: threads per block (a multiple of 32, at most
// 512) and the most blocks per SM the grid may hold; 0 picks the defaults.
constexpr int kGatherDefaultThreads = 256;
constexpr int kGatherDefaultBlocksPerSM = 8;
// shapes ri_gather_shape picks per hit pattern (from a sweep on B200: lists
// with host copies want the most warps in flight, device-only lists need
// about 1024 threads per SM and are flat beyond)
constexpr int kGatherHostThreads = 256, kGatherHostBlocksPerSM = 8;
constexpr int kGatherDeviceThreads = 512, kGatherDeviceBlocksPerSM = 1;
cudaError_t launch_gather(const GatherArgs& a, const ri_copy_desc* desc, int n_desc, int* status,
                          cudaStream_t s, int threads = 0, int blocks_per_sm = 0);
// Argument checks of ri_gather_buffers (pointers, alignment, sizes).
ri_status check_gather_buffers(const ri_gather_buffers* bufs);

// --------------------------------------------------------------- build
constexpr int kMaxSegLen = 16384;  // segment tokens (the sort stages labels in shared memory)

struct BuildLayout {
  // mu fp32 [BH][C][d]; mu_bf16 [BH][C][d] (MMA operand); nsplit
  // [BH*S][512][16] bf16 (-||mu_j||^2 / 2 in three bf16 parts, -inf past K_s;
  // plain K-major MMA operand layout); ust fp32 [BH*S][2] (max e_j, max c_j);
  // counts int32 [BH][C]; labels int32 [BH][M]; knorm fp32 [BH][M] (||k||);
  // queue of rows for the exact fix-up [BH*M] entries; members int32 [BH][M]
  // (positions within the segment, grouped by cluster in position order);
  // mstart int32 [BH*S][513] (first member of each cluster); ecs fp32
  // [BH*S][512][2] (e_j, c_j of each centroid, reduced into ust).
  size_t off_mu, off_mu_bf16, off_nsplit, off_ust, off_counts, off_labels, off_knorm, off_queue,
      off_members, off_mstart, off_ecs, total;
};
size_t build_queue_bytes(long long rows);
bool make_build_layout(const Geometry& g, BuildLayout* L);

struct BuildArgs {
  const void* K;
  const void* V;
  const int32_t* init_pos;
  ri_index out;
  char* ws;
};

ri_status launch_build(const Geometry& g, const BuildLayout& L, const BuildArgs& a,
                       cudaStream_t s);

cudaError_t launch_wait_timeout_selftest(int* status, unsigned long long limit_ns,
                                         cudaStream_t s);

// --------------------------------------------------------------- growing index
// Workspace of ri_index_append: the close's segment build from offset 0 (its
// status word is the call's), then the open tokens in position order
// (sK, sV [BH][seg_len][d]) and the built segment (a compact index of one
// segment per unit).
struct AppendLayout {
  Geometry gb;     // geometry of the close's build (seq_len = seg_len, no steady zone)
  BuildLayout bl;
  size_t off_sK, off_sV, off_Kp, off_Vp, off_perm, off_cent, off_counts, off_offsets, off_vsum;
  size_t total;
};
bool make_append_layout(const Geometry& g, const ri_index_config* cfg, AppendLayout* L);
cudaError_t launch_open_init(const Geometry& g, const ri_index& idx, cudaStream_t s);
cudaError_t launch_append(const Geometry& g, const ri_index& idx, const void* k_new,
                          const void* v_new, int32_t* assigned, int* status, cudaStream_t s);
cudaError_t launch_close_gather(const Geometry& g, const ri_index& idx, void* sK, void* sV,
                                int* status, cudaStream_t s);
cudaError_t launch_close_scatter(const Geometry& g, const ri_index& idx, const ri_index& seg,
                                 cudaStream_t s);

// Thread-local last error.
void set_error(const char* fmt, ...);
int num_sms();
// Raises a kernel's dynamic shared memory limit once per device (outside any
// stream capture after the first call on that device).  `slot` names the
// kernel in a fixed table (kSmemSlots entries).
constexpr int kSmemSlots = 16;
cudaError_t set_smem_once(int slot, const void* func, int bytes);

}  // namespace ri
