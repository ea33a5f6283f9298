/*
 * retroinfer.h -- C ABI of the wave-index decode path for NVIDIA B200 (sm_100a).
 *
 * The wave index is the attention-aware vector index of RetroInfer (arXiv
 * 2505.02922).  Sources, cited by page title and section:
 *   [P1] "微软新突破：RetroInfer如何让AI模型处理百万级文本不再'卡顿'？"
 *        (techwalker.com), section 三 (wave index, wave buffer).
 *   [P2] "KV缓存技术与RetroInfer系统在长上下文推理中的优化实践" (framerc.cn),
 *        §2.1 Wave索引, §2.2 Wave缓冲, §3.1 cache layout, §3.2 execution
 *        buffer assembly, §3.3 attention kernels.
 *   [P3] "RetroInfer: A Vector-Storage Approach for Scalable Long-Context LLM
 *        Inference" (chatpaper.ai), abstract.
 *   [P4] "RetroInfer: A Vector Storage Engine for Scalable Long-Context LLM
 *        Inference" (gist.science), "Technische Samenvatting" §2.
 *
 * Conventions for every call below:
 *  - Tensors are caller-owned DEVICE memory unless a parameter says "host".
 *    Device pointers must be 16-byte aligned.  bf16 = IEEE bfloat16 stored as
 *    uint16; fp32 = IEEE binary32.  Layouts are dense, row-major, in the order
 *    written ([B][H_kv][N][d] means d fastest).
 *  - Calls that take a stream are asynchronous on it (NULL = legacy default
 *    stream).  The current CUDA device must be the one that holds the
 *    stream and the tensors of the call.  Nothing is allocated by these
 *    calls; scratch memory is the caller's workspace, sized by the matching
 *    *_workspace() query, whose first 256 bytes (the status region) must be
 *    zero before its first use.
 *  - Invalid arguments are rejected on the host BEFORE any launch: the call
 *    returns an error status and ri_last_error() describes it.
 *  - Failures found on the device (a bounded wait that expired, an index that
 *    was out of range in device-resident input) are written to a status word
 *    at the start of the workspace; ri_read_device_status() reads and clears
 *    it.  The decode calls never clear it themselves (no extra launch per
 *    step): the first failure stays recorded until it is read.  The build
 *    and gather calls clear it when they start.
 *  - head_dim must be 128.  GQA: query head h_q uses KV head h_q / G.
 */
#ifndef RETROINFER_H_
#define RETROINFER_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* ri_stream_t; /* same type as cudaStream_t */

typedef enum {
  RI_OK = 0,
  RI_ERR_INVALID_ARG = 1, /* bad pointer, size or configuration value        */
  RI_ERR_UNSUPPORTED = 2, /* valid request outside what the kernels handle   */
  RI_ERR_WORKSPACE = 3,   /* workspace smaller than the *_workspace() query  */
  RI_ERR_CAPACITY = 4,    /* a cache or buffer capacity would be exceeded    */
  RI_ERR_CUDA = 5,        /* a CUDA runtime call failed                      */
  RI_ERR_TIMEOUT = 6,     /* a bounded device-side wait expired              */
  RI_ERR_HOST = 7         /* host-side failure (allocation, injected fault)  */
} ri_status;

/* Index geometry.  Zones [P2 §2.1 items 1-3; P1 三]: the steady zone is the
 * first `steady_initial` and last `steady_recent` tokens of every sequence;
 * the other M = max(0, N - steady_initial - steady_recent) "middle" tokens
 * are indexed.  Segmented clustering [P2 §2.1 pseudocode]: the middle tokens
 * are cut into contiguous segments of `seg_len` tokens (the last may be
 * short) and k-means runs on each segment with K_s = min(clusters_per_seg,
 * L_s) clusters.  Global cluster id = sum of K of earlier segments + local id.
 * Limits: 1 <= clusters_per_seg <= 512, 1 <= seg_len <= 16384, iters >= 0,
 * group_size 1..8, head_dim == 128. */
typedef struct {
  int32_t batch;            /* B                                    */
  int32_t num_kv_heads;     /* H_kv                                 */
  int32_t group_size;       /* G = H_q / H_kv                       */
  int32_t head_dim;         /* d (must be 128)                      */
  int32_t seq_len;          /* N, same for every sequence           */
  int32_t seg_len;          /* tokens per segment (8192)            */
  int32_t clusters_per_seg; /* K (512)                              */
  int32_t iters;            /* Lloyd iterations T (10)              */
  int32_t steady_initial;   /* 4                                    */
  int32_t steady_recent;    /* 64                                   */
  /* Growing index (ri_index_open / ri_index_append; 0 = seq_len for both,
   * a compact index):                                                    */
  int32_t base_len;         /* tokens the prefill build indexed     */
  int32_t capacity;         /* most tokens the layout has room for  */
} ri_index_config;

typedef struct {
  int32_t middle;       /* M                                         */
  int32_t num_segments; /* S = ceil(M / seg_len)                     */
  int32_t clusters;     /* C = sum of K_s over segments (growing: the
                           live clusters, open segment included)     */
  int32_t steady;       /* min(N, steady_initial + steady_recent)    */
  int32_t cluster_stride; /* clusters per unit in the index arrays (C
                             when compact)                           */
  int32_t row_stride;     /* Kp / Vp / perm rows per unit (M when
                             compact)                                */
} ri_geometry;

/* Derived sizes of a configuration.  Host only; validates the config. */
ri_status ri_index_geometry(const ri_index_config* cfg, ri_geometry* out);

/* The index of every (sequence, KV head).  All device memory, caller-owned,
 * written by ri_build_index and read by the decode calls.
 *  Kp, Vp    bf16 [B][H_kv][M][d]  cluster-contiguous copy of the middle
 *            tokens [P2 §3.1]: clusters in global id order, members of a
 *            cluster in position order.
 *  perm      int32 [B][H_kv][M]    absolute token position of each row.
 *  centroid  bf16 [B][H_kv][C][d]  round-to-nearest-even of the fp32 mean of
 *            the cluster's keys (an empty cluster keeps its last centroid).
 *  counts    int32 [B][H_kv][C]    cluster sizes n_c.
 *  offsets   int32 [B][H_kv][C+1]  row of each cluster's first member in
 *            Kp/Vp; offsets[C] = M.
 *  vsum      fp32 [B][H_kv][C][d]  sum of the members' values
 *            [P2 §2.1 `compute_cluster_sums`].
 *  Ks, Vs    bf16 [B][H_kv][steady][d]  steady-zone tokens in position order.
 *  labels    optional (may be NULL) int32 [B][H_kv][M]: cluster id within
 *            its segment of every middle token, in position order.
 *  objective optional (may be NULL) fp32 [B][H_kv][S]: per segment, the sum
 *            of squared distances of keys to their final centroid.          */
typedef struct {
  void* Kp;
  void* Vp;
  int32_t* perm;
  void* centroid;
  int32_t* counts;
  int32_t* offsets;
  float* vsum;
  void* Ks;
  void* Vs;
  int32_t* labels;
  float* objective;
} ri_index;

/* Bytes of workspace ri_build_index needs (0 on invalid config). */
size_t ri_build_index_workspace(const ri_index_config* cfg);

/* Segmented k-means index build [P2 §2.1 pseudocode; P3 abstract].
 * K, V      bf16 [B][H_kv][N][d] device, the keys and values.
 * init_pos  optional device int32 [B][H_kv][C]: for the clusters of segment
 *           s, distinct positions in [0, L_s) of the tokens whose keys seed
 *           the centroids; NULL selects positions floor(j * L_s / K_s).
 *           Out-of-range entries are clamped and flagged RI_ERR_INVALID_ARG
 *           in the device status word.
 * Lloyd's algorithm with squared Euclidean distance, ties to the lower
 * cluster id, a fixed number of iterations; labels and centroids returned are
 * those of the last iteration, so every non-empty centroid is the mean of its
 * final members.  Assignment runs on the tensor cores (tcgen05) with a
 * rigorous error bound; near ties are re-decided in fp32.
 * Returns before the work completes; errors in arguments return early. */
ri_status ri_build_index(const ri_index_config* cfg, const void* K, const void* V,
                         const int32_t* init_pos, const ri_index* out, void* workspace,
                         size_t workspace_bytes, ri_stream_t stream);

/* ---- Index maintenance during decode ---------------------------------
 * [P2 §2.1 item 1: the steady zone holds the first 4 and the most recent 64
 * tokens, so each decode step moves one token out of the recent window;
 * P2 §2.1 pseudocode: k-means per 8K-token segment.  The pages give no
 * mechanism; this is the reading the library implements.]
 * A growing index is described by a config with base_len (tokens of the
 * prefill build) < capacity; seq_len is the current length.  Every step
 * appends token seq_len: the token at seq_len - steady_recent leaves the
 * recent window and joins the *open segment* in the open cluster of its
 * nearest centroid (squared Euclidean distance to the stored bf16
 * centroids, ties to the lower id) among the K_last clusters of the last
 * closed segment that still have a free slot (ceil(2 seg_len / K_last)
 * slots per open cluster); that cluster's size and value sum grow by the
 * token, and it is scored with the same centroid.  When the open segment
 * holds seg_len tokens, k-means over them (position order, seeds
 * floor(j L / K), `iters` iterations) makes it a closed segment and a new
 * empty open segment of K = min(clusters_per_seg, seg_len) clusters follows.
 * Layout per unit (ri_index_geometry gives the strides): clusters
 * [cluster_stride], ids: the prefill's segments, the closed appended
 * segments, then the K open clusters (live clusters C = those); rows
 * [row_stride]: closed segments cluster-contiguous from row 0, the open
 * clusters' slots after every closed row the capacity allows, members in
 * arrival order; offsets[c] is cluster c's first row (counts[c] rows
 * follow), offsets[cluster_stride] = row_stride.  Ks / Vs keep the first
 * steady_initial tokens and the recent window as a ring (position p at
 * slot steady_initial + ((p - base_len) mod steady_recent)).  The decode
 * calls take the growing config with the current seq_len; labels and
 * objective are not kept. */

/* Copies a compact index built by ri_build_index (its config: cfg with
 * base_len = capacity = 0 and seq_len = cfg->base_len) into the layout of
 * the growing config cfg (seq_len == base_len < capacity) and sets up the
 * first open segment.  `out` arrays sized by cfg's strides. */
ri_status ri_index_open(const ri_index_config* cfg, const ri_index* compact, const ri_index* out,
                        ri_stream_t stream);

/* Bytes of workspace ri_index_append needs (0 unless cfg is growing). */
size_t ri_index_append_workspace(const ri_index_config* cfg);

/* One step of index maintenance for token cfg->seq_len of every (sequence,
 * KV head): k_new, v_new bf16 [B][H_kv][d] (its key and value) enter the
 * recent window, the leaving token joins the open segment, and the open
 * segment is closed by k-means when it becomes full.  Call before the
 * step's decode (whose config then has seq_len + 1).  assigned: optional
 * int32 [B][H_kv], the open cluster (0..K_last-1) each leaving token joined.
 * RI_ERR_CAPACITY when seq_len == capacity.  Device-side failures go to
 * the workspace status word (sticky, like the decode calls'). */
ri_status ri_index_append(const ri_index_config* cfg, const void* k_new, const void* v_new,
                          const ri_index* idx, int32_t* assigned, void* workspace,
                          size_t workspace_bytes, ri_stream_t stream);

/* Zone budgets in clusters: k_retrieval = round(0.018 C), k_estimation =
 * round(0.23 C) by default [P2 §2.1 items 2-3].  The zones are clamped to
 * C: R = top min(k_r, C), E = next min(k_e, C - |R|).  k_retrieval <= 4096. */
typedef struct {
  int32_t k_retrieval;
  int32_t k_estimation;
} ri_decode_config;

/* Default budgets for C clusters (round half up of 1.8 % and 23 %). */
ri_status ri_default_budgets(int32_t clusters, ri_decode_config* out);

/* Bytes of workspace the decode calls need (0 on invalid or unsupported
 * config).  The same workspace serves every decode call of the
 * configuration; it holds the status region, the per-head centroid scores of
 * the last scoring pass and the selection handed from ri_select_clusters to
 * ri_attend_selected. */
size_t ri_decode_workspace(const ri_index_config* cfg, const ri_decode_config* dcfg);

/* One decode step of tripartite attention [P3 abstract; P2 §2.1, §3.3]:
 *  - scores s[h][c] = q_h . centroid_c / sqrt(d) for every query head of a KV
 *    head; selection key r_c = sum over the G heads (r_c = -inf if n_c = 0);
 *  - R = the k_r clusters of largest r (ties to the lower id), E = the next
 *    k_e;
 *  - out_h = (sum_{i in steady u R} e^{x_i} v_i + sum_{c in E} e^{s_hc} Vsum_c)
 *          / (sum_{i in steady u R} e^{x_i} + sum_{c in E} n_c e^{s_hc}),
 *    x_i = q_h . k_i / sqrt(d); partial results merged by log-sum-exp.
 * q        bf16 [B][H_kv*G][d].
 * out      bf16 [B][H_kv*G][d].
 * lse      optional fp32 [B][H_kv*G]: natural log of the denominator.
 * sel_ids  optional int32 [B][H_kv][k_r + k_e]: R then E, each in increasing
 *          id order (entries past the clamped sizes are -1).
 * Reads Kp/Vp in place through `offsets`.  One thread-block cluster works on
 * each (sequence, KV head); C (clusters per sequence and KV head) must be at
 * most 65536, else RI_ERR_UNSUPPORTED.  A retrieval cluster whose rows fall
 * outside Kp, or a negative size, is not attended and RI_ERR_INVALID_ARG is
 * recorded in the status word. */
ri_status ri_decode_attention(const ri_index_config* cfg, const ri_decode_config* dcfg,
                              const void* q, const ri_index* idx, void* out, float* lse,
                              int32_t* sel_ids, void* workspace, size_t workspace_bytes,
                              ri_stream_t stream);

/* One decode step with the query and the output in host memory: copies
 * q_host (bf16 [B][H_kv*G][d]) to q_dev, runs ri_decode_attention on `stream`
 * (out_dev, lse, workspace as there; no selection output), copies out_dev to
 * out_host and waits for the stream, so out_host holds the step's output on
 * return.  q_dev and out_dev are device buffers of the same shape owned by
 * the caller (16-byte aligned); page-locked host buffers make the two copies
 * asynchronous with respect to other host work.  Errors: as
 * ri_decode_attention, plus RI_ERR_INVALID_ARG for a NULL host pointer and
 * RI_ERR_CUDA when a copy or the synchronisation fails (then out_host is not
 * valid).  The pages describe the decode step, not this convenience; it is
 * the call an application without device tensors of its own makes. */
ri_status ri_decode_attention_host(const ri_index_config* cfg, const ri_decode_config* dcfg,
                                   const void* q_host, void* q_dev, const ri_index* idx,
                                   void* out_dev, void* out_host, float* lse, void* workspace,
                                   size_t workspace_bytes, ri_stream_t stream);

/* ri_decode_attention without a caller workspace.  The pages describe no
 * such call; it exists for callers that must not allocate (or own) scratch:
 * the scratch is a fixed device array of RI_STATIC_SCRATCH_BYTES inside this
 * library, one per device.  Same arguments, results and checks as
 * ri_decode_attention, minus workspace/workspace_bytes, plus:
 *  - device_status: optional device int32.  When non-NULL the call's device
 *    status word (RI_OK, or the first device-side failure) is copied there,
 *    ordered on `stream` after the kernel.
 * Limits and rules:
 *  - Returns RI_ERR_CAPACITY when ri_decode_workspace() for (cfg, dcfg)
 *    exceeds RI_STATIC_SCRATCH_BYTES (4 MiB: e.g. one 128K-token sequence
 *    with 8 KV heads fits; batch 16 of 128K does not).
 *  - The array used is the current device's; the current device must hold
 *    `stream`, q, out and the index.
 *  - The first call on a device (and group size) looks up the array's
 *    address, sets the kernel's attributes and queries how many thread-block
 *    clusters the device holds (and loads the module if it is loaded
 *    lazily); make one call, or any call that can fail fast, before
 *    capturing a stream into a CUDA graph.  Those results are kept in fixed
 *    tables inside the library: no call allocates device or host memory.
 *  - Every call on a device shares the one array: calls whose executions
 *    overlap (on different streams or from different threads) race and
 *    give wrong results.  Order them on one stream.
 *  - Each call clears the status word (stream-ordered) before its kernel
 *    runs; nothing else in the array has to start at zero. */
#define RI_STATIC_SCRATCH_BYTES ((size_t)4 << 20)
ri_status ri_decode_attention_static(const ri_index_config* cfg, const ri_decode_config* dcfg,
                                     const void* q, const ri_index* idx, void* out, float* lse,
                                     int32_t* sel_ids, int32_t* device_status,
                                     ri_stream_t stream);

/* Steps S1-S2 alone (centroid scoring and cluster selection).  Writes
 * sel_ids (required here) and keeps scores and the selection in the
 * workspace for a following ri_attend_selected on the same workspace and
 * stream.  Also writes, when non-NULL, retr_rows int32 [B][H_kv][k_r + 1]:
 * the exclusive prefix sum of the sizes of the R clusters in id order (the
 * execution-buffer row of each retrieval cluster; last entry = total). */
ri_status ri_select_clusters(const ri_index_config* cfg, const ri_decode_config* dcfg,
                             const void* q, const ri_index* idx, int32_t* sel_ids,
                             int32_t* retr_rows, void* workspace, size_t workspace_bytes,
                             ri_stream_t stream);

/* Steps S4-S6 on the selection left in `workspace` by ri_select_clusters.
 * exec_K, exec_V: NULL to read the retrieval tokens in place from idx->Kp,
 * idx->Vp; otherwise bf16 [B][H_kv][exec_rows][d] execution buffers holding,
 * for every (sequence, head), the R clusters' rows packed in id order from
 * row 0 [P1 三: the execution buffer feeds attention]. */
ri_status ri_attend_selected(const ri_index_config* cfg, const ri_decode_config* dcfg,
                             const void* q, const ri_index* idx, const void* exec_K,
                             const void* exec_V, int32_t exec_rows, void* out, float* lse,
                             void* workspace, size_t workspace_bytes, ri_stream_t stream);

/* ---- Wave buffer: GPU block cache and execution-buffer gather ----------
 * [P2 §2.2 wave buffer (mapping table, LRU replacement, synchronous access
 * path); §3.1 cache layout (fixed 2 KB physical blocks: 8 rows x 128 bf16);
 * §3.2 execution buffer assembly; P4 §2B].  With the full K/V of a layer in
 * pinned host memory, each decode step (1) selects clusters on the device
 * (ri_select_clusters), (2) plans on the host which retrieval clusters are
 * served by the GPU block cache and which come over the host link
 * (ri_cache_plan), (3) gathers them into the execution buffer and admits the
 * misses into the cache (ri_gather_blocks, twice: fetch list, then admit
 * list), and (4) attends over the execution buffer (ri_attend_selected). */

/* One copy of n_rows consecutive K rows and the same V rows of one unit
 * (unit = b * H_kv + h).  Rows are relative to the unit's block of the
 * source / destination buffer (see ri_gather_buffers). */
typedef struct {
  int32_t unit;
  int32_t src_kind; /* RI_SRC_HOST, RI_SRC_CACHE or RI_SRC_EXEC */
  int32_t src_row;
  int32_t dst_kind; /* RI_DST_EXEC or RI_DST_CACHE */
  int32_t dst_row;
  int32_t n_rows;
} ri_copy_desc;
enum { RI_SRC_HOST = 0, RI_SRC_CACHE = 1, RI_SRC_EXEC = 2 };
enum { RI_DST_EXEC = 0, RI_DST_CACHE = 1 };

/* Cache geometry.  Each unit owns a pool of blocks_per_unit blocks of
 * block_rows rows; a cluster of n rows occupies ceil(n / block_rows) blocks.
 * Limits: units >= 1, blocks_per_unit >= 1, 1 <= block_rows <= 1024. */
typedef struct {
  int32_t units;
  int32_t blocks_per_unit;
  int32_t block_rows; /* 8 in the pages' layout */
} ri_cache_config;

/* Opaque host-side state: per unit the mapping table cluster -> blocks, the
 * LRU order of clusters and the free blocks.  Created empty; host memory
 * only (the device pool is caller-owned, see ri_gather_buffers). */
typedef struct ri_cache ri_cache;

/* Per-call counts from ri_cache_plan (summed over units).  Requested
 * clusters of zero rows are counted in empty_clusters only. */
typedef struct {
  int64_t hit_clusters, miss_clusters, uncached_clusters; /* uncached: served, not admitted */
  int64_t hit_rows, miss_rows;                            /* rows from the cache / the host */
  int64_t empty_clusters;                                 /* requested clusters of 0 rows  */
} ri_cache_stats;

ri_status ri_cache_create(const ri_cache_config* cfg, ri_cache** out);
/* Frees the host state.  A worker attached to the cache must be destroyed
 * first. */
void ri_cache_destroy(ri_cache* cache);

/* One step of the synchronous access path, on the host.  For every unit u:
 * the retrieval clusters are sel_ids[u * sel_stride + i], i < k_retrieval,
 * up to the first negative entry (id order, as ri_select_clusters writes
 * them); counts / offsets are the index's [units][C] / [units][C + 1] arrays
 * copied to the host.  The execution-buffer rows follow the clusters in this
 * order from row 0 (ri_select_clusters' retr_rows).  Lookup first (hit:
 * resident; a cluster of 0 rows is a hit and is not cached), then the misses
 * are admitted in order, evicting least recently used clusters not requested
 * in this step until the miss fits (a miss that cannot fit even after every
 * such eviction is served uncached and evicts nothing), and every
 * requested resident cluster becomes most recent in request order.  Writes
 * the copy plan: `fetch` (cache->exec for hits, host->exec for misses) and
 * `admit` (exec->cache for admitted misses), each split into copies of at
 * most 16 rows (a cluster's blocks that are adjacent in the pool share one
 * copy); *n_fetch / *n_admit get their lengths.  Fails with
 * RI_ERR_CAPACITY (state unchanged) when a list would exceed its capacity,
 * RI_ERR_INVALID_ARG for bad pointers, ids or sizes, or when a worker is
 * attached to the cache.  Not thread-safe for one cache. */
ri_status ri_cache_plan(ri_cache* cache, const int32_t* sel_ids, int32_t sel_stride,
                        int32_t k_retrieval, const int32_t* counts, const int32_t* offsets,
                        int32_t clusters, ri_copy_desc* fetch, int32_t fetch_cap,
                        int32_t* n_fetch, ri_copy_desc* admit, int32_t admit_cap,
                        int32_t* n_admit, ri_cache_stats* stats);

/* The blocks holding cluster `cluster` of unit `unit`, in row order, written
 * to blocks[0 .. cap); *n_blocks = their number (0: not resident).  Host
 * state only; RI_ERR_CAPACITY when cap is too small (*n_blocks still set).
 * Not to be called while a worker's update may be running. */
ri_status ri_cache_resident(const ri_cache* cache, int32_t unit, int32_t cluster,
                            int32_t* blocks, int32_t cap, int32_t* n_blocks);

/* Checks the invariants of the host state: per unit every block is free or
 * held by exactly one resident cluster, block chains have their recorded
 * lengths, and the LRU list holds exactly the resident clusters.  RI_OK or
 * RI_ERR_INVALID_ARG with ri_last_error() naming the first violation. */
ri_status ri_cache_validate(const ri_cache* cache);

/* Rows of the execution buffer one step can need, per unit: the sum of the
 * k_retrieval largest cluster sizes (the retrieval zone is the k_retrieval
 * top-scoring clusters, "KV缓存技术与RetroInfer系统在长上下文推理中的优化实践"
 * (framerc.cn) §2.2 execution buffer / §2.1 retrieval zone).  Host planning
 * for the buffer's allocation, made once per index and budget:
 *   counts  int32 [units][clusters], host memory (the index's sizes copied
 *           back); every entry >= 0
 *   out     int32 [units], host memory, written on success
 * k_retrieval >= clusters sums every size; 0 gives 0.  RI_ERR_INVALID_ARG for
 * NULL pointers, units < 1, clusters < 1, k_retrieval < 0 or a negative size
 * (out untouched); RI_ERR_CAPACITY when a sum exceeds INT32_MAX. */
ri_status ri_max_retrieval_rows(const int32_t* counts, int32_t units, int32_t clusters,
                                int32_t k_retrieval, int32_t* out);

/* Buffers of the gather: bf16 [units][rows][128] each, dense.
 *  host_K, host_V   the index's Kp, Vp in pinned (page-locked) host memory,
 *                   rows = M; read by the device through unified addressing.
 *  cache_K, cache_V device pool, rows = pool_rows (= blocks_per_unit *
 *                   block_rows); may be NULL when no descriptor uses them.
 *  exec_K, exec_V   device execution buffers, rows = exec_rows. */
typedef struct {
  const void* host_K;
  const void* host_V;
  void* cache_K;
  void* cache_V;
  void* exec_K;
  void* exec_V;
  int32_t units;
  int32_t M;
  int32_t pool_rows;
  int32_t exec_rows;
} ri_gather_buffers;

/* Executes n_desc copies (desc: device array) with 16-byte vector loads and
 * stores, one warp per copy.  Copies of one call must not overlap in their
 * destinations or write what another reads (ri_cache_plan's fetch and admit
 * lists satisfy this when run as two calls, fetch first).  A copy whose rows
 * fall outside its buffers is skipped and RI_ERR_INVALID_ARG recorded in
 * the status word of `workspace` (>= 256 device bytes; cleared by the call). */
ri_status ri_gather_blocks(const ri_gather_buffers* bufs, const ri_copy_desc* desc,
                           int32_t n_desc, void* workspace, ri_stream_t stream);

/* ---- Asynchronous cache update [P2 §2.2 异步更新路径: a background thread
 * runs the LRU replacement and updates the mapping table late, so the
 * update's cost hides behind GPU work; P4 §2B; P1 三] ------------------------
 * A worker attached to an ri_cache splits each ri_cache_plan step in two:
 *  (1) ri_cache_lookup, on the caller's critical path: waits until the
 *      previous step's update has been applied (host), makes `stream` wait
 *      for that update's admit copies (device), then reads the mapping table
 *      without changing it and writes the step's fetch list (cache->exec for
 *      resident clusters, host->exec for the others: the same list
 *      ri_cache_plan writes) and the step's lookup counts;
 *  (2) ri_cache_update_async, after the caller has issued the fetch copies
 *      on `stream`: records an event on `stream` and hands the update to the
 *      worker thread, which applies ri_cache_plan's replacement rule to the
 *      state, writes the admit list and, when admit_dev is given, copies the
 *      list to the device and runs the admit copies (ri_gather_blocks'
 *      kernel) on side_stream after the event.
 * Every step therefore sees the state and gets the fetch list ri_cache_plan
 * would have given it, so the execution buffer, and the attention over it,
 * are identical to the synchronous path's.
 * Failures of an update (injected, or a CUDA error issuing its copies) are
 * reported once, by the next ri_cache_lookup (which then does nothing and
 * may be called again) or ri_cache_worker_wait.  A failed update leaves a
 * consistent state: the clusters it admitted before failing keep their admit
 * copies; the step's other misses are not admitted and later units keep
 * their previous state (a CUDA error takes the update's admissions back). */
typedef struct ri_cache_worker ri_cache_worker;

typedef struct {
  ri_gather_buffers bufs;   /* as for ri_gather_blocks; units and pool_rows
                               must match the cache; ignored without admit_dev */
  ri_copy_desc* admit_dev;  /* device array of admit_cap descriptors, or NULL:
                               host-only worker (no device work; the admit
                               lists are left for the caller)              */
  ri_copy_desc* admit_host; /* host array of admit_cap descriptors (pinned when
                               admit_dev is given; NULL: worker-owned) */
  int32_t admit_cap;        /* bounds one step's admit copies (RI_ERR_CAPACITY
                               from the lookup when a step could exceed it) */
  void* gather_workspace;   /* >= 256 device bytes: status word of the admit
                               copies (sticky; read with ri_read_device_status) */
  ri_stream_t side_stream;  /* stream of the admit copies (best: non-blocking) */
  int32_t device;           /* CUDA device of the buffers and streams        */
  uint64_t wait_limit_ns;   /* limit of every wait on the worker (0 = 10 s)  */
  int32_t lookup_threads;   /* threads of the lookup, units split among them
                               [P2 §2.2 同步访问路径: multi-threaded lookup of
                               the mapping table]; 0 = min(8, cores / 2), never
                               more than the units                          */
} ri_cache_worker_config;

/* Starts the worker thread of `cache` (one worker per cache; ri_cache_plan is
 * refused while it is attached).  Creates two CUDA events on `device` when
 * admit_dev is given. */
ri_status ri_cache_worker_create(ri_cache* cache, const ri_cache_worker_config* cfg,
                                 ri_cache_worker** out);
/* Applies every handed-over update, waits (bounded) for their admit copies,
 * stops the thread and frees the worker; returns a failure not yet
 * reported. */
ri_status ri_cache_worker_destroy(ri_cache_worker* worker);

/* Step part (1); arguments as ri_cache_plan's, minus the admit list.  The
 * stats carry the lookup counts (hits, misses, rows, empty clusters;
 * uncached_clusters is 0: the update decides it).  RI_ERR_TIMEOUT when the
 * previous update was not applied within the limit (nothing done);
 * RI_ERR_CAPACITY when the fetch list, or the admit list of every miss,
 * could exceed its capacity (state unchanged, nothing handed over). */
ri_status ri_cache_lookup(ri_cache_worker* worker, const int32_t* sel_ids, int32_t sel_stride,
                          int32_t k_retrieval, const int32_t* counts, const int32_t* offsets,
                          int32_t clusters, ri_copy_desc* fetch, int32_t fetch_cap,
                          int32_t* n_fetch, ri_cache_stats* stats, ri_stream_t stream);

/* Step part (2): hands the last lookup's update to the worker.  Call after
 * the fetch copies were issued on `stream`; RI_ERR_INVALID_ARG without a
 * lookup to apply. */
ri_status ri_cache_update_async(ri_cache_worker* worker, ri_stream_t stream);

/* Waits (bounded) until every handed-over update has been applied; returns
 * the update counts of the last one (uncached_clusters) and its number of
 * admit copies, whose list is then in admit_host (or the worker's own list)
 * until the next update starts.  Returns a failure not yet reported. */
ri_status ri_cache_worker_wait(ri_cache_worker* worker, ri_cache_stats* stats, int32_t* n_admit);

/* Test hooks of the update path: update number fail_update (0 = the first
 * handed to this worker; -1 = none) stops after fail_after_admissions
 * admissions with RI_ERR_HOST; every update first sleeps delay_us
 * microseconds. */
ri_status ri_cache_worker_test_hooks(ri_cache_worker* worker, int64_t fail_update,
                                     int64_t fail_after_admissions, uint32_t delay_us);

/* ri_gather_blocks with the launch shape given: threads per block (0, or a
 * multiple of 32 in [32, 512]; one warp per copy) and the most blocks per SM
 * the grid may hold (0..64; 0 = default).  [P2 §3.2: the copy kernel adapts
 * its thread-block size to the cache-hit pattern.] */
ri_status ri_gather_blocks_shaped(const ri_gather_buffers* bufs, const ri_copy_desc* desc,
                                  int32_t n_desc, int32_t threads, int32_t blocks_per_sm,
                                  void* workspace, ri_stream_t stream);

/* The launch shape for a copy list of total_copies copies of which
 * host_copies read pinned host memory (cache misses): lists with host
 * copies get the most warps in flight, device-only lists fewer, larger
 * blocks (the shapes measured best for each on B200).  Host only. */
ri_status ri_gather_shape(int64_t host_copies, int64_t total_copies, int32_t* threads,
                          int32_t* blocks_per_sm);

/* Synchronises `stream` and returns the status word previous calls wrote
 * into `workspace` (RI_OK if no device-side failure was recorded); a failure
 * read is cleared, so the next read reports only later failures. */
ri_status ri_read_device_status(void* workspace, ri_stream_t stream);

/* Self-test of the bounded device wait: launches one kernel that waits for a
 * flag in `workspace` that nothing sets, giving up after `limit_ns`
 * nanoseconds and recording RI_ERR_TIMEOUT in the status word.  workspace
 * needs 256 bytes. */
ri_status ri_selftest_wait_timeout(void* workspace, uint64_t limit_ns, ri_stream_t stream);

/* Self-test of the decode kernel's own bounded waits: one ri_decode_attention
 * step (same arguments, lse and sel_ids not written) with one hand-off inside
 * the kernel left unreleased and every wait limited to limit_ns nanoseconds
 * (at most 10 s):
 *   hand_off 1: the first centroid tile's copy is never issued (the MMA
 *               issuer's wait expires);
 *   hand_off 2: the first tile's MMA completion is never signalled (the
 *               scoring epilogue's wait expires);
 *   hand_off 3: the cluster sizes loaded beside the scoring are never
 *               signalled ready (the scoring epilogue's wait expires).
 * The kernel records RI_ERR_TIMEOUT in the status word, every block returns
 * after the copies it issued have landed, and the device stays usable; `out`
 * holds no meaningful result. */
ri_status ri_selftest_decode_timeout(const ri_index_config* cfg, const ri_decode_config* dcfg,
                                     const void* q, const ri_index* idx, void* out,
                                     void* workspace, size_t workspace_bytes, int32_t hand_off,
                                     uint64_t limit_ns, ri_stream_t stream);

const char* ri_status_string(ri_status status);
/* Description of the last error of the calling thread ("" if none). */
const char* ri_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* RETROINFER_H_ */
