// Host side of the wave buffer's GPU block cache (RetroInfer,
// "KV缓存技术与RetroInfer系统在长上下文推理中的优化实践" (framerc.cn) §2.2 wave
// buffer: mapping table + LRU replacement, the synchronous access path and
// the asynchronous update path; §3.1: fixed physical blocks of 8 rows x 128
// bf16).  Per unit: a mapping table cluster -> chain of blocks, the LRU order
// of resident clusters and a stack of free blocks, all as flat arrays indexed
// by cluster id or block id (one step touches each requested cluster in O(1)
// plus its blocks).
//
// A step is split in two parts that both entry points share:
//  - lookup (read-only on the state): the fetch copies of every requested
//    retrieval cluster (cache->exec when resident, host->exec otherwise) and
//    one request record per cluster;
//  - update (the LRU replacement): admission of the misses, evicting least
//    recently used clusters that the step does not request, the admit copies
//    (exec->cache) and the new recency order.
// ri_cache_plan runs both in the caller's thread.  A cache worker runs the
// update on its own thread and issues the admit copies on its own stream
// (ri_cache_lookup / ri_cache_update_async), so the step waits only for the
// lookup.
#include <algorithm>
#include <chrono>
#include <condition_variable>
#include <cstdio>
#include <cstring>
#include <functional>
#include <mutex>
#include <new>
#include <thread>
#include <vector>

#include "internal.h"

namespace {

constexpr int kChunkRows = 16;  // rows per copy descriptor

struct Cluster {            // per cluster id
  int32_t head = -1;       // first block of the cluster's chain, -1 if not resident
  int32_t nblk = 0;        // blocks in the chain
  int32_t prev = -1;       // LRU links (-1 at the ends)
  int32_t next = -1;
  int32_t in_lru = 0;
};

struct Unit {
  std::vector<Cluster> cl;        // grown to the largest cluster count seen
  std::vector<int32_t> link;      // per block: next block of the same cluster, -1 at the end
  std::vector<int32_t> free;      // stack: the next block is free.back()
  int32_t lru_head = -1, lru_tail = -1;  // least / most recently used
  long long lru_blocks = 0;       // blocks held by the clusters in the LRU list

  void grow(int32_t clusters) {
    if ((int32_t)cl.size() < clusters) cl.resize(clusters);
  }
  void unlink(int32_t c) {
    Cluster& x = cl[c];
    if (x.prev >= 0) cl[x.prev].next = x.next; else lru_head = x.next;
    if (x.next >= 0) cl[x.next].prev = x.prev; else lru_tail = x.prev;
    x.prev = x.next = -1;
    x.in_lru = 0;
    lru_blocks -= x.nblk;
  }
  void push_back(int32_t c) {
    Cluster& x = cl[c];
    x.prev = lru_tail;
    x.next = -1;
    if (lru_tail >= 0) cl[lru_tail].next = c; else lru_head = c;
    lru_tail = c;
    x.in_lru = 1;
    lru_blocks += x.nblk;
  }
  // Frees the blocks of resident cluster c (already out of the LRU list).
  void release(int32_t c) {
    Cluster& y = cl[c];
    for (int b = y.head; b >= 0;) {
      const int nb = link[b];
      link[b] = -1;
      free.push_back(b);
      b = nb;
    }
    y.head = -1;
    y.nblk = 0;
  }
};

// One requested retrieval cluster of a step (clusters of zero rows are not
// recorded: they hold nothing to fetch or cache).
struct Req {
  int32_t c;     // cluster id
  int32_t n;     // rows
  int32_t erow;  // first execution-buffer row
  int32_t hit;   // resident at lookup
};

}  // namespace

struct ri_cache {
  ri_cache_config cfg;
  std::vector<Unit> units;
  std::vector<Req> req;            // the last lookup's requests, unit after unit
  std::vector<int32_t> req_start;  // [units + 1]: first request of each unit
  bool has_worker = false;         // lookups and updates go through the worker
};

namespace {

// Writes the copies of `rows` rows (src..., dst...) split into chunks.
inline void emit(ri_copy_desc* out, int32_t* n, int unit, int src_kind, int src_row,
                 int dst_kind, int dst_row, int rows) {
  for (int r = 0; r < rows; r += kChunkRows) {
    ri_copy_desc& d = out[(*n)++];
    d.unit = unit;
    d.src_kind = src_kind;
    d.src_row = src_row + r;
    d.dst_kind = dst_kind;
    d.dst_row = dst_row + r;
    d.n_rows = rows - r < kChunkRows ? rows - r : kChunkRows;
  }
}

// Copies of block-sized pieces, merged while both sides stay contiguous and
// the copy stays within kChunkRows rows.
struct Runs {
  ri_copy_desc* out;
  int32_t* n;
  int unit, src_kind, dst_kind;
  int src = 0, dst = 0, rows = 0;
  void add(int s, int d, int r) {
    if (rows > 0 && s == src + rows && d == dst + rows && rows + r <= kChunkRows) {
      rows += r;
      return;
    }
    flush();
    src = s;
    dst = d;
    rows = r;
  }
  void flush() {
    if (rows > 0) emit(out, n, unit, src_kind, src, dst_kind, dst, rows);
    rows = 0;
  }
};

inline long long chunks(long long rows) { return (rows + kChunkRows - 1) / kChunkRows; }

// Copies of a cluster of n rows split at block boundaries (upper bound of
// its block copies; adjacent blocks may merge into fewer).
inline long long block_chunks(long long n, int br) {
  long long t = 0;
  for (long long k = 0; k * br < n; ++k) t += chunks(n - k * br < br ? n - k * br : br);
  return t;
}

// How far ahead the per-cluster loops prefetch their table entries: the
// requested ids are sparse in tables of tens of thousands of clusters, so
// nearly every entry is a cache miss.
constexpr int kAhead = 16;

inline void prefetch_ids(const Unit& U, const int32_t* sel, int i, int k_retrieval,
                         const int32_t* cnt, const int32_t* off) {
  if (i < k_retrieval) {
    const int c = sel[i];
    if (c >= 0 && c < (int)U.cl.size()) {
      __builtin_prefetch(cnt + c);
      __builtin_prefetch(off + c);
      __builtin_prefetch(&U.cl[(size_t)c]);
    }
  }
}

// Per-unit sizes of one step (from the read-only pass).
struct UnitCount {
  long long nf = 0, na = 0, nreq = 0;
};

// Read-only pass over one unit's request: every requested id and size
// checked (ids ascending, below `clusters`, sizes and rows >= 0), the exact
// number of fetch copies and the number of admit copies if every miss were
// admitted counted.
ri_status validate_unit(const Unit& U, int u, const int32_t* sel, int32_t k_retrieval,
                        const int32_t* cnt, const int32_t* off, int32_t clusters, int br,
                        UnitCount* out) {
  UnitCount uc;
  int prev = -1;
  for (int i = 0; i < kAhead; ++i) prefetch_ids(U, sel, i, k_retrieval, cnt, off);
  for (int i = 0; i < k_retrieval; ++i) {
    const int c = sel[i];
    if (c < 0) break;
    prefetch_ids(U, sel, i + kAhead, k_retrieval, cnt, off);
    if (c >= clusters || c <= prev) {
      ri::set_error("cache: unit %d entry %d: cluster id %d out of range or not ascending", u, i,
                    c);
      return RI_ERR_INVALID_ARG;
    }
    prev = c;
    const int n = cnt[c];
    if (n < 0 || off[c] < 0) {
      ri::set_error("cache: unit %d cluster %d: negative size or row", u, c);
      return RI_ERR_INVALID_ARG;
    }
    if (n == 0) continue;
    ++uc.nreq;
    if (U.cl[(size_t)c].head >= 0) {
      uc.nf += block_chunks(n, br);
    } else {
      uc.nf += chunks(n);
      uc.na += block_chunks(n, br);
    }
  }
  *out = uc;
  return RI_OK;
}

// Lookup of one unit's requested clusters on the mapping table (no state
// change): fetch copies from `fetch` on and request records from `req` on.
// Returns the number of fetch copies written.
int32_t lookup_unit(const Unit& U, int u, const int32_t* sel, int k_retrieval, const int32_t* cnt,
                    const int32_t* off, int br, ri_copy_desc* fetch, Req* req,
                    ri_cache_stats& st) {
  int32_t nfo = 0;
  int run = 0;  // execution-buffer row of the next cluster
  for (int i = 0; i < kAhead; ++i) prefetch_ids(U, sel, i, k_retrieval, cnt, off);
  for (int i = 0; i < k_retrieval && sel[i] >= 0; ++i) {
    prefetch_ids(U, sel, i + kAhead, k_retrieval, cnt, off);
    const int c = sel[i], n = cnt[c];
    const int erow = run;
    run += n;
    if (n == 0) {
      ++st.empty_clusters;
      continue;
    }
    const Cluster& x = U.cl[(size_t)c];
    const bool hit = x.head >= 0;
    *req++ = Req{c, n, erow, hit ? 1 : 0};
    if (hit) {
      ++st.hit_clusters;
      st.hit_rows += n;
      Runs runs{fetch, &nfo, u, RI_SRC_CACHE, RI_DST_EXEC};
      int k = 0;
      for (int b = x.head; b >= 0; b = U.link[(size_t)b], ++k) {
        const int rows = n - k * br < br ? n - k * br : br;
        runs.add(b * br, erow + k * br, rows);
      }
      runs.flush();
    } else {
      ++st.miss_clusters;
      st.miss_rows += n;
      emit(fetch, &nfo, u, RI_SRC_HOST, off[c], RI_DST_EXEC, erow, n);
    }
  }
  return nfo;
}

// A fixed set of helper threads that run the per-unit tasks of a step
// together with the calling thread.
class Pool {
 public:
  explicit Pool(int helpers) {
    for (int i = 0; i < helpers; ++i) th_.emplace_back([this] { loop(); });
  }
  ~Pool() {
    {
      std::lock_guard<std::mutex> lk(m_);
      stop_ = true;
    }
    cv_.notify_all();
    for (std::thread& t : th_) t.join();
  }
  // Runs f(i) for i in [0, n) on the helpers and the caller; returns when
  // every task has finished.
  void run(int n, const std::function<void(int)>& f) {
    if (th_.empty() || n <= 1) {
      for (int i = 0; i < n; ++i) f(i);
      return;
    }
    {
      std::lock_guard<std::mutex> lk(m_);
      job_ = &f;
      n_ = n;
      next_ = 0;
      busy_ = (int)th_.size();
      ++gen_;
    }
    cv_.notify_all();
    work();
    std::unique_lock<std::mutex> lk(m_);
    done_.wait(lk, [this] { return busy_ == 0; });
    job_ = nullptr;
  }

 private:
  void work() {
    for (;;) {
      int i;
      {
        std::lock_guard<std::mutex> lk(m_);
        if (next_ >= n_) return;
        i = next_++;
      }
      (*job_)(i);
    }
  }
  void loop() {
    long long seen = 0;
    for (;;) {
      {
        std::unique_lock<std::mutex> lk(m_);
        cv_.wait(lk, [&] { return stop_ || gen_ != seen; });
        if (stop_) return;
        seen = gen_;
      }
      work();
      std::lock_guard<std::mutex> lk(m_);
      if (--busy_ == 0) done_.notify_all();
    }
  }
  std::vector<std::thread> th_;
  std::mutex m_;
  std::condition_variable cv_, done_;
  const std::function<void(int)>* job_ = nullptr;
  int n_ = 0, next_ = 0, busy_ = 0;
  long long gen_ = 0;
  bool stop_ = false;
};

// LRU replacement for one unit's requests.  Requested resident clusters
// leave the LRU list for the step (they cannot be evicted by it), so the next
// victim is always the list's head; each miss is admitted in request order
// unless it cannot fit even after every eviction (then it is served uncached
// and evicts nothing); the requested resident clusters become most recent, in
// request order.  `budget` counts the admissions left before an injected
// failure (< 0: none); when it reaches 0 the update stops admitting and
// returns true after restoring the recency order (a consistent state).
bool update_unit(Unit& U, int u, const Req* r, int nr, int br, ri_copy_desc* admit,
                 int32_t* nao, ri_cache_stats& st, long long* budget,
                 std::vector<int32_t>* admitted) {
  for (int i = 0; i < nr; ++i)
    if (r[i].hit && U.cl[r[i].c].in_lru) U.unlink(r[i].c);
  bool failed = false;
  for (int i = 0; i < nr && !failed; ++i) {
    if (r[i].hit) continue;
    if (*budget == 0) {
      failed = true;
      break;
    }
    const int c = r[i].c, n = r[i].n;
    const int need = (n + br - 1) / br;
    if ((long long)U.free.size() + U.lru_blocks < need) {
      ++st.uncached_clusters;
      continue;
    }
    while ((int)U.free.size() < need) {
      const int v = U.lru_head;
      U.unlink(v);
      U.release(v);
    }
    Cluster& x = U.cl[c];
    Runs runs{admit, nao, u, RI_SRC_EXEC, RI_DST_CACHE};
    int last = -1;
    for (int k = 0; k < need; ++k) {
      const int b = U.free.back();
      U.free.pop_back();
      if (last < 0) x.head = b; else U.link[last] = b;
      U.link[b] = -1;
      last = b;
      const int rows = n - k * br < br ? n - k * br : br;
      runs.add(r[i].erow + k * br, b * br, rows);
    }
    runs.flush();
    x.nblk = need;
    if (admitted) {
      admitted->push_back(u);
      admitted->push_back(c);
    }
    if (*budget > 0) --*budget;
  }
  for (int i = 0; i < nr; ++i)
    if (U.cl[r[i].c].head >= 0 && !U.cl[r[i].c].in_lru) U.push_back(r[i].c);
  return failed;
}

ri_status check_step_args(const void* cache, const int32_t* sel_ids, int32_t sel_stride,
                          int32_t k_retrieval, const int32_t* counts, const int32_t* offsets,
                          int32_t clusters, const void* fetch, const int32_t* n_fetch,
                          int32_t fetch_cap) {
  if (!cache || !sel_ids || !counts || !offsets || !fetch || !n_fetch) {
    ri::set_error("cache: NULL argument");
    return RI_ERR_INVALID_ARG;
  }
  if (k_retrieval < 0 || sel_stride < k_retrieval || clusters < 1 || fetch_cap < 0) {
    ri::set_error("cache: bad sizes (k_retrieval %d, sel_stride %d, clusters %d)", k_retrieval,
                  sel_stride, clusters);
    return RI_ERR_INVALID_ARG;
  }
  return RI_OK;
}

// Grows the per-unit tables to `clusters` ids.
ri_status prepare(ri_cache* cache, int32_t clusters) {
  try {
    for (Unit& U : cache->units) U.grow(clusters);
    cache->req_start.resize((size_t)cache->cfg.units + 1);
  } catch (...) {
    ri::set_error("cache: out of host memory");
    return RI_ERR_HOST;
  }
  return RI_OK;
}

// Validation and lookup of one step over every unit (the units as tasks of
// `pool` when given).  Fails without a state change when an id or size is
// invalid, or when the fetch list (or, when admit_cap >= 0, the admit list
// of every miss) could exceed its capacity.  On success the fetch list, the
// request records (cache->req / req_start) and the lookup counts are
// written.
ri_status lookup_step(ri_cache* cache, Pool* pool, const int32_t* sel_ids, int32_t sel_stride,
                      int32_t k_retrieval, const int32_t* counts, const int32_t* offsets,
                      int32_t clusters, ri_copy_desc* fetch, int32_t fetch_cap, int32_t admit_cap,
                      int32_t* n_fetch, ri_cache_stats* stats, const char* who) {
  ri_status s = prepare(cache, clusters);
  if (s != RI_OK) return s;
  const int nu = cache->cfg.units, br = cache->cfg.block_rows;
  std::vector<UnitCount> uc((size_t)nu);
  std::vector<ri_status> us((size_t)nu, RI_OK);
  std::vector<ri_cache_stats> ust((size_t)nu);
  auto unit_sel = [&](int u) { return sel_ids + (size_t)u * sel_stride; };
  auto unit_cnt = [&](int u) { return counts + (size_t)u * clusters; };
  auto unit_off = [&](int u) { return offsets + (size_t)u * (clusters + 1); };
  std::function<void(int)> vtask = [&](int u) {
    us[(size_t)u] = validate_unit(cache->units[(size_t)u], u, unit_sel(u), k_retrieval,
                                  unit_cnt(u), unit_off(u), clusters, br, &uc[(size_t)u]);
  };
  if (pool) pool->run(nu, vtask); else for (int u = 0; u < nu; ++u) vtask(u);
  long long nf = 0, na = 0, nreq = 0;
  for (int u = 0; u < nu; ++u) {
    if (us[(size_t)u] != RI_OK) {
      if (pool) validate_unit(cache->units[(size_t)u], u, unit_sel(u), k_retrieval, unit_cnt(u),
                              unit_off(u), clusters, br, &uc[(size_t)u]);  // this thread's error
      return us[(size_t)u];
    }
    nf += uc[(size_t)u].nf;
    na += uc[(size_t)u].na;
    nreq += uc[(size_t)u].nreq;
  }
  if (nf > fetch_cap || (admit_cap >= 0 && na > admit_cap)) {
    ri::set_error("%s: %lld fetch / up to %lld admit copies exceed capacity %d / %d", who, nf, na,
                  fetch_cap, admit_cap);
    return RI_ERR_CAPACITY;
  }
  std::vector<long long> fo((size_t)nu + 1, 0);
  try {
    cache->req.resize((size_t)nreq);
  } catch (...) {
    ri::set_error("cache: out of host memory");
    return RI_ERR_HOST;
  }
  cache->req_start[0] = 0;
  for (int u = 0; u < nu; ++u) {
    fo[(size_t)u + 1] = fo[(size_t)u] + uc[(size_t)u].nf;
    cache->req_start[(size_t)u + 1] = cache->req_start[(size_t)u] + (int32_t)uc[(size_t)u].nreq;
  }
  // each unit writes its copies from its upper-bound offset (merged block
  // copies can be fewer than counted); the lists are then closed up
  std::vector<int32_t> wrote((size_t)nu, 0);
  std::function<void(int)> ltask = [&](int u) {
    std::memset(&ust[(size_t)u], 0, sizeof(ri_cache_stats));
    wrote[(size_t)u] = lookup_unit(cache->units[(size_t)u], u, unit_sel(u), k_retrieval,
                                   unit_cnt(u), unit_off(u), br, fetch + fo[(size_t)u],
                                   cache->req.data() + cache->req_start[(size_t)u],
                                   ust[(size_t)u]);
  };
  if (pool) pool->run(nu, ltask); else for (int u = 0; u < nu; ++u) ltask(u);
  long long at = wrote[0];
  for (int u = 1; u < nu; ++u) {
    if (at != fo[(size_t)u] && wrote[(size_t)u] > 0)
      std::memmove(fetch + at, fetch + fo[(size_t)u], (size_t)wrote[(size_t)u] * sizeof(ri_copy_desc));
    at += wrote[(size_t)u];
  }
  nf = at;
  ri_cache_stats st;
  std::memset(&st, 0, sizeof(st));
  for (const ri_cache_stats& x : ust) {
    st.hit_clusters += x.hit_clusters;
    st.miss_clusters += x.miss_clusters;
    st.hit_rows += x.hit_rows;
    st.miss_rows += x.miss_rows;
    st.empty_clusters += x.empty_clusters;
  }
  *n_fetch = (int32_t)nf;
  if (stats) *stats = st;
  return RI_OK;
}

// The update of every unit from the last lookup's records.  Returns true
// when an injected failure stopped it (units after the failing one keep
// their state).
bool update_all(ri_cache* cache, ri_copy_desc* admit, int32_t* nao, ri_cache_stats& st,
                long long budget, std::vector<int32_t>* admitted) {
  const int br = cache->cfg.block_rows;
  for (int u = 0; u < cache->cfg.units; ++u) {
    const int32_t a = cache->req_start[(size_t)u], b = cache->req_start[(size_t)u + 1];
    if (update_unit(cache->units[(size_t)u], u, cache->req.data() + a, b - a, br, admit, nao, st,
                    &budget, admitted))
      return true;
  }
  return false;
}

}  // namespace

extern "C" {

ri_status ri_cache_create(const ri_cache_config* cfg, ri_cache** out) {
  if (!cfg || !out) {
    ri::set_error("cache config or output pointer is NULL");
    return RI_ERR_INVALID_ARG;
  }
  if (cfg->units < 1 || cfg->blocks_per_unit < 1 || cfg->block_rows < 1 ||
      cfg->block_rows > 1024 || (long long)cfg->blocks_per_unit * cfg->block_rows > (1ll << 30)) {
    ri::set_error("invalid cache config (units %d, blocks_per_unit %d, block_rows %d)",
                  cfg->units, cfg->blocks_per_unit, cfg->block_rows);
    return RI_ERR_INVALID_ARG;
  }
  ri_cache* c = new (std::nothrow) ri_cache;
  if (!c) {
    ri::set_error("out of host memory");
    return RI_ERR_HOST;
  }
  c->cfg = *cfg;
  try {
    c->units.resize(cfg->units);
    for (Unit& u : c->units) {
      u.link.assign(cfg->blocks_per_unit, -1);
      u.free.reserve(cfg->blocks_per_unit);
      for (int b = cfg->blocks_per_unit - 1; b >= 0; --b) u.free.push_back(b);
    }
    c->req_start.assign((size_t)cfg->units + 1, 0);
  } catch (...) {
    delete c;
    ri::set_error("out of host memory");
    return RI_ERR_HOST;
  }
  *out = c;
  return RI_OK;
}

void ri_cache_destroy(ri_cache* cache) { delete cache; }

ri_status ri_cache_plan(ri_cache* cache, const int32_t* sel_ids, int32_t sel_stride,
                        int32_t k_retrieval, const int32_t* counts, const int32_t* offsets,
                        int32_t clusters, ri_copy_desc* fetch, int32_t fetch_cap,
                        int32_t* n_fetch, ri_copy_desc* admit, int32_t admit_cap,
                        int32_t* n_admit, ri_cache_stats* stats) {
  ri_status s = check_step_args(cache, sel_ids, sel_stride, k_retrieval, counts, offsets,
                                clusters, fetch, n_fetch, fetch_cap);
  if (s != RI_OK) return s;
  if (!admit || !n_admit || admit_cap < 0) {
    ri::set_error("cache plan: NULL admit list or negative capacity");
    return RI_ERR_INVALID_ARG;
  }
  if (cache->has_worker) {
    ri::set_error("cache plan: the cache has a worker; use ri_cache_lookup");
    return RI_ERR_INVALID_ARG;
  }
  // the state changes only when every id is valid and both lists fit
  int32_t nfo = 0, nao = 0;
  ri_cache_stats st;
  s = lookup_step(cache, nullptr, sel_ids, sel_stride, k_retrieval, counts, offsets, clusters,
                  fetch, fetch_cap, admit_cap, &nfo, &st, "cache plan");
  if (s != RI_OK) return s;
  update_all(cache, admit, &nao, st, -1, nullptr);
  *n_fetch = nfo;
  *n_admit = nao;
  if (stats) *stats = st;
  return RI_OK;
}

ri_status ri_cache_resident(const ri_cache* cache, int32_t unit, int32_t cluster,
                            int32_t* blocks, int32_t cap, int32_t* n_blocks) {
  if (!cache || !n_blocks || (cap > 0 && !blocks) || cap < 0) {
    ri::set_error("cache resident: NULL argument or negative capacity");
    return RI_ERR_INVALID_ARG;
  }
  if (unit < 0 || unit >= cache->cfg.units || cluster < 0) {
    ri::set_error("cache resident: unit %d or cluster %d out of range", unit, cluster);
    return RI_ERR_INVALID_ARG;
  }
  const Unit& U = cache->units[(size_t)unit];
  *n_blocks = 0;
  if (cluster >= (int32_t)U.cl.size()) return RI_OK;
  const Cluster& x = U.cl[(size_t)cluster];
  int k = 0;
  for (int b = x.head; b >= 0; b = U.link[(size_t)b], ++k)
    if (k < cap) blocks[k] = b;
  *n_blocks = k;
  if (k > cap) {
    ri::set_error("cache resident: %d blocks exceed capacity %d", k, cap);
    return RI_ERR_CAPACITY;
  }
  return RI_OK;
}

ri_status ri_cache_validate(const ri_cache* cache) {
  if (!cache) {
    ri::set_error("cache validate: NULL cache");
    return RI_ERR_INVALID_ARG;
  }
  const int nb = cache->cfg.blocks_per_unit;
  std::vector<int8_t> seen;
  try {
    seen.resize((size_t)nb);
  } catch (...) {
    ri::set_error("cache validate: out of host memory");
    return RI_ERR_HOST;
  }
  for (int u = 0; u < cache->cfg.units; ++u) {
    const Unit& U = cache->units[(size_t)u];
    std::fill(seen.begin(), seen.end(), 0);
    for (int32_t b : U.free) {
      if (b < 0 || b >= nb || seen[(size_t)b] || U.link[(size_t)b] != -1) {
        ri::set_error("cache validate: unit %d: free block %d repeated, out of range or linked",
                      u, b);
        return RI_ERR_INVALID_ARG;
      }
      seen[(size_t)b] = 1;
    }
    // the LRU list: well linked, every member resident, block count matches
    long long lru_n = 0, lru_blocks = 0;
    int prev = -1;
    for (int c = U.lru_head; c >= 0; c = U.cl[(size_t)c].next) {
      const Cluster& x = U.cl[(size_t)c];
      if (x.prev != prev || !x.in_lru || x.head < 0 || ++lru_n > (long long)U.cl.size()) {
        ri::set_error("cache validate: unit %d: LRU list broken at cluster %d", u, c);
        return RI_ERR_INVALID_ARG;
      }
      lru_blocks += x.nblk;
      prev = c;
    }
    if (prev != U.lru_tail || lru_blocks != U.lru_blocks) {
      ri::set_error("cache validate: unit %d: LRU tail or block count wrong", u);
      return RI_ERR_INVALID_ARG;
    }
    long long resident = 0;
    for (size_t c = 0; c < U.cl.size(); ++c) {
      const Cluster& x = U.cl[c];
      if (x.head < 0) {
        if (x.nblk != 0 || x.in_lru) {
          ri::set_error("cache validate: unit %d: cluster %zu not resident but holds state", u,
                        c);
          return RI_ERR_INVALID_ARG;
        }
        continue;
      }
      ++resident;
      if (!x.in_lru) {
        ri::set_error("cache validate: unit %d: resident cluster %zu not in the LRU list", u, c);
        return RI_ERR_INVALID_ARG;
      }
      int k = 0;
      for (int b = x.head; b >= 0; b = U.link[(size_t)b]) {
        if (b >= nb || seen[(size_t)b] || ++k > x.nblk) {
          ri::set_error("cache validate: unit %d: cluster %zu: block chain broken at %d", u, c,
                        b);
          return RI_ERR_INVALID_ARG;
        }
        seen[(size_t)b] = 1;
      }
      if (k != x.nblk) {
        ri::set_error("cache validate: unit %d: cluster %zu holds %d of %d blocks", u, c, k,
                      x.nblk);
        return RI_ERR_INVALID_ARG;
      }
    }
    if (resident != lru_n) {
      ri::set_error("cache validate: unit %d: %lld resident clusters, %lld in the LRU list", u,
                    resident, lru_n);
      return RI_ERR_INVALID_ARG;
    }
    for (int b = 0; b < nb; ++b)
      if (!seen[(size_t)b]) {
        ri::set_error("cache validate: unit %d: block %d neither free nor held", u, b);
        return RI_ERR_INVALID_ARG;
      }
  }
  return RI_OK;
}

ri_status ri_max_retrieval_rows(const int32_t* counts, int32_t units, int32_t clusters,
                                int32_t k_retrieval, int32_t* out) {
  if (!counts || !out || units < 1 || clusters < 1 || k_retrieval < 0) {
    ri::set_error("max_retrieval_rows: NULL pointer or bad sizes (units %d, clusters %d, k %d)",
                  units, clusters, k_retrieval);
    return RI_ERR_INVALID_ARG;
  }
  const size_t total = (size_t)units * clusters;
  for (size_t i = 0; i < total; ++i) {
    if (counts[i] < 0) {
      ri::set_error("max_retrieval_rows: negative cluster size at entry %zu", i);
      return RI_ERR_INVALID_ARG;
    }
  }
  const int k = k_retrieval < clusters ? k_retrieval : clusters;
  std::vector<int32_t> row, res((size_t)units);
  try {
    row.resize((size_t)clusters);
  } catch (...) {
    ri::set_error("max_retrieval_rows: out of host memory");
    return RI_ERR_HOST;
  }
  for (int32_t u = 0; u < units; ++u) {
    std::copy(counts + (size_t)u * clusters, counts + (size_t)(u + 1) * clusters, row.begin());
    if (k > 0 && k < clusters)
      std::nth_element(row.begin(), row.begin() + (k - 1), row.end(), std::greater<int32_t>());
    long long sum = 0;
    for (int i = 0; i < k; ++i) sum += row[(size_t)i];
    if (sum > 0x7fffffffLL) {
      ri::set_error("max_retrieval_rows: unit %d needs %lld rows", u, sum);
      return RI_ERR_CAPACITY;
    }
    res[(size_t)u] = (int32_t)sum;
  }
  std::copy(res.begin(), res.end(), out);
  return RI_OK;
}

}  // extern "C"

// ------------------------------------------------------------ cache worker
// The asynchronous update path ("KV缓存技术与RetroInfer系统在长上下文推理中的优化实践"
// (framerc.cn) §2.2 异步更新路径: a background thread runs the LRU replacement
// and updates the mapping table late; "RetroInfer: A Vector Storage Engine for
// Scalable Long-Context LLM Inference" (gist.science) §2B: the CPU-side buffer
// manager replaces asynchronously while the GPU computes).
//
// Ordering.  Step t: ri_cache_lookup (caller thread) waits until update t-1
// has been applied on the host, makes the step's stream wait for update
// t-1's admit copies, and looks the request up; the caller issues the fetch
// copies; ri_cache_update_async records an event after them and wakes the
// worker, which applies update t to the state, writes the admit list, and on
// its side stream (after the event) copies the list to the device, runs the
// admit copies and records its own event.  So every lookup sees the state the
// synchronous ri_cache_plan would have produced, the admit copies read the
// execution buffer after the fetch copies wrote it and before the next
// step's fetch overwrites it, and a hit on a cluster admitted in step t reads
// its blocks after they were written.
struct ri_cache_worker {
  ri_cache* cache = nullptr;
  ri_cache_worker_config cfg;
  bool device = false;                  // admit copies issued on the device
  Pool* pool = nullptr;                 // helper threads of the lookup (NULL: one thread)
  std::vector<ri_copy_desc> admit_own;  // host list when the caller gives none
  ri_copy_desc* admit = nullptr;        // host admit list of the running update
  std::vector<int32_t> admitted;        // (unit, cluster) pairs admitted by the update
  cudaEvent_t ev_fetch = nullptr;       // after the step's fetch copies (step stream)
  cudaEvent_t ev_admit = nullptr;       // after the admit copies (side stream)
  bool admit_recorded = false;          // ev_admit recorded at least once
  std::thread th;
  std::mutex m;
  std::condition_variable cv;
  long long submitted = 0, completed = 0;  // updates handed over / applied
  bool stop = false;
  bool lookup_open = false;  // a lookup whose update is not handed over yet
  // result of the last applied update (read by the caller after a wait)
  ri_status status = RI_OK;  // first failure not yet reported
  char message[256] = "";
  ri_cache_stats last_stats;
  int32_t last_n_admit = 0;
  long long total_admit = 0;
  // test hooks
  long long fail_update = -1;  // index of the update that fails (-1: none)
  long long fail_after = 0;    // admissions it makes before failing
  uint32_t delay_us = 0;       // sleep at the start of every update
};

namespace {

unsigned long long wait_limit_ns(const ri_cache_worker* w) {
  return w->cfg.wait_limit_ns ? w->cfg.wait_limit_ns : 10000000000ull;
}

// Waits (caller thread) until every handed-over update has been applied.
bool wait_applied(ri_cache_worker* w, std::unique_lock<std::mutex>& lk) {
  return w->cv.wait_for(lk, std::chrono::nanoseconds(wait_limit_ns(w)),
                        [w] { return w->completed == w->submitted; });
}

// Polls an event until it completed or the limit passed (worker thread).
cudaError_t poll_event(cudaEvent_t ev, unsigned long long limit_ns) {
  const auto t0 = std::chrono::steady_clock::now();
  for (;;) {
    const cudaError_t e = cudaEventQuery(ev);
    if (e != cudaErrorNotReady) return e;
    if ((unsigned long long)std::chrono::duration_cast<std::chrono::nanoseconds>(
            std::chrono::steady_clock::now() - t0)
            .count() > limit_ns)
      return cudaErrorNotReady;
    std::this_thread::sleep_for(std::chrono::microseconds(20));
  }
}

void note_failure(ri_cache_worker* w, ri_status s, const char* msg) {
  std::lock_guard<std::mutex> lk(w->m);
  if (w->status == RI_OK) {
    w->status = s;
    snprintf(w->message, sizeof(w->message), "%s", msg);
  }
}

// One update (worker thread); the state is the worker's until it returns.
void run_update(ri_cache_worker* w, long long seq) {
  if (w->delay_us) std::this_thread::sleep_for(std::chrono::microseconds(w->delay_us));
  char msg[200];
  // the pinned host list may still be read by the previous update's copy
  if (w->device && w->admit_recorded) {
    const cudaError_t e = poll_event(w->ev_admit, wait_limit_ns(w));
    if (e != cudaSuccess) {
      snprintf(msg, sizeof(msg), "cache worker: previous admit copies %s (update %lld skipped)",
               e == cudaErrorNotReady ? "did not finish in time" : cudaGetErrorString(e), seq);
      note_failure(w, e == cudaErrorNotReady ? RI_ERR_TIMEOUT : RI_ERR_CUDA, msg);
      return;
    }
  }
  ri_cache_stats st;
  std::memset(&st, 0, sizeof(st));
  int32_t nao = 0;
  w->admitted.clear();
  const long long budget = seq == w->fail_update ? w->fail_after : -1;
  const bool failed = update_all(w->cache, w->admit, &nao, st, budget, &w->admitted);
  if (w->device) {
    const cudaStream_t side = reinterpret_cast<cudaStream_t>(w->cfg.side_stream);
    cudaError_t e = cudaStreamWaitEvent(side, w->ev_fetch, 0);
    if (e == cudaSuccess && nao > 0)
      e = cudaMemcpyAsync(w->cfg.admit_dev, w->admit, (size_t)nao * sizeof(ri_copy_desc),
                          cudaMemcpyHostToDevice, side);
    if (e == cudaSuccess && nao > 0) {
      ri::GatherArgs a;
      const ri_gather_buffers& b = w->cfg.bufs;
      a.host_K = b.host_K;
      a.host_V = b.host_V;
      a.cache_K = b.cache_K;
      a.cache_V = b.cache_V;
      a.exec_K = b.exec_K;
      a.exec_V = b.exec_V;
      a.units = b.units;
      a.M = b.M;
      a.pool_rows = b.pool_rows;
      a.exec_rows = b.exec_rows;
      e = ri::launch_gather(a, w->cfg.admit_dev, nao, static_cast<int*>(w->cfg.gather_workspace),
                            side, ri::kGatherDeviceThreads, ri::kGatherDeviceBlocksPerSM);
    }
    if (e == cudaSuccess) e = cudaEventRecord(w->ev_admit, side);
    if (e == cudaSuccess) {
      w->admit_recorded = true;
    } else {
      // the admitted clusters' blocks were never written: take them out again
      for (size_t i = 0; i + 1 < w->admitted.size(); i += 2) {
        Unit& U = w->cache->units[(size_t)w->admitted[i]];
        const int c = w->admitted[i + 1];
        if (U.cl[(size_t)c].in_lru) U.unlink(c);
        U.release(c);
      }
      nao = 0;
      snprintf(msg, sizeof(msg), "cache worker: admit copies of update %lld: %s", seq,
               cudaGetErrorString(e));
      note_failure(w, RI_ERR_CUDA, msg);
    }
  }
  if (failed) {
    snprintf(msg, sizeof(msg),
             "cache worker: update %lld failed (injected) after %lld admissions; the rest of "
             "the step was not admitted",
             seq, w->fail_after);
    note_failure(w, RI_ERR_HOST, msg);
  }
  std::lock_guard<std::mutex> lk(w->m);
  w->last_stats = st;
  w->last_n_admit = nao;
  w->total_admit += nao;
}

void worker_main(ri_cache_worker* w) {
  if (w->device) cudaSetDevice(w->cfg.device);
  std::unique_lock<std::mutex> lk(w->m);
  for (;;) {
    w->cv.wait(lk, [w] { return w->stop || w->submitted > w->completed; });
    if (w->submitted == w->completed) break;  // stop, nothing pending
    const long long seq = w->completed;
    lk.unlock();
    run_update(w, seq);
    lk.lock();
    ++w->completed;
    w->cv.notify_all();
  }
}

}  // namespace

extern "C" {

ri_status ri_cache_worker_create(ri_cache* cache, const ri_cache_worker_config* cfg,
                                 ri_cache_worker** out) {
  if (!cache || !cfg || !out) {
    ri::set_error("cache worker: NULL argument");
    return RI_ERR_INVALID_ARG;
  }
  if (cache->has_worker) {
    ri::set_error("cache worker: the cache already has a worker");
    return RI_ERR_INVALID_ARG;
  }
  if (cfg->admit_cap < 0) {
    ri::set_error("cache worker: negative admit capacity");
    return RI_ERR_INVALID_ARG;
  }
  const bool device = cfg->admit_dev != nullptr;
  if (device) {
    if (!cfg->admit_host || !cfg->gather_workspace) {
      ri::set_error("cache worker: admit_dev needs admit_host (pinned) and gather_workspace");
      return RI_ERR_INVALID_ARG;
    }
    const ri_status s = ri::check_gather_buffers(&cfg->bufs);
    if (s != RI_OK) return s;
    if (cfg->bufs.units != cache->cfg.units ||
        cfg->bufs.pool_rows != cache->cfg.blocks_per_unit * cache->cfg.block_rows ||
        !cfg->bufs.cache_K || !cfg->bufs.exec_K) {
      ri::set_error("cache worker: gather buffers do not match the cache (units %d/%d, pool "
                    "rows %d/%d) or lack the pool or execution buffer",
                    cfg->bufs.units, cache->cfg.units, cfg->bufs.pool_rows,
                    cache->cfg.blocks_per_unit * cache->cfg.block_rows);
      return RI_ERR_INVALID_ARG;
    }
  }
  ri_cache_worker* w = new (std::nothrow) ri_cache_worker;
  if (!w) {
    ri::set_error("cache worker: out of host memory");
    return RI_ERR_HOST;
  }
  w->cache = cache;
  w->cfg = *cfg;
  w->device = device;
  std::memset(&w->last_stats, 0, sizeof(w->last_stats));
  try {
    if (cfg->admit_host) {
      w->admit = cfg->admit_host;
    } else {
      w->admit_own.resize((size_t)std::max(1, cfg->admit_cap));
      w->admit = w->admit_own.data();
    }
    w->admitted.reserve(1024);
  } catch (...) {
    delete w;
    ri::set_error("cache worker: out of host memory");
    return RI_ERR_HOST;
  }
  if (device) {
    int prev = 0;
    cudaError_t e = cudaGetDevice(&prev);
    if (e == cudaSuccess) e = cudaSetDevice(cfg->device);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&w->ev_fetch, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&w->ev_admit, cudaEventDisableTiming);
    cudaSetDevice(prev);
    if (e != cudaSuccess) {
      if (w->ev_fetch) cudaEventDestroy(w->ev_fetch);
      if (w->ev_admit) cudaEventDestroy(w->ev_admit);
      delete w;
      ri::set_error("cache worker: event creation: %s", cudaGetErrorString(e));
      return RI_ERR_CUDA;
    }
  }
  try {
    int threads = cfg->lookup_threads;
    if (threads <= 0) {
      const int hw = (int)std::thread::hardware_concurrency();
      threads = std::min(8, std::max(1, hw / 2));
    }
    threads = std::min(threads, cache->cfg.units);
    if (threads > 1) w->pool = new Pool(threads - 1);
    w->th = std::thread(worker_main, w);
  } catch (...) {
    delete w->pool;
    if (w->ev_fetch) cudaEventDestroy(w->ev_fetch);
    if (w->ev_admit) cudaEventDestroy(w->ev_admit);
    delete w;
    ri::set_error("cache worker: cannot start the thread");
    return RI_ERR_HOST;
  }
  cache->has_worker = true;
  *out = w;
  return RI_OK;
}

ri_status ri_cache_worker_destroy(ri_cache_worker* w) {
  if (!w) return RI_OK;
  {
    std::lock_guard<std::mutex> lk(w->m);
    w->stop = true;
  }
  w->cv.notify_all();
  w->th.join();  // applies every handed-over update first
  ri_status s = w->status;
  if (s != RI_OK) ri::set_error("%s", w->message);
  if (w->device) {
    // the admit list and descriptors must outlive the last copies
    if (w->admit_recorded && poll_event(w->ev_admit, wait_limit_ns(w)) != cudaSuccess &&
        s == RI_OK) {
      ri::set_error("cache worker: the last admit copies did not finish");
      s = RI_ERR_TIMEOUT;
    }
    cudaEventDestroy(w->ev_fetch);
    cudaEventDestroy(w->ev_admit);
  }
  w->cache->has_worker = false;
  delete w->pool;
  delete w;
  return s;
}

ri_status ri_cache_lookup(ri_cache_worker* w, const int32_t* sel_ids, int32_t sel_stride,
                          int32_t k_retrieval, const int32_t* counts, const int32_t* offsets,
                          int32_t clusters, ri_copy_desc* fetch, int32_t fetch_cap,
                          int32_t* n_fetch, ri_cache_stats* stats, ri_stream_t stream) {
  ri_status s = check_step_args(w, sel_ids, sel_stride, k_retrieval, counts, offsets, clusters,
                                fetch, n_fetch, fetch_cap);
  if (s != RI_OK) return s;
  {
    std::unique_lock<std::mutex> lk(w->m);
    if (!wait_applied(w, lk)) {
      ri::set_error("cache lookup: the previous update was not applied within %llu ns",
                    wait_limit_ns(w));
      return RI_ERR_TIMEOUT;
    }
    if (w->status != RI_OK) {  // reported once; the state is consistent
      s = w->status;
      w->status = RI_OK;
      ri::set_error("%s", w->message);
      return s;
    }
  }
  if (w->device && w->admit_recorded) {
    const cudaError_t e =
        cudaStreamWaitEvent(reinterpret_cast<cudaStream_t>(stream), w->ev_admit, 0);
    if (e != cudaSuccess) {
      ri::set_error("cache lookup: cudaStreamWaitEvent: %s", cudaGetErrorString(e));
      return RI_ERR_CUDA;
    }
  }
  int32_t nfo = 0;
  ri_cache_stats st;
  s = lookup_step(w->cache, w->pool, sel_ids, sel_stride, k_retrieval, counts, offsets, clusters,
                  fetch, fetch_cap, w->cfg.admit_cap, &nfo, &st, "cache lookup");
  if (s != RI_OK) return s;
  *n_fetch = nfo;
  if (stats) *stats = st;
  w->lookup_open = true;
  return RI_OK;
}

ri_status ri_cache_update_async(ri_cache_worker* w, ri_stream_t stream) {
  if (!w) {
    ri::set_error("cache update: NULL worker");
    return RI_ERR_INVALID_ARG;
  }
  if (!w->lookup_open) {
    ri::set_error("cache update: no lookup to apply");
    return RI_ERR_INVALID_ARG;
  }
  if (w->device) {
    const cudaError_t e = cudaEventRecord(w->ev_fetch, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
      ri::set_error("cache update: cudaEventRecord: %s", cudaGetErrorString(e));
      return RI_ERR_CUDA;
    }
  }
  {
    std::lock_guard<std::mutex> lk(w->m);
    w->lookup_open = false;
    ++w->submitted;
  }
  w->cv.notify_all();
  return RI_OK;
}

ri_status ri_cache_worker_wait(ri_cache_worker* w, ri_cache_stats* stats, int32_t* n_admit) {
  if (!w) {
    ri::set_error("cache worker wait: NULL worker");
    return RI_ERR_INVALID_ARG;
  }
  std::unique_lock<std::mutex> lk(w->m);
  if (!wait_applied(w, lk)) {
    ri::set_error("cache worker wait: the update was not applied within %llu ns",
                  wait_limit_ns(w));
    return RI_ERR_TIMEOUT;
  }
  if (stats) *stats = w->last_stats;
  if (n_admit) *n_admit = w->last_n_admit;
  const ri_status s = w->status;
  if (s != RI_OK) {
    w->status = RI_OK;
    ri::set_error("%s", w->message);
  }
  return s;
}

ri_status ri_cache_worker_test_hooks(ri_cache_worker* w, int64_t fail_update,
                                     int64_t fail_after_admissions, uint32_t delay_us) {
  if (!w || fail_after_admissions < 0) {
    ri::set_error("cache worker hooks: NULL worker or negative admission count");
    return RI_ERR_INVALID_ARG;
  }
  std::unique_lock<std::mutex> lk(w->m);
  if (!wait_applied(w, lk)) {
    ri::set_error("cache worker hooks: an update is still running");
    return RI_ERR_TIMEOUT;
  }
  w->fail_update = fail_update;
  w->fail_after = fail_after_admissions;
  w->delay_us = delay_us;
  return RI_OK;
}

}  // extern "C"
