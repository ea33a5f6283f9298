// Host side of the wave buffer's GPU block cache (RetroInfer,
// "KV缓存技术与RetroInfer系统在长上下文推理中的优化实践" (framerc.cn) §2.2 wave
// buffer: mapping table + LRU replacement, synchronous access path; §3.1:
// fixed physical blocks of 8 rows x 128 bf16).  Per unit: a mapping table
// cluster -> chain of blocks, the LRU order of resident clusters and a stack
// of free blocks, all as flat arrays indexed by cluster id or block id (one
// step touches each requested cluster in O(1) plus its blocks).
// ri_cache_plan turns one step's retrieval clusters into copy descriptors
// for ri_gather_blocks.
#include <algorithm>
#include <functional>
#include <new>
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
};

}  // namespace

struct ri_cache {
  ri_cache_config cfg;
  std::vector<Unit> units;
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
  if (!cache || !sel_ids || !counts || !offsets || !fetch || !n_fetch || !admit || !n_admit) {
    ri::set_error("cache plan: NULL argument");
    return RI_ERR_INVALID_ARG;
  }
  if (k_retrieval < 0 || sel_stride < k_retrieval || clusters < 1 || fetch_cap < 0 ||
      admit_cap < 0) {
    ri::set_error("cache plan: bad sizes (k_retrieval %d, sel_stride %d, clusters %d)",
                  k_retrieval, sel_stride, clusters);
    return RI_ERR_INVALID_ARG;
  }
  const int br = cache->cfg.block_rows;
  const int nu = cache->cfg.units;
  try {
    for (Unit& U : cache->units) U.grow(clusters);
  } catch (...) {
    ri::set_error("cache plan: out of host memory");
    return RI_ERR_HOST;
  }
  // one read-only pass: every requested id and size checked, and the exact
  // fetch copies / admit copies if every miss were admitted counted; the
  // state changes only when all is valid and both lists fit
  auto chunks = [](long long rows) { return (rows + kChunkRows - 1) / kChunkRows; };
  long long nf = 0, na = 0;
  for (int u = 0; u < nu; ++u) {
    const Unit& U = cache->units[u];
    int prev = -1;
    for (int i = 0; i < k_retrieval; ++i) {
      const int c = sel_ids[(size_t)u * sel_stride + i];
      if (c < 0) break;
      if (c >= clusters || c <= prev) {
        ri::set_error("cache plan: unit %d entry %d: cluster id %d out of range or not ascending",
                      u, i, c);
        return RI_ERR_INVALID_ARG;
      }
      prev = c;
      const int n = counts[(size_t)u * clusters + c];
      const int row = offsets[(size_t)u * (clusters + 1) + c];
      if (n < 0 || row < 0) {
        ri::set_error("cache plan: unit %d cluster %d: negative size or row", u, c);
        return RI_ERR_INVALID_ARG;
      }
      if (n == 0) continue;
      if (U.cl[c].head >= 0) {
        for (long long k = 0; k * br < n; ++k) nf += chunks(n - k * br < br ? n - k * br : br);
      } else {
        nf += chunks(n);
        for (long long k = 0; k * br < n; ++k) na += chunks(n - k * br < br ? n - k * br : br);
      }
    }
  }
  if (nf > fetch_cap || na > admit_cap) {
    ri::set_error("cache plan: %lld fetch / up to %lld admit copies exceed capacity %d / %d",
                  nf, na, fetch_cap, admit_cap);
    return RI_ERR_CAPACITY;
  }
  int32_t nfo = 0, nao = 0;
  ri_cache_stats st = {0, 0, 0, 0, 0};
  for (int u = 0; u < nu; ++u) {
    Unit& U = cache->units[u];
    const int32_t* sel = sel_ids + (size_t)u * sel_stride;
    const int32_t* cnt = counts + (size_t)u * clusters;
    const int32_t* off = offsets + (size_t)u * (clusters + 1);
    int nid = 0;
    while (nid < k_retrieval && sel[nid] >= 0) ++nid;
    // lookup before any admission; requested resident clusters leave the
    // LRU list for the step (they cannot be evicted by it), so the next
    // victim is always the list's head
    for (int i = 0; i < nid; ++i)
      if (U.cl[sel[i]].in_lru) U.unlink(sel[i]);
    int run = 0;  // execution-buffer row of the next cluster
    for (int i = 0; i < nid; ++i) {
      const int c = sel[i], n = cnt[c];
      const int erow = run;
      run += n;
      if (n == 0) {
        ++st.hit_clusters;
        continue;
      }
      Cluster& x = U.cl[c];
      if (x.head >= 0) {
        ++st.hit_clusters;
        st.hit_rows += n;
        Runs runs{fetch, &nfo, u, RI_SRC_CACHE, RI_DST_EXEC};
        int k = 0;
        for (int b = x.head; b >= 0; b = U.link[b], ++k) {
          const int rows = n - k * br < br ? n - k * br : br;
          runs.add(b * br, erow + k * br, rows);
        }
        runs.flush();
        continue;
      }
      ++st.miss_clusters;
      st.miss_rows += n;
      emit(fetch, &nfo, u, RI_SRC_HOST, off[c], RI_DST_EXEC, erow, n);
      const int need = (n + br - 1) / br;
      if ((long long)U.free.size() + U.lru_blocks < need) {
        // cannot fit even after every eviction: served uncached, nothing evicted
        ++st.uncached_clusters;
        continue;
      }
      while ((int)U.free.size() < need) {
        const int v = U.lru_head;
        U.unlink(v);
        Cluster& y = U.cl[v];
        for (int b = y.head; b >= 0;) {
          const int nb = U.link[b];
          U.link[b] = -1;
          U.free.push_back(b);
          b = nb;
        }
        y.head = -1;
        y.nblk = 0;
      }
      Runs runs{admit, &nao, u, RI_SRC_EXEC, RI_DST_CACHE};
      int last = -1;
      for (int k = 0; k < need; ++k) {
        const int b = U.free.back();
        U.free.pop_back();
        if (last < 0) x.head = b; else U.link[last] = b;
        U.link[b] = -1;
        last = b;
        const int rows = n - k * br < br ? n - k * br : br;
        runs.add(erow + k * br, b * br, rows);
      }
      runs.flush();
      x.nblk = need;
    }
    // requested resident clusters become most recent, in request order
    for (int i = 0; i < nid; ++i)
      if (U.cl[sel[i]].head >= 0) U.push_back(sel[i]);
  }
  *n_fetch = nfo;
  *n_admit = nao;
  if (stats) *stats = st;
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
