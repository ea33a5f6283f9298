// Host side of the wave buffer's GPU block cache (RetroInfer,
// "KV缓存技术与RetroInfer系统在长上下文推理中的优化实践" (framerc.cn) §2.2 wave
// buffer: mapping table + LRU replacement, synchronous access path; §3.1:
// fixed physical blocks of 8 rows x 128 bf16).  Per unit: a mapping table
// cluster -> blocks, the LRU order of resident clusters and a stack of free
// blocks.  ri_cache_plan turns one step's retrieval clusters into copy
// descriptors for ri_gather_blocks.
#include <algorithm>
#include <functional>
#include <iterator>
#include <list>
#include <new>
#include <unordered_map>
#include <vector>

#include "internal.h"

namespace {

constexpr int kChunkRows = 16;  // rows per copy descriptor

struct Entry {
  std::vector<int> blocks;
  std::list<int>::iterator pos;  // in the LRU list
};

struct Unit {
  std::unordered_map<int, Entry> table;
  std::list<int> lru;            // least recently used first
  long long lru_blocks = 0;      // blocks held by the clusters in `lru`
  std::vector<int> free;         // stack: the next block is free.back()
};

}  // namespace

struct ri_cache {
  ri_cache_config cfg;
  std::vector<Unit> units;
};

namespace {

// Appends the copies of `rows` rows (src..., dst...) split into chunks.
bool emit(std::vector<ri_copy_desc>& out, int unit, int src_kind, int src_row, int dst_kind,
          int dst_row, int rows) {
  for (int r = 0; r < rows; r += kChunkRows) {
    ri_copy_desc d;
    d.unit = unit;
    d.src_kind = src_kind;
    d.src_row = src_row + r;
    d.dst_kind = dst_kind;
    d.dst_row = dst_row + r;
    d.n_rows = rows - r < kChunkRows ? rows - r : kChunkRows;
    out.push_back(d);
  }
  return true;
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
  // validate every requested id and size first: the state changes only on success
  for (int u = 0; u < nu; ++u) {
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
    }
  }
  // sizing pass (read only): exact fetch copies, admit copies if every miss
  // were admitted; the state changes only when both lists fit
  auto chunks = [](long long rows) { return (rows + kChunkRows - 1) / kChunkRows; };
  long long nf = 0, na = 0;
  for (int u = 0; u < nu; ++u) {
    const Unit& U = cache->units[u];
    for (int i = 0; i < k_retrieval; ++i) {
      const int c = sel_ids[(size_t)u * sel_stride + i];
      if (c < 0) break;
      const int n = counts[(size_t)u * clusters + c];
      if (n == 0) continue;
      if (U.table.count(c)) {
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
  std::vector<ri_copy_desc> f, a;
  ri_cache_stats st = {0, 0, 0, 0, 0};
  try {
    f.reserve((size_t)nf);
    a.reserve((size_t)na);
    for (int u = 0; u < nu; ++u) {
      Unit& U = cache->units[u];
      std::vector<int> ids;
      for (int i = 0; i < k_retrieval; ++i) {
        const int c = sel_ids[(size_t)u * sel_stride + i];
        if (c < 0) break;
        ids.push_back(c);
      }
      auto rows_of = [&](int c) { return counts[(size_t)u * clusters + c]; };
      auto first_row = [&](int c) { return offsets[(size_t)u * (clusters + 1) + c]; };
      // lookup before any admission; requested resident clusters leave the
      // LRU list for the step (they cannot be evicted by it), so the next
      // victim is always the list's front
      std::vector<char> hit(ids.size());
      std::vector<int> erow(ids.size());
      int run = 0;
      for (size_t i = 0; i < ids.size(); ++i) {
        erow[i] = run;
        run += rows_of(ids[i]);
        auto it = U.table.find(ids[i]);
        hit[i] = rows_of(ids[i]) == 0 || it != U.table.end();
        if (it != U.table.end()) {
          U.lru.erase(it->second.pos);
          U.lru_blocks -= (long long)it->second.blocks.size();
        }
      }
      for (size_t i = 0; i < ids.size(); ++i) {
        const int c = ids[i], n = rows_of(c);
        if (n == 0) {
          ++st.hit_clusters;
          continue;
        }
        if (hit[i]) {
          ++st.hit_clusters;
          st.hit_rows += n;
          const std::vector<int>& bl = U.table[c].blocks;
          for (size_t k = 0; k < bl.size(); ++k) {
            const int rows = n - (int)k * br < br ? n - (int)k * br : br;
            emit(f, u, RI_SRC_CACHE, bl[k] * br, RI_DST_EXEC, erow[i] + (int)k * br, rows);
          }
          continue;
        }
        ++st.miss_clusters;
        st.miss_rows += n;
        emit(f, u, RI_SRC_HOST, first_row(c), RI_DST_EXEC, erow[i], n);
        const int need = (n + br - 1) / br;
        if ((long long)U.free.size() + U.lru_blocks < need) {
          // cannot fit even after every eviction: served uncached, nothing evicted
          ++st.uncached_clusters;
          continue;
        }
        while ((int)U.free.size() < need) {
          const int v = U.lru.front();
          U.lru.pop_front();
          std::vector<int>& vb = U.table[v].blocks;
          U.lru_blocks -= (long long)vb.size();
          U.free.insert(U.free.end(), vb.begin(), vb.end());
          U.table.erase(v);
        }
        Entry e;
        for (int k = 0; k < need; ++k) {
          e.blocks.push_back(U.free.back());
          U.free.pop_back();
        }
        for (int k = 0; k < need; ++k) {
          const int rows = n - k * br < br ? n - k * br : br;
          emit(a, u, RI_SRC_EXEC, erow[i] + k * br, RI_DST_CACHE, e.blocks[k] * br, rows);
        }
        U.table.emplace(c, std::move(e));
      }
      // requested resident clusters become most recent, in request order
      for (int c : ids) {
        auto it = U.table.find(c);
        if (it == U.table.end()) continue;
        U.lru.push_back(c);
        U.lru_blocks += (long long)it->second.blocks.size();
        it->second.pos = std::prev(U.lru.end());
      }
    }
  } catch (...) {
    ri::set_error("cache plan: out of host memory");
    return RI_ERR_HOST;
  }
  for (size_t i = 0; i < f.size(); ++i) fetch[i] = f[i];
  for (size_t i = 0; i < a.size(); ++i) admit[i] = a[i];
  *n_fetch = (int32_t)f.size();
  *n_admit = (int32_t)a.size();
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
