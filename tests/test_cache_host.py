"""Host-side block cache (ri_cache_plan) against the oracle's cache model.

The library's plan must be exactly the copies the oracle model implies: per
requested retrieval cluster, in id order, cache->exec copies of its blocks for
a hit, one host->exec copy for a miss, and exec->cache copies for an admitted
miss, each split into copies of at most 16 rows; block ids included (both
sides take free blocks from the same stack discipline).  Pure host code: no
GPU needed."""
import numpy as np
import pytest

import oracle as O

R = pytest.importorskip("kv_cache_vector_segmented_b200")

CHUNK = 16


def _chunks(unit, sk, sr, dk, dr, n):
    return [(unit, sk, sr + r, dk, dr + r, min(CHUNK, n - r)) for r in range(0, n, CHUNK)]


def _block_copies(unit, sk, dk, pieces):
    """Copies of a cluster's block-sized pieces (src row, dst row, rows) in
    order, adjacent pieces merged while the copy stays within CHUNK rows."""
    out, cur = [], None
    for s, d, r in pieces:
        if cur and s == cur[0] + cur[2] and d == cur[1] + cur[2] and cur[2] + r <= CHUNK:
            cur = (cur[0], cur[1], cur[2] + r)
            continue
        if cur:
            out += _chunks(unit, sk, cur[0], dk, cur[1], cur[2])
        cur = (s, d, r)
    if cur:
        out += _chunks(unit, sk, cur[0], dk, cur[1], cur[2])
    return out


def expected_plan(models, sel, k_r, counts, offsets, br):
    fetch, admit = [], []
    stats = dict(hit_clusters=0, miss_clusters=0, uncached_clusters=0, hit_rows=0, miss_rows=0)
    for u, model in enumerate(models):
        ids = [int(c) for c in sel[u, :k_r] if c >= 0]
        erow, run = {}, 0
        for c in ids:
            erow[c] = run
            run += int(counts[u, c])
        before = {c: list(model.slot_of[c]) for c in ids if c in model.slot_of}
        model.access(ids)
        for c in ids:
            n = int(counts[u, c])
            if n == 0:
                stats["hit_clusters"] += 1
                continue
            if c in before:
                stats["hit_clusters"] += 1
                stats["hit_rows"] += n
                fetch += _block_copies(u, R.SRC_CACHE, R.DST_EXEC,
                                       [(b * br, erow[c] + k * br, min(br, n - k * br))
                                        for k, b in enumerate(before[c])])
                continue
            stats["miss_clusters"] += 1
            stats["miss_rows"] += n
            fetch += _chunks(u, R.SRC_HOST, int(offsets[u, c]), R.DST_EXEC, erow[c], n)
            if c in model.slot_of:
                admit += _block_copies(u, R.SRC_EXEC, R.DST_CACHE,
                                       [(erow[c] + k * br, b * br, min(br, n - k * br))
                                        for k, b in enumerate(model.slot_of[c])])
            else:
                stats["uncached_clusters"] += 1
    return fetch, admit, stats


def _rows(a):
    return [tuple(int(x) for x in r) for r in a]


def _index_arrays(sizes_per_unit):
    counts = np.asarray(sizes_per_unit, dtype=np.int32)
    offsets = np.zeros((counts.shape[0], counts.shape[1] + 1), dtype=np.int32)
    offsets[:, 1:] = np.cumsum(counts, axis=1)
    return counts, offsets


def _run(units, cap_blocks, br, counts, offsets, steps, k_r):
    lib_cache = R.BlockCache(units, cap_blocks, br)
    models = [O.LRUClusterCache(cap_blocks, blocks=lambda c, u=u: -(-int(counts[u, c]) // br))
              for u in range(units)]
    for sel in steps:
        f, a, st = lib_cache.plan(sel, k_r, counts, offsets)
        ef, ea, est = expected_plan(models, sel, k_r, counts, offsets, br)
        assert _rows(f) == ef
        assert _rows(a) == ea
        assert st == est
    lib_cache.close()


def _sel(rows, k_r):
    out = np.full((len(rows), k_r + 3), -1, dtype=np.int32)
    for u, ids in enumerate(rows):
        out[u, :len(ids)] = sorted(ids)
    return out


@pytest.mark.parametrize("golden,br", [("lru_sequence.txt", 8), ("lru_blocks_sequence.txt", 8)])
def test_plan_matches_golden_sequences(golden, br):
    from tests.test_oracle_pins import _golden_rows
    rows = _golden_rows(golden)
    cap = int(rows[0].split()[1])
    body = rows[1:]
    blocks = {}
    if body and body[0].startswith("blocks"):
        blocks = {int(k): int(v) for k, v in (t.split(":") for t in body[0].split()[1:])}
        body = body[1:]
    C = 8
    sizes = [blocks.get(c, 1) * br - (c % 3) for c in range(C)]  # ceil(n / br) = blocks
    counts, offsets = _index_arrays([sizes])
    k_r = 6
    steps = [_sel([[int(x) for x in r.split("|")[0].split()]], k_r) for r in body]
    _run(1, cap, br, counts, offsets, steps, k_r)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_plan_matches_model_random(seed):
    rng = np.random.default_rng(seed)
    units, C, k_r, br = 3, 64, 12, 8
    sizes = rng.integers(0, 40, size=(units, C))
    sizes[:, ::17] = 0  # some empty clusters
    counts, offsets = _index_arrays(sizes)
    cap = int(rng.integers(4, 30))
    steps = []
    hot = [rng.choice(C, size=20, replace=False) for _ in range(units)]
    for _ in range(25):
        rows = []
        for u in range(units):
            pool = hot[u] if rng.random() < 0.7 else np.arange(C)
            rows.append(rng.choice(pool, size=int(rng.integers(0, k_r + 1)), replace=False))
        steps.append(_sel(rows, k_r))
    _run(units, cap, br, counts, offsets, steps, k_r)


def test_cluster_larger_than_the_cache_is_served_uncached():
    """A cluster needing more blocks than the whole cache is copied from host
    memory every time and never admitted; the residents stay in place."""
    br = 8
    counts, offsets = _index_arrays([[8, 40, 16, 3]])  # cluster 1: 5 blocks
    steps = [_sel([[0, 2]], 3), _sel([[1]], 3), _sel([[0, 1, 2]], 3), _sel([[1, 3]], 3)]
    _run(1, 4, br, counts, offsets, steps, 3)
    c = R.BlockCache(1, 4, br)
    c.plan(steps[0], 3, counts, offsets)
    f, a, st = c.plan(steps[1], 3, counts, offsets)
    assert st["uncached_clusters"] == 1 and len(a) == 0
    assert all(int(r[1]) == R.SRC_HOST for r in f)
    f, a, st = c.plan(steps[2], 3, counts, offsets)
    assert st["hit_clusters"] == 2 and st["uncached_clusters"] == 1
    c.close()


def test_plan_rejects_bad_input_and_keeps_state():
    counts, offsets = _index_arrays([[9, 3, 16, 1]])
    c = R.BlockCache(1, 2, 8)
    with pytest.raises(R.RIError):
        c.plan(np.array([[2, 1, -1]], dtype=np.int32), 2, counts, offsets)  # not ascending
    with pytest.raises(R.RIError):
        c.plan(np.array([[0, 7, -1]], dtype=np.int32), 2, counts, offsets)  # out of range
    # capacity failure of the output lists leaves the state untouched
    sel = np.array([[0, 2, -1]], dtype=np.int32)
    fetch = np.zeros((1, 6), dtype=np.int32)
    admit = np.zeros((8, 6), dtype=np.int32)
    import ctypes
    nf, na = ctypes.c_int32(), ctypes.c_int32()
    st = R.lib.ri_cache_plan(c._h, sel.ctypes.data, 3, 2, counts.ctypes.data,
                             offsets.ctypes.data, 4, fetch.ctypes.data, 1, ctypes.byref(nf),
                             admit.ctypes.data, 8, ctypes.byref(na), None)
    assert st == R.STATUS_CODES["RI_ERR_CAPACITY"]
    f, a, s = c.plan(sel, 2, counts, offsets)  # first real step: both miss
    assert s["miss_clusters"] == 2 and s["hit_clusters"] == 0
    c.close()


def test_cache_create_rejects_bad_config():
    with pytest.raises(R.RIError):
        R.BlockCache(0, 4, 8)
    with pytest.raises(R.RIError):
        R.BlockCache(1, 0, 8)
    with pytest.raises(R.RIError):
        R.BlockCache(1, 4, 0)


@pytest.mark.parametrize("seed", [0, 1])
def test_max_retrieval_rows_matches_sorted_sums(seed):
    """Sum of the k largest sizes per unit, against a full sort."""
    rng = np.random.default_rng(seed)
    counts = rng.integers(0, 60, size=(5, 300)).astype(np.int32)
    counts[2] = 0                      # a unit with only empty clusters
    counts[3, ::7] = 200               # ties among the largest
    for k in (0, 1, 5, 147, 299, 300, 1000):
        want = np.sort(counts, axis=1)[:, ::-1][:, :k].sum(axis=1)
        np.testing.assert_array_equal(R.max_retrieval_rows(counts, k), want)


def test_max_retrieval_rows_rejects_bad_input():
    with pytest.raises(R.RIError):
        R.max_retrieval_rows(np.array([[3, -1, 2]], dtype=np.int32), 2)
    with pytest.raises(R.RIError):
        R.max_retrieval_rows(np.array([[3, 1, 2]], dtype=np.int32), -1)
    big = np.full((1, 3), 2 ** 30, dtype=np.int32)
    with pytest.raises(R.RIError):
        R.max_retrieval_rows(big, 3)   # 3 * 2^30 rows do not fit an int32
