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
    stats = dict(hit_clusters=0, miss_clusters=0, uncached_clusters=0, hit_rows=0, miss_rows=0,
                 empty_clusters=0)
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
                stats["empty_clusters"] += 1
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
    c.validate()
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


# ---------------------------------------------------------------- cache worker
# The asynchronous update path ("KV缓存技术与RetroInfer系统在长上下文推理中的优化实践"
# (framerc.cn) §2.2 异步更新路径): lookup on the caller's thread, LRU update on
# the worker's.  Host-only workers (no device buffers) run here without a GPU.

def _random_steps(seed, units=3, C=64, k_r=12, n_steps=25):
    rng = np.random.default_rng(seed)
    sizes = rng.integers(0, 40, size=(units, C))
    sizes[:, ::17] = 0
    counts, offsets = _index_arrays(sizes)
    cap = int(rng.integers(4, 30))
    hot = [rng.choice(C, size=20, replace=False) for _ in range(units)]
    steps = []
    for _ in range(n_steps):
        rows = []
        for u in range(units):
            pool = hot[u] if rng.random() < 0.7 else np.arange(C)
            rows.append(rng.choice(pool, size=int(rng.integers(0, k_r + 1)), replace=False))
        steps.append(_sel(rows, k_r))
    return counts, offsets, cap, steps


def _lookup_keys(st):
    return {k: v for k, v in st.items() if k != "uncached_clusters"}


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
@pytest.mark.parametrize("delay_us", [0, 3000])
def test_worker_steps_equal_the_synchronous_plan(seed, delay_us):
    """Per step: the lookup's fetch list and counts, and the update's admit
    list and uncached count, equal ri_cache_plan's on a second cache fed the
    same steps.  With a delayed worker the lookup has to wait for the
    previous update; the results must not change."""
    units, k_r, br = 3, 12, 8
    counts, offsets, cap, steps = _random_steps(seed, units=units, k_r=k_r)
    sync = R.BlockCache(units, cap, br)
    acache = R.BlockCache(units, cap, br)
    w = R.CacheWorker(acache, admit_cap=units * 2000)
    w.test_hooks(delay_us=delay_us)
    for sel in steps:
        f, a, st = sync.plan(sel, k_r, counts, offsets)
        fl, lst = w.lookup(sel, k_r, counts, offsets)
        assert _rows(fl) == _rows(f)
        assert _lookup_keys(lst) == _lookup_keys(st) and lst["uncached_clusters"] == 0
        w.update_async()
        ust, al = w.wait()
        assert _rows(al) == _rows(a)
        assert ust["uncached_clusters"] == st["uncached_clusters"]
    w.close()
    acache.validate()
    for u in range(units):
        for c in range(counts.shape[1]):
            assert acache.resident(u, c) == sync.resident(u, c)
    sync.close()
    acache.close()


def test_worker_lookup_waits_for_the_previous_update():
    """Back-to-back steps with no wait in between: each lookup must see the
    previous step's admissions (a miss admitted at step t is a hit at t+1)."""
    br = 8
    counts, offsets = _index_arrays([[8, 16, 8, 8]])
    c = R.BlockCache(1, 8, br)
    w = R.CacheWorker(c, admit_cap=64)
    w.test_hooks(delay_us=20000)  # 20 ms per update: the lookup must block
    f0, s0 = w.lookup(_sel([[0, 1]], 3), 3, counts, offsets)
    assert s0["miss_clusters"] == 2
    w.update_async()
    f1, s1 = w.lookup(_sel([[0, 1, 2]], 3), 3, counts, offsets)
    assert s1["hit_clusters"] == 2 and s1["miss_clusters"] == 1
    assert [int(r[1]) for r in f1] == [R.SRC_CACHE, R.SRC_CACHE, R.SRC_HOST]
    w.update_async()
    w.close()
    c.validate()
    assert len(c.resident(0, 2)) == 1
    c.close()


def test_worker_wait_limit_expires_and_recovers():
    import time
    counts, offsets = _index_arrays([[8, 16, 8, 8]])
    c = R.BlockCache(1, 8, 8)
    w = R.CacheWorker(c, admit_cap=64, wait_limit_ns=30_000_000)  # 30 ms
    w.test_hooks(delay_us=300_000)                               # 300 ms update
    w.lookup(_sel([[0, 1]], 3), 3, counts, offsets)
    w.update_async()
    with pytest.raises(R.RIError) as e:
        w.lookup(_sel([[0, 2]], 3), 3, counts, offsets)
    assert e.value.status == R.STATUS_CODES["RI_ERR_TIMEOUT"]
    time.sleep(0.4)
    f, st = w.lookup(_sel([[0, 2]], 3), 3, counts, offsets)  # the update has landed
    assert st["hit_clusters"] == 1 and st["miss_clusters"] == 1
    w.update_async()
    w.close()
    c.validate()
    c.close()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_worker_injected_failure_leaves_a_consistent_cache(seed):
    """Update number `t` fails before its first admission.  The failure is
    reported once by the next lookup; the state is then exactly the oracle
    model's after: units before the failing one updated, the failing unit's
    requested residents made most recent (nothing admitted or evicted), later
    units untouched.  From there on the worker again matches the model."""
    units, k_r, br = 3, 12, 8
    counts, offsets, cap, steps = _random_steps(seed + 10, units=units, k_r=k_r, n_steps=14)
    t = 6
    c = R.BlockCache(units, cap, br)
    w = R.CacheWorker(c, admit_cap=units * 2000)
    w.test_hooks(fail_update=t, fail_after=0)
    models = [O.LRUClusterCache(cap, blocks=lambda cl, u=u: -(-int(counts[u, cl]) // br))
              for u in range(units)]
    failed_seen = False
    for i, sel in enumerate(steps):
        if i == t + 1:
            with pytest.raises(R.RIError) as e:
                w.lookup(sel, k_r, counts, offsets)
            assert e.value.status == R.STATUS_CODES["RI_ERR_HOST"]
            failed_seen = True
        fl, _ = w.lookup(sel, k_r, counts, offsets)
        if i == t:
            # the failing update on the model: units in order until the first
            # with a miss, which only refreshes its requested residents
            for u in range(units):
                ids = [int(x) for x in sel[u, :k_r] if x >= 0 and counts[u, x] > 0]
                if any(x not in models[u].slot_of for x in ids):
                    models[u].access([x for x in ids if x in models[u].slot_of])
                    break
                models[u].access(ids)
            w.update_async()
            continue
        ef, ea, _ = expected_plan(models, sel, k_r, counts, offsets, br)
        assert _rows(fl) == ef
        w.update_async()
        _, al = w.wait()
        assert _rows(al) == ea
    assert failed_seen
    w.close()
    c.validate()
    c.close()


def test_worker_failure_after_some_admissions_keeps_invariants():
    units, k_r, br = 3, 12, 8
    counts, offsets, cap, steps = _random_steps(7, units=units, k_r=k_r, n_steps=12)
    c = R.BlockCache(units, cap, br)
    w = R.CacheWorker(c, admit_cap=units * 2000)
    w.test_hooks(fail_update=4, fail_after=2)
    errors = 0
    for sel in steps:
        try:
            fl, st = w.lookup(sel, k_r, counts, offsets)
        except R.RIError as e:
            assert e.status == R.STATUS_CODES["RI_ERR_HOST"]
            errors += 1
            fl, st = w.lookup(sel, k_r, counts, offsets)
        # every cache-sourced copy reads blocks of a resident requested cluster
        for r in fl:
            if int(r[1]) == R.SRC_CACHE:
                assert 0 <= int(r[2]) and int(r[2]) + int(r[5]) <= cap * br
        w.update_async()
        try:
            w.wait()
        except R.RIError as e:  # the failure is reported once, by the first to ask
            assert e.status == R.STATUS_CODES["RI_ERR_HOST"]
            errors += 1
        c.validate()
    assert errors == 1
    w.close()
    c.close()


def test_worker_refusals():
    counts, offsets = _index_arrays([[8, 16, 8, 8]])
    c = R.BlockCache(1, 8, 8)
    w = R.CacheWorker(c, admit_cap=1)
    with pytest.raises(R.RIError):          # update without a lookup
        w.update_async()
    with pytest.raises(R.RIError):          # ri_cache_plan while a worker is attached
        c.plan(_sel([[0]], 3), 3, counts, offsets)
    with pytest.raises(R.RIError) as e:     # admit list could overflow: state unchanged
        w.lookup(_sel([[0, 1]], 3), 3, counts, offsets)
    assert e.value.status == R.STATUS_CODES["RI_ERR_CAPACITY"]
    f, st = w.lookup(_sel([[0]], 3), 3, counts, offsets)
    assert st["miss_clusters"] == 1
    w.update_async()
    w.close()
    c.validate()
    f, a, st = c.plan(_sel([[0]], 3), 3, counts, offsets)  # detached: plan works again
    assert st["hit_clusters"] == 1
    c.close()


def test_validate_accepts_a_fresh_cache_and_rejects_null():
    assert R.lib.ri_cache_validate(None) == R.STATUS_CODES["RI_ERR_INVALID_ARG"]
    c = R.BlockCache(2, 5, 8)
    c.validate()
    c.close()
