"""Pins of the oracle against things other than itself: library routines,
brute force on tiny inputs, closed forms, hand-derived golden files and the
invariants the pages' method implies.  CPU only."""
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp, softmax

import oracle as O
import synthetic as S

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name), encoding="utf-8") as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line)
    return rows


# ---------------------------------------------------------------- formats
def test_bf16_round_matches_torch_conversion():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(200000).astype(np.float32) * 30,
                        rng.standard_normal(1000).astype(np.float32) * 1e-39,
                        np.array([0.0, -0.0, 1.0, 65504.0, 3.0e38], np.float32)])
    ref = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    np.testing.assert_array_equal(O.bf16_round(x), ref)


def test_bf16_round_single_rounding_from_fp64():
    # 1 + 2^-8 + 2^-30 lies just above the bf16 halfway point 1 + 2^-8: a
    # single rounding goes up; rounding through fp32 first would tie and go
    # to even (down).
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert O.bf16_round(x) == 1.0 + 2.0 ** -7


# ---------------------------------------------------------------- zones
def test_zone_budgets_golden():
    rows = _golden_rows("zone_budgets.txt")
    budgets = [r for r in rows if len(r.split()) == 3]
    steady = [r for r in rows if len(r.split()) == 5]
    assert len(budgets) == 3 and len(steady) == 5
    for r in budgets:
        C, kr, ke = map(int, r.split())
        assert O.default_budgets(C) == (kr, ke)
    for r in steady:
        N, ns, M, nseg, last = map(int, r.split())
        assert len(O.steady_positions(N)) == ns
        assert O.middle_range(N)[1] == M
        segs = O.segments(M)
        assert len(segs) == nseg
        if nseg:
            assert segs[-1][1] == last


@pytest.mark.parametrize("N", [1, 67, 68, 69, 100, 8192, 8260, 16452, 20000])
def test_zones_partition_positions(N):
    sp = set(O.steady_positions(N).tolist())
    m0, M = O.middle_range(N)
    mid = set(range(m0, m0 + M))
    assert not (sp & mid)
    assert sp | mid == set(range(N))
    segs = O.segments(M)
    assert sum(L for _, L, _ in segs) == M
    assert all(K == min(512, L) for _, L, K in segs)
    assert all(s == 8192 * i for i, (s, _, _) in enumerate(segs))


# ---------------------------------------------------------------- k-means
def test_assign_matches_direct_difference_bruteforce():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((300, 7))
    mu = rng.standard_normal((23, 7))
    mu[5] = mu[3]                    # duplicate centroid: ties -> lower index
    X[:10] = mu[3]                   # rows exactly on the duplicated centroid
    lab = O.assign(X, mu)
    for i in range(X.shape[0]):
        d = [sum((X[i, k] - mu[j, k]) ** 2 for k in range(7)) for j in range(23)]
        best = min(d)
        assert lab[i] == min(j for j in range(23) if d[j] <= best + 1e-12)
    assert (lab[:10] == 3).all()


def test_kmeans_golden_empty_cluster():
    rows = dict((r.split()[0], r.split()[1:]) for r in _golden_rows("kmeans_empty_cluster.txt"))
    X = np.array(rows["points"], dtype=float)[:, None]
    res = O.kmeans(X, np.array(rows["seeds"], dtype=int), iters=1)
    np.testing.assert_array_equal(res["labels"], np.array(rows["labels"], dtype=int))
    np.testing.assert_array_equal(res["counts"], np.array(rows["counts"], dtype=int))
    np.testing.assert_array_equal(res["mu"][:, 0], np.array(rows["centroids"], dtype=float))


def _blobs(rng, n_blobs, per, dim, sep):
    centres = np.zeros((n_blobs, dim))
    centres[:, 0] = np.arange(n_blobs) * sep            # blobs sep apart along axis 0
    centres[:, 1:] = rng.standard_normal((n_blobs, dim - 1))
    lab = np.repeat(np.arange(n_blobs), per)
    rng.shuffle(lab)
    X = centres[lab] + rng.standard_normal((lab.size, dim))
    return X, lab


@pytest.mark.parametrize("dim", [1, 2, 16])
def test_kmeans_recovers_planted_partition(dim):
    rng = np.random.default_rng(dim)
    X, lab = _blobs(rng, 6, 40, dim, sep=20.0)
    init = np.array([np.flatnonzero(lab == b)[0] for b in range(6)])
    res = O.kmeans(X, init, iters=5)
    # cluster j was seeded inside blob j -> labels equal the planted ones
    np.testing.assert_array_equal(res["labels"], lab)
    for b in range(6):
        np.testing.assert_allclose(res["mu"][b], X[lab == b].mean(axis=0), rtol=0, atol=1e-12)


def test_kmeans_matches_sklearn_lloyd():
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(7)
    X, lab = _blobs(rng, 12, 30, 8, sep=3.0)
    init = np.array([np.flatnonzero(lab == b)[0] for b in range(12)])
    ours = O.kmeans(X, init, iters=30)
    km = KMeans(n_clusters=12, init=X[init].copy(), n_init=1, max_iter=30, tol=0.0,
                algorithm="lloyd").fit(X)
    np.testing.assert_array_equal(ours["labels"], km.labels_)
    np.testing.assert_allclose(ours["mu"], km.cluster_centers_, rtol=0, atol=1e-9)
    assert abs(ours["history"][-1] - km.inertia_) <= 1e-8 * km.inertia_


def test_kmeans_invariants_on_mixture():
    kv = S.make_kv(1, 1, 2068, seed=5)
    X = kv.K[0, 0, 4:4 + 2000].double().numpy()
    init = np.random.default_rng(0).choice(2000, 128, replace=False)
    res = O.kmeans(X, init, iters=6)
    assert res["counts"].sum() == 2000
    h = res["history"]
    assert all(h[i + 1] <= h[i] * (1 + 1e-12) for i in range(len(h) - 1))
    for j in np.flatnonzero(res["counts"]):
        np.testing.assert_allclose(res["mu"][j], X[res["labels"] == j].mean(axis=0), atol=1e-12)
    # each final label is a nearest centroid under the previous centroids
    prev = O.kmeans(X, init, iters=5)["mu"]
    d = ((X[:, None, :] - prev[None, :, :]) ** 2).sum(-1)
    assert (d[np.arange(2000), res["labels"]] <= d.min(axis=1) + 1e-9).all()


def test_kmeans_one_token_per_cluster_has_zero_objective():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((50, 5))
    res = O.kmeans(X, np.arange(50), iters=3)
    np.testing.assert_array_equal(res["labels"], np.arange(50))
    assert res["history"][-1] == 0.0


# ---------------------------------------------------------------- index layout
def _head(N, seed=0):
    kv = S.make_kv(1, 1, N, seed=seed)
    return kv, kv.K[0, 0].double().numpy(), kv.V[0, 0].double().numpy()


@pytest.mark.parametrize("N", [9000, 16452 + 300])
def test_index_layout_invariants(N):
    kv, Kh, Vh = _head(N)
    idx = O.build_index_head(Kh, Vh, None, iters=3)
    m0, M = O.middle_range(N)
    segs = O.segments(M)
    assert idx["C"] == sum(k for _, _, k in segs)
    assert sorted(idx["perm"].tolist()) == list(range(m0, m0 + M))        # bijection
    np.testing.assert_array_equal(idx["Kp"], Kh[idx["perm"]])
    np.testing.assert_array_equal(idx["Vp"], Vh[idx["perm"]])
    assert idx["counts"].sum() == M
    cb = 0
    for (start, L, Ks) in segs:                                          # sizes sum per segment
        assert idx["counts"][cb:cb + Ks].sum() == L
        cb += Ks
    np.testing.assert_array_equal(idx["offsets"][1:] - idx["offsets"][:-1], idx["counts"])
    # per cluster: members in position order, value sum by token-wise loop
    for c in range(0, idx["C"], 37):
        rows = range(idx["offsets"][c], idx["offsets"][c] + idx["counts"][c])
        pos = [int(idx["perm"][r]) for r in rows]
        assert pos == sorted(pos)
        acc = np.zeros(128)
        for p in pos:
            acc += Vh[p]
        np.testing.assert_allclose(idx["vsum"][c], acc, atol=1e-9)
        if pos:
            # centroid is a bf16 value within half a bf16 ulp of the members' mean
            cen = idx["centroid"][c]
            mean = Kh[pos].mean(axis=0)
            t = torch.from_numpy(cen).float()
            np.testing.assert_array_equal(t.to(torch.bfloat16).double().numpy(), cen)
            ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(mean), 1e-30))) - 7)
            assert (np.abs(cen - mean) <= 0.5 * ulp * (1 + 1e-12)).all()
    sp = O.steady_positions(N)
    np.testing.assert_array_equal(idx["Ks"], Kh[sp])


# ---------------------------------------------------------------- selection
def test_select_matches_python_sort_and_tie_rule():
    rng = np.random.default_rng(11)
    r = np.round(rng.standard_normal(400), 1)          # many exact ties
    r[[3, 50]] = -np.inf
    for k_r, k_e in [(0, 0), (5, 30), (17, 100), (400, 0), (390, 50)]:
        R, E = O.select_clusters(r, k_r, k_e)
        order = sorted(range(400), key=lambda c: (-r[c], c))
        assert R.tolist() == sorted(order[:min(k_r, 400)])
        assert E.tolist() == sorted(order[min(k_r, 400):min(k_r + k_e, 400)])


def test_select_is_permutation_invariant():
    rng = np.random.default_rng(12)
    r = rng.standard_normal(1000)
    R, E = O.select_clusters(r, 18, 230)
    p = rng.permutation(1000)
    R2, E2 = O.select_clusters(r[p], 18, 230)
    assert sorted(p[R2].tolist()) == R.tolist()
    assert sorted(p[E2].tolist()) == E.tolist()


# ---------------------------------------------------------------- attention
def _sdpa_fp64(q, K, V):
    """Full softmax attention by torch's library routine, fp64."""
    qt = torch.from_numpy(q)[None, :, None, :]
    Kt = torch.from_numpy(K)[None, None].expand(1, q.shape[0], -1, -1)
    Vt = torch.from_numpy(V)[None, None].expand(1, q.shape[0], -1, -1)
    return torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt)[0, :, 0].numpy()


@pytest.mark.parametrize("N", [9000, 20000])
def test_full_retrieval_equals_full_attention(N):
    """Spec invariant: retrieval covering every cluster (no estimation)
    is exact attention over all N tokens."""
    kv, Kh, Vh = _head(N, seed=2)
    q = S.make_queries(kv, 4)[0].double().numpy()
    idx = O.build_index_head(Kh, Vh, None, iters=2)
    res = O.tripartite_attention(q, idx, idx["C"], 0)
    ref = _sdpa_fp64(q, Kh, Vh)
    np.testing.assert_allclose(res["out"], ref, rtol=1e-10, atol=1e-12)
    lse_ref = logsumexp((q @ Kh.T) / math.sqrt(128), axis=1)
    np.testing.assert_allclose(res["lse"], lse_ref, rtol=1e-12)


@pytest.mark.parametrize("N", [68 + 300, 68 + 512])
def test_singleton_clusters_estimation_is_exact(N):
    """Spec invariant: when every cluster holds one token, the
    estimation term equals exact attention."""
    kv, Kh, Vh = _head(N, seed=4)
    q = S.make_queries(kv, 4)[0].double().numpy()
    idx = O.build_index_head(Kh, Vh, None, iters=2)
    assert (idx["counts"] == 1).all()
    res = O.tripartite_attention(q, idx, 0, idx["C"])
    np.testing.assert_allclose(res["out"], _sdpa_fp64(q, Kh, Vh), rtol=1e-10, atol=1e-12)


def test_identical_key_cluster_is_estimated_exactly():
    kv, Kh, Vh = _head(9000, seed=6)
    q = S.make_queries(kv, 4)[0].double().numpy()
    m0, M = O.middle_range(9000)
    lab = kv.component[0, 0, m0:m0 + M].copy()
    # make cluster 7 of segment 0 a set of identical (bf16) keys
    members = np.flatnonzero(lab[:8192] == 7)
    Kh = Kh.copy()
    Kh[m0 + members] = Kh[m0 + members[0]]
    idx = O.index_from_labels(Kh, Vh, lab)
    r = (q @ idx["centroid"].T).sum(0)
    r = np.where(idx["counts"] > 0, r, -np.inf)
    order = np.lexsort((np.arange(idx["C"]), -r))
    k_r = int(np.flatnonzero(order == 7)[0])        # cluster 7 is the first estimated one
    a = O.tripartite_attention(q, idx, k_r, 40)
    b = O.tripartite_attention(q, idx, k_r + 1, 39)  # ...or the last retrieved one
    assert 7 in a["E"] and 7 in b["R"]
    np.testing.assert_allclose(a["out"], b["out"], rtol=1e-11, atol=1e-13)


def test_tripartite_against_softmax_over_pseudo_tokens():
    """The estimation term is exact attention over pseudo-tokens: cluster c
    becomes one token of score s_c + log n_c carrying value Vsum_c / n_c.
    Checked with scipy's softmax / logsumexp."""
    kv, Kh, Vh = _head(20000, seed=8)
    q = S.make_queries(kv, 4)[0].double().numpy()
    idx = O.build_index_head(Kh, Vh, None, iters=2)
    k_r, k_e = O.default_budgets(idx["C"])
    res = O.tripartite_attention(q, idx, k_r, k_e)
    rows = np.concatenate([np.arange(idx["offsets"][c], idx["offsets"][c] + idx["counts"][c])
                           for c in res["R"]])
    Kx = np.concatenate([idx["Ks"], idx["Kp"][rows]])
    Vx = np.concatenate([idx["Vs"], idx["Vp"][rows]])
    E = res["E"][idx["counts"][res["E"]] > 0]
    n = idx["counts"][E].astype(float)
    for g in range(4):
        sc = np.concatenate([(Kx @ q[g]) / math.sqrt(128),
                             (idx["centroid"][E] @ q[g]) / math.sqrt(128) + np.log(n)])
        vals = np.concatenate([Vx, idx["vsum"][E] / n[:, None]])
        w = softmax(sc)
        np.testing.assert_allclose(res["out"][g], w @ vals, rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(res["lse"][g], logsumexp(sc), rtol=1e-12)
    # realised zone sizes: retrieval about 1.8 %, estimation about 23 % of the middle
    M = O.middle_range(20000)[1]
    assert 0.005 < (res["exact_tokens"] - 68) / M < 0.05
    assert 0.15 < res["estimated_tokens"] / M < 0.32


@pytest.mark.parametrize("N", [1, 30, 68])
def test_short_context_is_all_steady(N):
    kv, Kh, Vh = _head(N, seed=9)
    q = S.make_queries(kv, 4)[0].double().numpy()
    idx = O.build_index_head(Kh, Vh, None, iters=2)
    assert idx["C"] == 0
    res = O.tripartite_attention(q, idx, 9, 118)
    np.testing.assert_allclose(res["out"], _sdpa_fp64(q, Kh, Vh), rtol=1e-10, atol=1e-12)


def test_empty_clusters_rank_last():
    kv, Kh, Vh = _head(9000, seed=10)
    q = S.make_queries(kv, 4)[0].double().numpy()
    m0, M = O.middle_range(9000)
    lab = kv.component[0, 0, m0:m0 + M] % 300        # clusters 300..511 of segment 0 empty
    idx = O.index_from_labels(Kh, Vh, lab)
    res = O.tripartite_attention(q, idx, 100, 250)
    live = np.flatnonzero(idx["counts"] > 0)
    assert set(res["R"]).issubset(live)
    assert len(set(res["E"]) - set(live)) == max(0, 350 - len(live))


# ---------------------------------------------------------------- seeding
def test_strided_init_golden():
    """Default seeding floor(j * L / K) against hand-derived positions."""
    n = 0
    for r in _golden_rows("strided_init.txt"):
        kind, rest = r.split(None, 1)
        if kind == "full":
            head, vals = rest.split(":")
            L, K = (int(x) for x in head.split())
            want = [int(x) for x in vals.split()]
            assert len(want) == K
            assert O.strided_init(L, K).tolist() == want
        else:
            head, vals = rest.split("@")
            L, K = (int(x) for x in head.split())
            got = O.strided_init(L, K)
            assert len(got) == K
            for t in vals.split():
                j, v = (int(x) for x in t.split("="))
                assert int(got[j]) == v, (L, K, j)
        n += 1
    assert n == 6


@pytest.mark.parametrize("L,K", [(8124, 512), (300, 64), (513, 512), (16384, 512), (5, 5)])
def test_strided_init_spacing(L, K):
    """Seeds are distinct, start at 0, stay inside the segment and are evenly
    spaced: consecutive gaps are floor(L/K) or ceil(L/K)."""
    p = O.strided_init(L, K)
    assert p[0] == 0 and p[-1] < L and len(np.unique(p)) == K
    gaps = np.diff(p)
    assert set(gaps.tolist()) <= {L // K, -(-L // K)}


# ---------------------------------------------------------------- LRU model
def test_lru_model_golden_blocks_sequence():
    rows = _golden_rows("lru_blocks_sequence.txt")
    cap = int(rows[0].split()[1])
    sizes = {int(k): int(v) for k, v in (t.split(":") for t in rows[1].split()[1:])}
    cache = O.LRUClusterCache(cap, blocks=lambda c: sizes[c])
    for r in rows[2:]:
        req, hits, misses, resident = [p.split() for p in r.split("|")]
        h, m = cache.access([int(x) for x in req])
        assert h == [int(x) for x in hits if x != "-"]
        assert m == [int(x) for x in misses if x != "-"]
        assert sorted(cache.slot_of) == sorted(int(x) for x in resident)
        used = [b for bl in cache.slot_of.values() for b in bl]
        assert len(used) == len(set(used)) and len(used) + len(cache.free) == cap
        assert all(len(cache.slot_of[c]) == sizes[c] for c in cache.slot_of)


def test_lru_model_golden_sequence():
    rows = _golden_rows("lru_sequence.txt")
    cap = int(rows[0].split()[1])
    cache = O.LRUClusterCache(cap)
    for r in rows[1:]:
        req, hits, misses, resident = [p.split() for p in r.split("|")]
        h, m = cache.access([int(x) for x in req])
        assert h == [int(x) for x in hits if x != "-"]
        assert m == [int(x) for x in misses if x != "-"]
        assert sorted(cache.slot_of) == sorted(int(x) for x in resident)
        used = [b for bl in cache.slot_of.values() for b in bl]
        assert len(used) == len(set(used)) == len(cache.slot_of)


# ---------------------------------------------------------------- index maintenance
def _growing_golden():
    rows = _golden_rows("growing_index.txt")
    g = {"keys": {}, "append": [], "members": {}, "centroid": {}, "vsum": {}}
    for r in rows:
        t = r.split()
        if t[0] == "params":
            g["params"] = {k: int(v) for k, v in (x.split("=") for x in t[1:])}
        elif t[0] == "key":
            g["keys"][int(t[1])] = (float(t[2]), float(t[3]))
        elif t[0] == "append":
            g["append"].append((int(t[1]), int(t[2]), len(t) > 3 and t[3] == "close"))
        elif t[0] in ("prefill_members", "closed_members"):
            g["members"][int(t[1])] = [int(x) for x in t[3:]]
        elif t[0] in ("prefill_centroid", "closed_centroid"):
            g["centroid"][int(t[1])] = [float(x) for x in t[3:]]
        elif t[0] == "close_labels":
            g["close_labels"] = [int(x) for x in t[1:]]
        elif t[0] == "final_steady":
            g["steady"] = [int(x) for x in t[1:]]
        elif t[0] == "final_counts":
            g["counts"] = [int(x) for x in t[1:]]
        elif t[0] == "final_vsum":
            g["vsum"][int(t[1])] = [float(x) for x in t[3:]]
    return g


def test_growing_index_golden_sequence():
    """Hand-derived prefill, four moves into the open segment, its close by
    k-means and one move after the close."""
    g = _growing_golden()
    p = g["params"]
    n = len(g["keys"])
    K = np.array([g["keys"][i] for i in range(n)])
    V = np.array([(i, 1.0) for i in range(n)])
    gi = O.GrowingIndex(K, V, p["base_len"], iters=p["iters"], seg_len=p["seg_len"],
                        clusters_per_seg=p["clusters"], s0=p["s0"], s1=p["s1"])
    for c in (0, 1):
        assert gi.members[c] == g["members"][c]
        np.testing.assert_array_equal(gi.centroid[c], g["centroid"][c])
    for moved, cl, closes in g["append"]:
        r = gi.append()
        assert (r["moved"], r["cluster"], r["closed"]) == (moved, cl, closes)
        if closes:
            assert list(gi.last_labels) == g["close_labels"]
            for c in (2, 3):
                assert gi.members[c] == g["members"][c]
                np.testing.assert_array_equal(gi.centroid[c], g["centroid"][c])
    idx = gi.to_index()
    assert list(gi.steady()) == g["steady"]
    assert list(idx["counts"]) == g["counts"]
    for c, v in g["vsum"].items():
        np.testing.assert_array_equal(idx["vsum"][c], v)


def _growing_case(seed, N_max=700, base_len=68 + 150, seg_len=64, clusters=8, d=16):
    rng = np.random.default_rng(seed)
    centres = rng.standard_normal((12, d))
    lab = rng.integers(0, 12, N_max)
    K = O.bf16_round(centres[lab] + 0.3 * rng.standard_normal((N_max, d)))
    V = O.bf16_round(rng.standard_normal((N_max, d)))
    return K, V, O.GrowingIndex(K, V, base_len, iters=4, seg_len=seg_len,
                                clusters_per_seg=clusters)


@pytest.mark.parametrize("seed", [0, 1])
def test_growing_index_invariants(seed):
    """After every append: sizes sum to the middle count, every middle
    position is in exactly one cluster, value sums are member sums, the
    steady zone is the first 4 and last 64 positions, and every open member
    sits at a nearest target with room (brute force, direct differences)."""
    K, V, gi = _growing_case(seed)
    closes = 0
    while gi.N < K.shape[0]:
        before = [len(m) for m in gi.open]
        targets = [t.copy() for t in gi.targets]
        r = gi.append()
        closes += r["closed"]
        if not r["closed"]:
            dist = [float(((K[r["moved"]] - t) ** 2).sum()) for t in targets]
            room = [j for j in range(len(targets)) if before[j] < gi.cap]
            best = min(room, key=lambda j: (dist[j], j))
            assert r["cluster"] == best
        idx = gi.to_index()
        M = gi.N - 4 - 64
        assert idx["counts"].sum() == M
        assert sorted(idx["perm"].tolist()) == list(range(4, 4 + M))
        assert list(gi.steady()) == list(range(4)) + list(range(gi.N - 64, gi.N))
        for c in range(idx["C"]):
            a, n = idx["offsets"][c], idx["counts"][c]
            np.testing.assert_allclose(idx["vsum"][c], V[idx["perm"][a:a + n]].sum(axis=0),
                                       atol=1e-12)
    assert closes >= 7


def test_growing_index_full_slots_send_tokens_to_the_next_nearest():
    """Every key equal: all go to target 0 until its slots are full, then to
    target 1, and so on (lower id on ties, only clusters with room)."""
    d, seg_len, clusters = 4, 64, 8          # 16 slots per open cluster
    N_max = 68 + seg_len + 40
    rng = np.random.default_rng(3)
    K = O.bf16_round(rng.standard_normal((N_max, d)))
    K[68 + seg_len - 64:] = K[0]              # the moving tokens: one repeated key
    V = np.ones((N_max, d))
    gi = O.GrowingIndex(K, V, 68 + seg_len, iters=2, seg_len=seg_len, clusters_per_seg=clusters)
    d2 = gi.open_distances(K[0])
    order = sorted(range(len(gi.targets)), key=lambda j: (d2[j], j))
    got = [gi.append()["cluster"] for _ in range(2 * gi.cap + 1)]
    assert got == [order[0]] * gi.cap + [order[1]] * gi.cap + [order[2]]


def test_growing_index_equals_one_shot_build_when_segments_line_up():
    """A prefill of one full segment plus seg_len appends gives the same
    closed clusters as building the longer sequence in one go (both seeded
    by floor(j L / K)): the window, the move order and the close reproduce
    the segmented build."""
    d, seg_len, clusters, iters = 8, 128, 16, 5
    base_len = 4 + seg_len + 64
    N_end = base_len + seg_len
    rng = np.random.default_rng(11)
    centres = rng.standard_normal((20, d))
    K = O.bf16_round(centres[rng.integers(0, 20, N_end)] + 0.3 * rng.standard_normal((N_end, d)))
    V = O.bf16_round(rng.standard_normal((N_end, d)))
    gi = O.GrowingIndex(K, V, base_len, iters=iters, seg_len=seg_len, clusters_per_seg=clusters)
    for _ in range(seg_len):
        gi.append()
    one = O.build_index_head(K, V, None, iters, seg_len, clusters)
    assert one["C"] == 2 * clusters == len(gi.members)
    for c in range(one["C"]):
        a, n = one["offsets"][c], one["counts"][c]
        assert gi.members[c] == one["perm"][a:a + n].tolist()
        np.testing.assert_array_equal(gi.centroid[c], one["centroid"][c])
