"""GPU parity of the segmented k-means index build against the oracle.

Bars (the benchmark spec): assignments >= 99.9 % identical and objective within 0.1 %
at a fixed seed, seeding and iteration count.  The layout outputs are checked
exactly against their definitions on the device's own labels: the
permutation is a bijection, rows are the permuted keys and values, offsets
are the prefix sums of the sizes, value sums are sums of members, centroids
are the bf16 rounding of the members' mean."""
import numpy as np
import pytest
import torch

import oracle as O
import synthetic as S
from tests import _util as U

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def R():
    if not torch.cuda.is_available():
        pytest.skip("needs CUDA")
    import kv_cache_vector_segmented_b200 as R
    return R


def _seeds(B, H, N, seg_len=8192, clusters=512, seed=3):
    m0, M = O.middle_range(N)
    segs = O.segments(M, seg_len, clusters)
    return S.init_positions([s[1] for s in segs], [s[2] for s in segs], B, H, seed=seed)


def _check_layout(R, kv, idx, seg_len, clusters):
    """Exact structural checks of the device index against its own labels."""
    B, H, N, d = kv.K.shape
    m0, M = O.middle_range(N)
    segs = O.segments(M, seg_len, clusters)
    K64 = kv.K.double()
    V64 = kv.V.double()
    perm = idx.perm.cpu().long()
    counts = idx.counts.cpu().long()
    offsets = idx.offsets.cpu().long()
    labels = idx.labels.cpu().long()
    Kp = idx.Kp.cpu()
    Vp = idx.Vp.cpu()
    vsum = idx.vsum.cpu().double()
    cen = idx.centroid.cpu()
    for b in range(B):
        for h in range(H):
            p = perm[b, h]
            assert torch.equal(torch.sort(p).values, torch.arange(m0, m0 + M))
            assert torch.equal(Kp[b, h], kv.K[b, h, p])
            assert torch.equal(Vp[b, h], kv.V[b, h, p])
            assert int(offsets[b, h, -1]) == M
            assert torch.equal(offsets[b, h, 1:] - offsets[b, h, :-1], counts[b, h])
            cb = 0
            for (start, L, Ks) in segs:
                lab = labels[b, h, start:start + L]
                assert int(lab.min()) >= 0 and int(lab.max()) < Ks
                n = torch.bincount(lab, minlength=Ks)
                assert torch.equal(n, counts[b, h, cb:cb + Ks])
                assert int(n.sum()) == L
                pos = m0 + start + torch.arange(L)
                # rows of each cluster: its members in position order
                order = torch.sort(lab, stable=True).indices
                assert torch.equal(p[start:start + L], pos[order])
                sums = torch.zeros(Ks, d, dtype=torch.float64).index_add_(0, lab, V64[b, h, pos])
                np.testing.assert_allclose(vsum[b, h, cb:cb + Ks].numpy(), sums.numpy(),
                                           rtol=1e-5, atol=1e-4)
                ks = torch.zeros(Ks, d, dtype=torch.float64).index_add_(0, lab, K64[b, h, pos])
                live = n > 0
                mean = ks[live] / n[live, None]
                c = cen[b, h, cb:cb + Ks][live].double()
                # bf16 of the fp32 mean: within one bf16 ulp of the exact mean
                ulp = torch.exp2(torch.floor(torch.log2(mean.abs().clamp_min(1e-30))) - 7)
                assert ((c - mean).abs() <= ulp * 1.0001 + 1e-6).all()
                cb += Ks


def _compare_kmeans(R, B, H, N, iters, seg_len=8192, clusters=512, seed=0, use_init=True,
                    sample_units=None):
    dev = torch.device("cuda:0")
    kv = S.make_kv(B, H, N, seed=seed)
    ip = _seeds(B, H, N, seg_len, clusters, seed=seed + 50) if use_init else None
    cfg = R.IndexConfig.make(B, H, 4, N, seg_len=seg_len, clusters_per_seg=clusters, iters=iters)
    idx = R.build_index(kv.K.to(dev), kv.V.to(dev), cfg,
                        init_pos=None if ip is None else torch.from_numpy(ip).to(dev))
    ws = idx._build_ws
    assert R.read_device_status(ws) == 0
    m0, M = O.middle_range(N)
    segs = O.segments(M, seg_len, clusters)
    labels = idx.labels.cpu().numpy()
    obj = idx.objective.cpu().numpy()
    units = [(b, h, s) for b in range(B) for h in range(H) for s in range(len(segs))]
    if sample_units is not None:
        units = [units[i] for i in sample_units]
    agree = total = 0
    for (b, h, s) in units:
        start, L, Ks = segs[s]
        cb = sum(x[2] for x in segs[:s])
        X = kv.K[b, h, m0 + start:m0 + start + L].double().numpy()
        init = O.strided_init(L, Ks) if ip is None else ip[b, h, cb:cb + Ks]
        res = O.kmeans(X, init, iters)
        got = labels[b, h, start:start + L]
        agree += int((got == res["labels"]).sum())
        total += L
        o_ref = O.objective(X, res["labels"], res["mu"])
        assert abs(obj[b, h, s] - o_ref) <= U.OBJ_RTOL * max(o_ref, 1e-30) + 1e-3, \
            f"unit {(b, h, s)}: objective {obj[b, h, s]} vs {o_ref}"
    frac = agree / total
    assert frac >= U.ASSIGN_AGREE, f"assignment agreement {frac}"
    return kv, idx, frac


def test_kmeans_single_segment_8k(R):
    """One KV head, 8K context (one segment of 8124 middle tokens, 512
    clusters), 10 Lloyd iterations from seeded positions."""
    kv, idx, frac = _compare_kmeans(R, 1, 1, 8192, 10)
    _check_layout(R, kv, idx, 8192, 512)


def test_kmeans_ragged_multihead(R):
    kv, idx, frac = _compare_kmeans(R, 2, 2, 8192 + 68 + 3000, 5, seed=1)
    _check_layout(R, kv, idx, 8192, 512)


def test_kmeans_small_segments_and_strided_seeds(R):
    kv, idx, frac = _compare_kmeans(R, 1, 3, 68 + 1000, 4, seg_len=300, clusters=64, seed=2,
                                    use_init=False)
    _check_layout(R, kv, idx, 300, 64)


def test_kmeans_max_segment_length(R):
    """Segments of the largest supported length (16384 tokens, 512
    clusters) plus a ragged 500-token last segment: the counting sort's
    largest shared-memory footprint and 512 positions per warp."""
    kv, idx, frac = _compare_kmeans(R, 1, 1, 68 + 16384 + 500, 3, seg_len=16384, seed=12)
    _check_layout(R, kv, idx, 16384, 512)


def test_kmeans_one_token_per_cluster(R):
    """K_s = L_s: every token is its own centroid, objective zero."""
    kv, idx, frac = _compare_kmeans(R, 1, 1, 68 + 200, 3, seed=4)
    assert frac == 1.0
    assert float(idx.objective.abs().max()) == 0.0
    _check_layout(R, kv, idx, 8192, 512)


def test_kmeans_zero_iterations(R):
    """T = 0: labels are the assignment to the seeds, centroids the seeds."""
    kv, idx, frac = _compare_kmeans(R, 1, 1, 68 + 3000, 0, seed=5)


def test_kmeans_short_context_all_steady(R):
    dev = torch.device("cuda:0")
    kv = S.make_kv(1, 2, 50, seed=6)
    cfg = R.IndexConfig.make(1, 2, 4, 50)
    idx = R.build_index(kv.K.to(dev), kv.V.to(dev), cfg)
    torch.cuda.synchronize()
    assert torch.equal(idx.Ks.cpu(), kv.K) and torch.equal(idx.Vs.cpu(), kv.V)
    assert idx.offsets.cpu().tolist() == [[[0], [0]]]


def test_kmeans_invalid_seed_positions_flagged(R):
    """Out-of-range seed positions are clamped on the device and reported in
    the status word (no out-of-bounds access)."""
    dev = torch.device("cuda:0")
    N = 68 + 2000
    kv = S.make_kv(1, 1, N, seed=7)
    ip = _seeds(1, 1, N)
    ip[0, 0, 3] = 5000
    ip[0, 0, 7] = -2
    cfg = R.IndexConfig.make(1, 1, 4, N, iters=2)
    idx = R.build_index(kv.K.to(dev), kv.V.to(dev), cfg, init_pos=torch.from_numpy(ip).to(dev))
    assert R.read_device_status(idx._build_ws) == R.STATUS_CODES["RI_ERR_INVALID_ARG"]


def test_kmeans_llama_128k_full_size_sampled(R):
    """Index build at full size (8 KV heads x 128K tokens, 16 segments of 512
    clusters, 10 iterations); the oracle re-runs a sample of (head, segment)
    units, including a short last segment."""
    kv, idx, frac = _compare_kmeans(R, 1, 8, 131072, 10, seed=8,
                                    sample_units=[0, 37, 127, 15])
    # structural invariants on every unit
    counts = idx.counts.cpu().long()
    assert int(counts.sum()) == 8 * (131072 - 68)
    assert (idx.offsets.cpu()[..., -1] == 131072 - 68).all()


def test_build_then_decode_end_to_end(R):
    """Device-built index decoded on the device vs oracle index decoded by the
    oracle (k-means differences included, so only the output bar applies)."""
    dev = torch.device("cuda:0")
    B, H, G, N = 1, 2, 4, 20000
    kv = S.make_kv(B, H, N, seed=9)
    q = S.make_queries(kv, G, seed=10)
    ip = _seeds(B, H, N, seed=11)
    cfg = R.IndexConfig.make(B, H, G, N, iters=10)
    idx = R.build_index(kv.K.to(dev), kv.V.to(dev), cfg, init_pos=torch.from_numpy(ip).to(dev))
    out, lse, sel = R.decode(q.to(dev), idx)
    heads = U.oracle_index_heads(kv, cfg_iters=10, init_pos=ip)
    k_r, k_e = O.default_budgets(heads[0][0]["C"])
    ora = O.decode(q.double().numpy(), heads, k_r, k_e)
    U.compare_output(out, ora["out"])
