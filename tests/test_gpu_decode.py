"""GPU parity of tripartite decode attention against the oracle.

Both sides decode the same index (built by the oracle, held on the device
exactly as the library stores it).  Bars: selected ids bit-exact except for
ties within 1e-4 in score; output max-abs error <= 2e-2 x ||o|| per query head
(spec tolerances, written in tests/_util.py)."""
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


def _run_case(R, B, H, G, N, k=None, iters=None, use_labels=True, seed=0, seg_len=8192,
              clusters=512, want_sel=True):
    dev = torch.device("cuda:0")
    kv = S.make_kv(B, H, N, seed=seed)
    q = S.make_queries(kv, G, seed=seed + 1)
    heads = U.oracle_index_heads(kv, cfg_iters=iters, use_labels=use_labels, seg_len=seg_len,
                                 clusters=clusters)
    cfg = R.IndexConfig.make(B, H, G, N, seg_len=seg_len, clusters_per_seg=clusters)
    idx = U.to_device_index(R, cfg, heads, dev)
    C = idx.geom.clusters
    dcfg = R.default_budgets(C) if k is None else R.DecodeConfig(*k)
    out, lse, sel = R.decode(q.to(dev), idx, dcfg, want_sel=want_sel)
    torch.cuda.synchronize()
    cons = U.as_consumed(heads)
    ora = O.decode(q.double().numpy(), cons, dcfg.k_retrieval, dcfg.k_estimation)
    tol = U.compare_selection(sel, ora, dcfg.k_retrieval, dcfg.k_estimation, q, cons, G) \
        if want_sel and C else 0
    worst = U.compare_output(out, ora["out"])
    np.testing.assert_allclose(lse.cpu().numpy(), ora["lse"], rtol=1e-4, atol=1e-4)
    return dict(out=out, lse=lse, sel=sel, ora=ora, tolerated=tol, worst=worst, idx=idx, q=q,
                dcfg=dcfg, cfg=cfg)


def test_decode_single_segment_kmeans_index(R):
    """8K context, one KV head, GQA group of 4, index from 10 Lloyd iterations."""
    r = _run_case(R, 1, 1, 4, 8192, iters=10, use_labels=False)
    assert r["tolerated"] <= 2


@pytest.mark.parametrize("B,H,G,N", [(2, 3, 7, 2 * 8192 + 68 + 1000), (1, 2, 1, 8192 + 68 + 5),
                                     (3, 1, 8, 8192 + 300), (1, 1, 2, 68 + 700)])
def test_decode_ragged_multihead(R, B, H, G, N):
    r = _run_case(R, B, H, G, N, use_labels=True, seed=B * 100 + N % 97)
    assert r["tolerated"] <= 4


@pytest.mark.parametrize("N", [1, 5, 50, 68])
def test_decode_all_steady(R, N):
    """N <= 68: no index, exact attention over every token."""
    _run_case(R, 1, 2, 4, N, use_labels=True, want_sel=False)


def test_decode_one_middle_token(R):
    _run_case(R, 1, 1, 4, 69, use_labels=True)


def test_decode_small_segments(R):
    """Non-default segmentation: 300-token segments of 64 clusters."""
    _run_case(R, 2, 2, 4, 68 + 1000, use_labels=True, seg_len=300, clusters=64, seed=31)


@pytest.mark.parametrize("k", [(0, 0), (0, 1000), (1000, 0), (17, 100000), (600, 600)])
def test_decode_budget_edges(R, k):
    """Steady only; estimation only; retrieval only (full attention when it
    covers every cluster); budgets past C (clamped)."""
    _run_case(R, 1, 2, 4, 8192 + 68 + 2000, k=k, use_labels=True, seed=7)


def test_decode_full_retrieval_is_full_attention(R):
    dev = torch.device("cuda:0")
    kv = S.make_kv(1, 2, 9000, seed=11)
    q = S.make_queries(kv, 4, seed=12)
    heads = U.oracle_index_heads(kv, use_labels=True)
    cfg = R.IndexConfig.make(1, 2, 4, 9000)
    idx = U.to_device_index(R, cfg, heads, dev)
    C = idx.geom.clusters
    out, lse, _ = R.decode(q.to(dev), idx, R.DecodeConfig(C, 0))
    Kf = kv.K.to(dev).float()
    Vf = kv.V.to(dev).float()
    qf = q.to(dev).float().view(1, 2, 4, 128)
    ref = torch.nn.functional.scaled_dot_product_attention(qf.unsqueeze(3), Kf.unsqueeze(2),
                                                           Vf.unsqueeze(2)).squeeze(3)
    ref = ref.reshape(1, 8, 128)
    err = (out.float() - ref).abs().amax(-1)
    assert (err <= U.OUT_TOL * ref.norm(dim=-1)).all()


def test_decode_with_empty_clusters(R):
    dev = torch.device("cuda:0")
    kv = S.make_kv(1, 1, 8192 + 68 + 500, seed=21)
    q = S.make_queries(kv, 4, seed=22)
    N = kv.K.shape[2]
    m0, M = O.middle_range(N)
    lab = kv.component[0, 0, m0:m0 + M] % 200          # clusters 200.. empty in segment 0
    Kh, Vh = kv.K[0, 0].double().numpy(), kv.V[0, 0].double().numpy()
    heads = [[O.index_from_labels(Kh, Vh, lab)]]
    cfg = R.IndexConfig.make(1, 1, 4, N)
    idx = U.to_device_index(R, cfg, heads, dev)
    for k in [(150, 200), (300, 300)]:
        d = R.DecodeConfig(*k)
        out, lse, sel = R.decode(q.to(dev), idx, d, want_sel=True)
        ora = O.decode(q.double().numpy(), U.as_consumed(heads), *k)
        U.compare_selection(sel, ora, *k, q, U.as_consumed(heads), 4)
        U.compare_output(out, ora["out"])


def test_decode_llama_128k_full_size(R):
    """Llama-3.1-8B geometry at 128K context (8 KV heads, GQA 4), the size the
    benchmark times; index from the generator's planted partition."""
    r = _run_case(R, 1, 8, 4, 131072, use_labels=True, seed=3)
    assert r["tolerated"] <= 8
    fr = [(len(r["ora"]["R"][0][h]), len(r["ora"]["E"][0][h])) for h in range(8)]
    assert all(x == (147, 1884) for x in fr)


def test_decode_is_deterministic(R):
    dev = torch.device("cuda:0")
    kv = S.make_kv(2, 2, 20000, seed=5)
    q = S.make_queries(kv, 4, seed=6).to(dev)
    heads = U.oracle_index_heads(kv, use_labels=True)
    cfg = R.IndexConfig.make(2, 2, 4, 20000)
    idx = U.to_device_index(R, cfg, heads, dev)
    a = R.decode(q, idx, want_sel=True)
    b = R.decode(q, idx, want_sel=True)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])


def test_select_then_attend_equals_decode(R):
    """The split calls (S1-S2, then S4-S6 in place or from a packed execution
    buffer) reproduce the one-call decode bit for bit."""
    dev = torch.device("cuda:0")
    kv = S.make_kv(1, 2, 30000, seed=8)
    q = S.make_queries(kv, 4, seed=9).to(dev)
    heads = U.oracle_index_heads(kv, use_labels=True)
    cfg = R.IndexConfig.make(1, 2, 4, 30000)
    idx = U.to_device_index(R, cfg, heads, dev)
    d = R.default_budgets(idx.geom.clusters)
    ref_out, ref_lse, ref_sel = R.decode(q, idx, d, want_sel=True)
    ws = R.alloc_workspace(R.decode_workspace_bytes(cfg, d), dev)
    sel, rows = R.select_clusters(q, idx, d, ws)
    assert torch.equal(sel, ref_sel)
    lse = torch.empty_like(ref_lse)
    out, _ = R.attend_selected(q, idx, d, ws, lse=lse)
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
    # pack the retrieval clusters' rows into execution buffers (torch copies;
    # the library's gather kernel is tested separately)
    tot = int(rows[:, :, -1].max())
    exK = torch.zeros((1, 2, tot + 3, 128), dtype=torch.bfloat16, device=dev)
    exV = torch.zeros_like(exK)
    for h in range(2):
        for i, c in enumerate(sel[0, h, :d.k_retrieval].tolist()):
            o, n = int(idx.offsets[0, h, c]), int(idx.counts[0, h, c])
            r0 = int(rows[0, h, i])
            exK[0, h, r0:r0 + n] = idx.Kp[0, h, o:o + n]
            exV[0, h, r0:r0 + n] = idx.Vp[0, h, o:o + n]
    out2, _ = R.attend_selected(q, idx, d, ws, exec_K=exK, exec_V=exV)
    assert torch.equal(out2, ref_out)


def test_decoder_host_buffers_equal_device_call(R):
    """Decoder.step_host (ri_decode_attention_host: query and output in
    page-locked host memory, copies and the wait inside the call) returns
    the device call's output bit for bit, step after step."""
    dev = torch.device("cuda:0")
    kv = S.make_kv(1, 2, 30000, seed=18)
    heads = U.oracle_index_heads(kv, use_labels=True)
    cfg = R.IndexConfig.make(1, 2, 4, 30000)
    idx = U.to_device_index(R, cfg, heads, dev)
    dec = R.Decoder(idx)
    o_host = torch.empty((1, 8, 128), dtype=torch.bfloat16).pin_memory()
    for seed in (19, 20, 21):
        q = S.make_queries(kv, 4, seed=seed)
        ref, _ = dec(q.to(dev))
        ref = ref.cpu()
        got = dec.step_host(q.pin_memory(), o_host)
        assert got is o_host and torch.equal(o_host, ref)
    assert R.read_device_status(dec.ws) == 0


def test_wait_timeout_selftest_reports_status(R):
    dev = torch.device("cuda:0")
    ws = R.alloc_workspace(1024, dev)
    R.selftest_wait_timeout(ws, 20_000_000)  # 20 ms
    assert R.read_device_status(ws) == R.STATUS_CODES["RI_ERR_TIMEOUT"]
    # the context is still healthy
    x = torch.ones(4, device=dev)
    assert float(x.sum()) == 4.0


# ---------------------------------------------------------------- selection
def _decode_index(R, heads, B, H, G, N, seg_len=8192, clusters=512):
    dev = torch.device("cuda:0")
    cfg = R.IndexConfig.make(B, H, G, N, seg_len=seg_len, clusters_per_seg=clusters)
    return U.to_device_index(R, cfg, heads, dev)


def test_decode_heavy_ties_are_broken_by_id(R):
    """Every centroid equal: all selection keys tie exactly on both sides,
    so R must be the k_r lowest ids and E the next k_e, bit for bit.  More
    than 256 keys share the boundary bucket, which takes the radix walk over
    the order key and the per-block id count."""
    dev = torch.device("cuda:0")
    kv = S.make_kv(1, 2, 3 * 8192 + 68, seed=41)
    q = S.make_queries(kv, 4, seed=42)
    heads = U.oracle_index_heads(kv, use_labels=True)
    for o in heads[0]:
        o["centroid"][:] = o["centroid"][0]
    idx = _decode_index(R, heads, 1, 2, 4, kv.K.shape[2])
    for k in [(147, 300), (0, 700), (1000, 200), (5, 1531)]:
        d = R.DecodeConfig(*k)
        out, lse, sel = R.decode(q.to(dev), idx, d, want_sel=True)
        ora = O.decode(q.double().numpy(), U.as_consumed(heads), *k)
        for h in range(2):
            C = heads[0][h]["C"]
            kr = min(k[0], C)
            ke = min(k[1], C - kr)
            live = np.flatnonzero(heads[0][h]["counts"] > 0)
            order = np.concatenate([live, np.flatnonzero(heads[0][h]["counts"] == 0)])
            assert sel[0, h, :kr].tolist() == sorted(order[:kr].tolist())
            assert sel[0, h, k[0]:k[0] + ke].tolist() == sorted(order[kr:kr + ke].tolist())
        U.compare_output(out, ora["out"])
        np.testing.assert_allclose(lse.cpu().numpy(), ora["lse"], rtol=1e-4, atol=1e-4)


def test_decode_zero_query_selects_lowest_ids(R):
    """q = 0: every score is exactly 0, the selection is the lowest ids and
    the output is the plain average of the attended values."""
    dev = torch.device("cuda:0")
    kv = S.make_kv(1, 1, 2 * 8192 + 500, seed=43)
    q = torch.zeros((1, 4, 128), dtype=torch.bfloat16)
    heads = U.oracle_index_heads(kv, use_labels=True)
    idx = _decode_index(R, heads, 1, 1, 4, kv.K.shape[2])
    d = R.default_budgets(idx.geom.clusters)
    out, lse, sel = R.decode(q.to(dev), idx, d, want_sel=True)
    ora = O.decode(q.double().numpy(), U.as_consumed(heads), d.k_retrieval, d.k_estimation)
    assert U.compare_selection(sel, ora, d.k_retrieval, d.k_estimation, q, U.as_consumed(heads),
                               4) == 0
    U.compare_output(out, ora["out"])


@pytest.mark.parametrize("B,H,G,N", [(5, 4, 4, 9000),     # 20 units
                                     (8, 8, 4, 5000),     # 64 units: small clusters of blocks
                                     (10, 16, 2, 3000),   # 160 units: more than one wave
                                     (1, 1, 8, 40000)])   # one unit, every block of a cluster
def test_decode_cluster_shapes(R, B, H, G, N):
    """Unit counts that give different thread-block cluster sizes (and more
    units than clusters resident at once)."""
    r = _run_case(R, B, H, G, N, use_labels=True, seed=B * 7 + H, clusters=256 if N < 9000 else 512)
    assert r["tolerated"] <= B * H


# ---------------------------------------------------------------- bounded waits
@pytest.mark.parametrize("hand_off", [1, 2, 3])
def test_decode_kernel_wait_expires_and_reports_timeout(R, hand_off):
    """One hand-off inside the decode kernel never released (a tile copy, an
    MMA completion, the cluster sizes beside the scoring) with a 2 ms limit: the kernel
    records RI_ERR_TIMEOUT and returns, and the next normal call on the same
    workspace and context gives the oracle's answer."""
    dev = torch.device("cuda:0")
    kv = S.make_kv(1, 2, 8192 + 68 + 3000, seed=44)
    q = S.make_queries(kv, 4, seed=45)
    heads = U.oracle_index_heads(kv, use_labels=True)
    idx = _decode_index(R, heads, 1, 2, 4, kv.K.shape[2])
    d = R.default_budgets(idx.geom.clusters)
    ws = R.alloc_workspace(R.decode_workspace_bytes(idx.cfg, d), dev)
    R.selftest_decode_timeout(q.to(dev), idx, d, ws, hand_off, 2_000_000)
    assert R.read_device_status(ws) == R.STATUS_CODES["RI_ERR_TIMEOUT"]
    out, lse, sel = R.decode(q.to(dev), idx, d, workspace=ws, want_sel=True)
    assert R.read_device_status(ws) == 0
    ora = O.decode(q.double().numpy(), U.as_consumed(heads), d.k_retrieval, d.k_estimation)
    U.compare_output(out, ora["out"])
