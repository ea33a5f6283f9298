"""Index maintenance during decode on the GPU against the oracle.

"KV缓存技术与RetroInfer系统在长上下文推理中的优化实践" (framerc.cn) §2.1 item 1
(the recent window of 64 moves by one token per step) and the §2.1 pseudocode
(k-means per segment); the pages give no mechanism, the reading is the one
both sides implement (oracle.GrowingIndex, ri_index_append).

The oracle follows the GPU's prefill clustering and, at every close, the
GPU's k-means labels (checked against the oracle's own k-means on the same
tokens); every other decision is checked: each leaving token's open cluster
must be a nearest one with room (distances within 1e-5 relative), sizes
must match exactly, value sums within fp32 rounding, and decode after the
appends must match the oracle's tripartite attention at the usual bars."""
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


def _prefill_dict(idx, b, h, C0):
    return dict(perm=idx.perm[b, h].cpu().numpy().astype(np.int64),
                counts=idx.counts[b, h, :C0].cpu().numpy().astype(np.int64),
                offsets=idx.offsets[b, h, :C0 + 1].cpu().numpy().astype(np.int64),
                centroid=idx.centroid[b, h, :C0].float().cpu().numpy().astype(np.float64))


def _closed_labels(grow, b, h, first_id, K, first_pos, seg_len):
    """Labels (0..K-1) of the positions of a segment just closed on the GPU."""
    counts = grow.counts[b, h, first_id:first_id + K].cpu().numpy()
    offs = grow.offsets[b, h, first_id:first_id + K].cpu().numpy()
    perm = grow.perm[b, h].cpu().numpy()
    lab = np.full(seg_len, -1, dtype=np.int64)
    for j in range(K):
        lab[perm[offs[j]:offs[j] + counts[j]] - first_pos] = j
    assert (lab >= 0).all()
    return lab


def _check_state(grow, oracles, V64):
    B, H = grow.cfg.batch, grow.cfg.num_kv_heads
    C = grow.geom.clusters
    for b in range(B):
        for h in range(H):
            o = oracles[b][h].to_index()
            assert o["C"] == C
            np.testing.assert_array_equal(grow.counts[b, h, :C].cpu().numpy(), o["counts"])
            np.testing.assert_allclose(grow.vsum[b, h, :C].cpu().numpy().astype(np.float64),
                                       o["vsum"], rtol=1e-5, atol=1e-3)
            # the recent window: same tokens (a ring on the GPU)
            ks = grow.Ks[b, h].float().cpu().numpy()
            want = o["Ks"].astype(np.float32)
            got_rows = sorted(map(tuple, ks))
            assert got_rows == sorted(map(tuple, want))


def _decode_check(R, grow, oracles, kv_q):
    d = R.default_budgets(grow.geom.clusters)
    out, lse, sel = R.decode(kv_q, grow, d, want_sel=True)
    torch.cuda.synchronize()
    heads = [[oracles[b][h].to_index() for h in range(grow.cfg.num_kv_heads)]
             for b in range(grow.cfg.batch)]
    heads = U.as_consumed(heads)
    qd = kv_q.cpu()
    ora = O.decode(qd.double().numpy(), heads, d.k_retrieval, d.k_estimation)
    tol = U.compare_selection(sel.cpu(), ora, d.k_retrieval, d.k_estimation, qd, heads,
                              grow.cfg.group_size)
    U.compare_output(out.cpu(), ora["out"])
    np.testing.assert_allclose(lse.cpu().numpy(), ora["lse"], rtol=1e-4, atol=1e-4)
    return tol


def _run(R, B, H, G, seg_len, clusters, base_len, n_append, check_every, seed):
    dev = torch.device("cuda:0")
    cap = base_len + n_append
    kv = S.make_kv(B, H, cap, seed=seed)
    Kd, Vd = kv.K.to(dev), kv.V.to(dev)
    cfg = R.IndexConfig.make(B, H, G, base_len, seg_len=seg_len, clusters_per_seg=clusters,
                             iters=6)
    compact = R.build_index(Kd[:, :, :base_len].contiguous(), Vd[:, :, :base_len].contiguous(),
                            cfg)
    torch.cuda.synchronize()
    assert R.read_device_status(compact._build_ws) == 0
    grow = R.index_open(compact, cap)
    C0 = compact.geom.clusters
    K64, V64 = kv.K.double().numpy(), kv.V.double().numpy()
    oracles = [[O.GrowingIndex(K64[b, h], V64[b, h], base_len, iters=6, seg_len=seg_len,
                               clusters_per_seg=clusters,
                               prefill=_prefill_dict(compact, b, h, C0)) for h in range(H)]
               for b in range(B)]
    ws = R.alloc_workspace(R.index_append_workspace_bytes(grow.cfg), dev)
    assigned = torch.empty((B, H), dtype=torch.int32, device=dev)
    q = S.make_queries(kv, G, seed=seed + 1).to(dev)
    _check_state(grow, oracles, V64)
    tol = _decode_check(R, grow, oracles, q)
    closes, km_agree, km_total = 0, 0, 0
    for t in range(n_append):
        N = grow.cfg.seq_len
        g_before = (grow.geom.clusters, grow.cfg.seq_len)
        R.index_append(grow, Kd[:, :, N].contiguous(), Vd[:, :, N].contiguous(), ws, assigned)
        a = assigned.cpu().numpy()
        closing = (N + 1 - base_len) % seg_len == 0
        K_open = min(clusters, seg_len)
        for b in range(B):
            for h in range(H):
                gi = oracles[b][h]
                labels = None
                if closing:
                    first_id = g_before[0] - K_open
                    labels = _closed_labels(grow, b, h, first_id, K_open, gi.open_start, seg_len)
                    X = K64[b, h, gi.open_start:gi.open_start + seg_len]
                    own = O.kmeans(X, O.strided_init(seg_len, K_open), 6)["labels"]
                    km_agree += int((own == labels).sum())
                    km_total += seg_len
                gi.append(chosen=int(a[b, h]), close_labels=labels)
        closes += closing
        if (t + 1) % check_every == 0 or t == n_append - 1 or closing:
            assert R.read_device_status(ws) == 0
            _check_state(grow, oracles, V64)
            tol += _decode_check(R, grow, oracles, q)
    assert grow.cfg.seq_len == cap
    if km_total:
        assert km_agree >= 0.999 * km_total - 1, (km_agree, km_total)
    return closes, tol


def test_append_150_tokens_default_segments(R):
    """150 appended tokens on the default geometry (8K segments of 512
    clusters, prefill of two segments and a short one), decode checked every
    50 tokens."""
    closes, tol = _run(R, B=1, H=2, G=4, seg_len=8192, clusters=512, base_len=68 + 2 * 8192 + 700,
                       n_append=150, check_every=50, seed=71)
    assert closes == 0 and tol <= 8


def test_append_through_two_closes(R):
    """Short segments (512 tokens, 32 clusters) so the open segment closes
    twice; the prefill's last segment is short (100 tokens), so the first
    open segment follows its clusters."""
    closes, tol = _run(R, B=2, H=2, G=4, seg_len=512, clusters=32, base_len=68 + 2 * 512 + 100,
                       n_append=1100, check_every=200, seed=72)
    assert closes == 2 and tol <= 16
