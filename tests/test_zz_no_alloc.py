"""ri_decode_attention_static (scratch in the library's fixed device array)
against ri_decode_attention (caller workspace).

Both run the same kernel on the same inputs, so results must be identical bit
for bit.  Two calls in a row with different queries check that the shared
scratch carries nothing from one call into the next.  This file is collected
last on purpose: the static path must also give the same answers after every
other test has run in the process."""
import ctypes

import pytest
import torch

import oracle as O
import synthetic as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def R():
    if not torch.cuda.is_available():
        pytest.skip("needs CUDA")
    import kv_cache_vector_segmented_b200 as R
    return R


def _index(R, B, H, G, N, seed):
    dev = torch.device("cuda:0")
    kv = S.make_kv(B, H, N, seed=seed)
    m0, M = O.middle_range(N)
    segs = O.segments(M, 8192, 512)
    ip = S.init_positions([s[1] for s in segs], [s[2] for s in segs], B, H, seed=seed + 1)
    cfg = R.IndexConfig.make(B, H, G, N, iters=4)
    idx = R.build_index(kv.K.to(dev), kv.V.to(dev), cfg, init_pos=torch.from_numpy(ip).to(dev))
    q0 = S.make_queries(kv, G, seed=seed + 2)
    q1 = S.drift_queries(q0, 2, seed=seed + 3)[-1]
    return idx, [q0.to(dev), q1.contiguous().to(dev)]


@pytest.mark.parametrize("B,H,G,N", [(1, 2, 4, 20000),     # three segments, ragged tail
                                     (1, 8, 4, 131072)])   # Llama-3-8B geometry, 128K
def test_static_matches_workspace_two_calls(R, B, H, G, N):
    idx, qs = _index(R, B, H, G, N, seed=21)
    dcfg = R.default_budgets(idx.geom.clusters)
    assert R.decode_workspace_bytes(idx.cfg, dcfg) <= R.STATIC_SCRATCH_BYTES
    status = torch.full((1,), -1, dtype=torch.int32, device=qs[0].device)
    for q in qs:  # two calls in a row through the same static scratch
        o_s, l_s, s_s = R.decode_static(q, idx, dcfg, want_sel=True, device_status=status)
        o_w, l_w, s_w = R.decode(q, idx, dcfg, want_sel=True)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(s_s, s_w)
        assert torch.equal(o_s, o_w)
        assert torch.equal(l_s, l_w)


def test_static_rejects_oversize(R):
    """Batch 16 x 4 KV heads at 128K needs 18 MiB of scratch: refused on the
    host with RI_ERR_CAPACITY before any pointer is looked at or any launch."""
    cfg = R.IndexConfig.make(16, 4, 7, 131072)
    dcfg = R.default_budgets(R.geometry(cfg).clusters)
    assert R.decode_workspace_bytes(cfg, dcfg) > R.STATIC_SCRATCH_BYTES
    cidx = R.CIndex()
    st = R.lib.ri_decode_attention_static(ctypes.byref(cfg), ctypes.byref(dcfg), None,
                                          ctypes.byref(cidx), None, None, None, None, None)
    assert st == R.STATUS_CODES["RI_ERR_CAPACITY"]
