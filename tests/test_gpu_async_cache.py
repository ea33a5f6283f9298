"""Asynchronous cache update against the synchronous access path, on the
million-token geometry with K/V rows in pinned host memory.

"KV缓存技术与RetroInfer系统在长上下文推理中的优化实践" (framerc.cn) §2.2: the
synchronous access path looks the clusters up and starts the copies at once;
the update path (LRU replacement, mapping table) runs on a background thread.
The two paths must serve every step the same execution buffer, so the
attention outputs are bit-identical: both sides decode the same index with the
same selection, one through ri_cache_plan, the other through a cache worker
whose admit copies run on a side stream.  At the end every cluster the
worker's cache holds resident must have its rows in the device pool."""
import numpy as np
import pytest
import torch

import synthetic as S

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def R():
    if not torch.cuda.is_available():
        pytest.skip("needs CUDA")
    import kv_cache_vector_segmented_b200 as R
    return R


@pytest.fixture(scope="module")
def setup(R):
    dev = torch.device("cuda:0")
    B, H, G, N = 1, 8, 4, 1 << 20
    kv = S.make_kv(B, H, N, seed=61)
    cfg = R.IndexConfig.make(B, H, G, N, iters=3)
    idx = R.build_index(kv.K.to(dev), kv.V.to(dev), cfg)
    torch.cuda.synchronize()
    assert R.read_device_status(idx._build_ws) == 0
    C = idx.geom.clusters
    d = R.default_budgets(C)
    hK = idx.Kp.cpu().pin_memory()
    hV = idx.Vp.cpu().pin_memory()
    counts = idx.counts.cpu().numpy().reshape(B * H, C)
    offsets = idx.offsets.cpu().numpy().reshape(B * H, C + 1)
    qs = S.drift_queries(S.make_queries(kv, G, seed=62), 10, seed=63)
    del kv
    return dict(dev=dev, B=B, H=H, G=G, cfg=cfg, idx=idx, d=d, hK=hK, hV=hV, counts=counts,
                offsets=offsets, qs=qs)


def _pool(R, s, cache):
    dev, B, H = s["dev"], s["B"], s["H"]
    cK = torch.zeros((B, H, cache.pool_rows, 128), dtype=torch.bfloat16, device=dev)
    return cK, torch.zeros_like(cK)


def _exec(s, k_r):
    rows = int(np.sort(s["counts"], axis=1)[:, ::-1][:, :k_r].sum(axis=1).max())
    eK = torch.empty((s["B"], s["H"], rows, 128), dtype=torch.bfloat16, device=s["dev"])
    return eK, torch.empty_like(eK)


def _check_pool(R, s, cache, cK, cV, br):
    """Every resident cluster's blocks hold its rows (K and V)."""
    counts, offsets = s["counts"], s["offsets"]
    hK = s["hK"].reshape(counts.shape[0], -1, 128)
    hV = s["hV"].reshape(counts.shape[0], -1, 128)
    pK = cK.reshape(counts.shape[0], -1, 128).cpu()
    pV = cV.reshape(counts.shape[0], -1, 128).cpu()
    checked = 0
    for u in range(counts.shape[0]):
        src, dst = [], []
        for c in np.nonzero(counts[u])[0]:
            blocks = cache.resident(u, int(c))
            if not blocks:
                continue
            n = int(counts[u, c])
            assert len(blocks) == -(-n // br)
            for k, b in enumerate(blocks):
                r = min(br, n - k * br)
                src.append(np.arange(offsets[u, c] + k * br, offsets[u, c] + k * br + r))
                dst.append(np.arange(b * br, b * br + r))
            checked += 1
        if src:
            si = torch.from_numpy(np.concatenate(src))
            di = torch.from_numpy(np.concatenate(dst))
            assert torch.equal(pK[u, di], hK[u, si]) and torch.equal(pV[u, di], hV[u, si])
    return checked


@pytest.mark.parametrize("fail", [False, True])
def test_async_update_equals_synchronous_path(R, setup, fail):
    s = setup
    dev, B, H, G = s["dev"], s["B"], s["H"], s["G"]
    idx, d, counts, offsets = s["idx"], s["d"], s["counts"], s["offsets"]
    k_r, C, br = d.k_retrieval, idx.geom.clusters, 8
    cap = max(1, int(0.05 * ((counts.astype(np.int64) + br - 1) // br).sum(axis=1).max()))
    sync = R.BlockCache(B * H, cap, br)
    acache = R.BlockCache(B * H, cap, br)
    sK, sV = _pool(R, s, sync)
    aK, aV = _pool(R, s, acache)
    seK, seV = _exec(s, k_r)
    aeK, aeV = _exec(s, k_r)
    ws = R.alloc_workspace(R.decode_workspace_bytes(s["cfg"], d), dev)
    gws = R.alloc_workspace(256, dev)
    wgws = R.alloc_workspace(256, dev)
    w = R.CacheWorker(acache, host_K=s["hK"], host_V=s["hV"], cache_K=aK, cache_V=aV,
                      exec_K=aeK, exec_V=aeV, gather_workspace=wgws)
    if fail:
        w.test_hooks(fail_update=4, fail_after=3)
    out_s = torch.empty((B, H * G, 128), dtype=torch.bfloat16, device=dev)
    out_a = torch.empty_like(out_s)
    lse_s = torch.empty((B, H * G), dtype=torch.float32, device=dev)
    lse_a = torch.empty_like(lse_s)
    reported, hit_rows, a_hit_rows = 0, 0, 0
    for step, q in enumerate(s["qs"]):
        qd = q.contiguous().to(dev)
        sel, _ = R.select_clusters(qd, idx, d, ws)
        sel_h = sel.cpu().numpy().reshape(B * H, -1)[:, :k_r]
        # synchronous access path
        fetch, admit, st = sync.plan(sel_h, k_r, counts, offsets)
        hit_rows += st["hit_rows"]
        for plan in (fetch, admit):
            R.gather_blocks(torch.from_numpy(plan).to(dev), s["hK"], s["hV"], seK, seV, gws, sK,
                            sV)
        R.attend_selected(qd, idx, d, ws, exec_K=seK, exec_V=seV, out=out_s, lse=lse_s)
        # lookup on the critical path, update on the worker
        try:
            fl, ast = w.lookup(sel_h, k_r, counts, offsets)
        except R.RIError as e:
            assert fail and e.status == R.STATUS_CODES["RI_ERR_HOST"] and step == 5
            reported += 1
            fl, ast = w.lookup(sel_h, k_r, counts, offsets)
        a_hit_rows += ast["hit_rows"]
        if not fail or step <= 4:
            assert ast["hit_rows"] == st["hit_rows"] and ast["miss_rows"] == st["miss_rows"]
            assert np.array_equal(fl, fetch)
        R.gather_blocks(w.fetch_to_device(), s["hK"], s["hV"], aeK, aeV, gws, aK, aV)
        w.update_async()
        R.attend_selected(qd, idx, d, ws, exec_K=aeK, exec_V=aeV, out=out_a, lse=lse_a)
        torch.cuda.synchronize()
        assert R.read_device_status(ws) == 0 and R.read_device_status(gws) == 0
        assert torch.equal(out_a, out_s) and torch.equal(lse_a, lse_s), f"step {step}"
    assert reported == (1 if fail else 0)
    assert hit_rows > 0 and a_hit_rows > 0
    w.close()
    torch.cuda.synchronize()
    assert R.read_device_status(wgws) == 0
    acache.validate()
    assert _check_pool(R, s, acache, aK, aV, br) > 0
    sync.close()
    acache.close()
