"""Full-size decode parity for the batched and the million-token workloads,
on sampled (sequence, KV head) units the oracle decodes one by one.

* Qwen2.5-7B geometry, batched decode: batch 16, 4 KV heads, GQA 7, 128K
  context, 8K segments x 512 clusters; three consecutive steps with query
  drift.
* Llama3-8B-1048K geometry: batch 1, 8 KV heads, GQA 4, 1M context
  (65 536 clusters per head, k_r = 1180, k_e = 15 073); the index's K/V rows
  live in pinned host memory behind a GPU block cache of 5 % of the blocks;
  each step selects, plans the cache, gathers the execution buffer and
  attends over it.

Both sides decode the same index (the generator's planted partition, built by
the oracle unit by unit).  Bars as everywhere: ids bit-exact except ties
within 1e-4 in score, output max-abs error <= 2e-2 x ||o||."""
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


def _index_and_samples(R, cfg, kv, dev, keep):
    idx = R.Index.empty(cfg, dev, labels=False, objective=False)
    kept = {}
    for b in range(cfg.batch):
        for h in range(cfg.num_kv_heads):
            o = U.oracle_index_unit(kv, b, h)
            U.put_unit(idx, b, h, o)
            if (b, h) in keep:
                kept[(b, h)] = U.consumed_unit(o)
            del o
    return idx, kept


def _check_units(q, sel, out, kept, G, k_r, k_e):
    tolerated = 0
    for (b, h), o in kept.items():
        qu = q[b:b + 1, h * G:(h + 1) * G]
        ora = O.decode(qu.double().numpy(), [[o]], k_r, k_e)
        tolerated += U.compare_selection(sel[b:b + 1, h:h + 1], ora, k_r, k_e, qu, [[o]], G)
        U.compare_output(out[b:b + 1, h * G:(h + 1) * G], ora["out"])
    return tolerated


def test_decode_qwen_batch16_128k(R):
    dev = torch.device("cuda:0")
    B, H, G, N = 16, 4, 7, 131072
    kv = S.make_kv(B, H, N, seed=41)
    cfg = R.IndexConfig.make(B, H, G, N)
    keep = {(0, 0), (5, 3), (11, 1), (15, 3)}
    idx, kept = _index_and_samples(R, cfg, kv, dev, keep)
    d = R.default_budgets(idx.geom.clusters)
    assert (d.k_retrieval, d.k_estimation) == (147, 1884)
    ws = R.alloc_workspace(R.decode_workspace_bytes(cfg, d), dev)
    tolerated = 0
    for q in S.drift_queries(S.make_queries(kv, G, seed=42), 3, seed=43):
        out, lse, sel = R.decode(q.contiguous().to(dev), idx, d, workspace=ws, want_sel=True)
        torch.cuda.synchronize()
        assert R.read_device_status(ws) == 0
        tolerated += _check_units(q, sel.cpu(), out.cpu(), kept, G, d.k_retrieval,
                                  d.k_estimation)
    assert tolerated <= 16


def test_decode_llama_1m_host_kv_with_block_cache(R):
    dev = torch.device("cuda:0")
    B, H, G, N = 1, 8, 4, 1 << 20
    kv = S.make_kv(B, H, N, seed=51)
    cfg = R.IndexConfig.make(B, H, G, N)
    keep = {(0, 0), (0, 6)}
    idx, kept = _index_and_samples(R, cfg, kv, dev, keep)
    del kv.K, kv.V
    C = idx.geom.clusters
    d = R.default_budgets(C)
    assert (C, d.k_retrieval, d.k_estimation) == (65536, 1180, 15073)
    k_r = d.k_retrieval
    # K/V rows to pinned host memory; the device keeps centroids, sizes, sums
    hK = idx.Kp.cpu().pin_memory()
    hV = idx.Vp.cpu().pin_memory()
    counts = idx.counts.cpu().numpy().reshape(B * H, C)
    offsets = idx.offsets.cpu().numpy().reshape(B * H, C + 1)
    br = 8
    blocks = (counts.astype(np.int64) + br - 1) // br
    cache = R.BlockCache(B * H, max(1, int(0.05 * blocks.sum(axis=1).max())), br)
    cK = torch.zeros((B, H, cache.pool_rows, 128), dtype=torch.bfloat16, device=dev)
    cV = torch.zeros_like(cK)
    exec_rows = int(np.sort(counts, axis=1)[:, ::-1][:, :k_r].sum(axis=1).max())
    eK = torch.empty((B, H, exec_rows, 128), dtype=torch.bfloat16, device=dev)
    eV = torch.empty_like(eK)
    ws = R.alloc_workspace(R.decode_workspace_bytes(cfg, d), dev)
    gws = R.alloc_workspace(256, dev)
    out = torch.empty((B, H * G, 128), dtype=torch.bfloat16, device=dev)
    tolerated, hit_rows = 0, 0
    qs = S.drift_queries(S.make_queries(kv, G, seed=52), 3, seed=53)
    for q in qs:
        qd = q.contiguous().to(dev)
        sel, rr = R.select_clusters(qd, idx, d, ws)
        fetch, admit, st = cache.plan(sel.cpu().numpy().reshape(B * H, -1), k_r, counts, offsets)
        hit_rows += st["hit_rows"]
        for plan in (fetch, admit):
            R.gather_blocks(torch.from_numpy(plan).to(dev), hK, hV, eK, eV, gws, cK, cV)
        R.attend_selected(qd, idx, d, ws, exec_K=eK, exec_V=eV, out=out)
        torch.cuda.synchronize()
        assert R.read_device_status(gws) == 0 and R.read_device_status(ws) == 0
        tolerated += _check_units(q, sel.cpu(), out.cpu(), kept, G, k_r, d.k_estimation)
    assert hit_rows > 0
    assert tolerated <= 16
    cache.close()
