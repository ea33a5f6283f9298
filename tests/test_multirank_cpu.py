"""World-size-2 gloo run of the multi-rank host logic on CPU: unit sharding
covers every (sequence, KV head) once, the timing reduction is the max over
ranks, and every rank's oracle shard equals the same units of a one-process
run (the path needs no exchange between ranks)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from kv_cache_vector_segmented_b200.shard import max_over_ranks, shard_range, sum_over_ranks


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle as O
        import synthetic as S
        B, H, G, N = 3, 1, 4, 68 + 700
        b0, b1 = shard_range(B, rank, world)
        # every rank generates the full (seeded) batch and decodes its shard
        kv = S.make_kv(B, H, N, seed=0)
        q = S.make_queries(kv, G, seed=1).double().numpy()
        outs = {}
        for b in range(b0, b1):
            idx = O.build_index_head(kv.K[b, 0].double().numpy(), kv.V[b, 0].double().numpy(),
                                     None, iters=2)
            k_r, k_e = O.default_budgets(idx["C"])
            outs[b] = O.tripartite_attention(q[b, :G], idx, k_r, k_e)["out"]
        covered = sum_over_ranks([1.0 if b0 <= b < b1 else 0.0 for b in range(B)])
        t = max_over_ranks([10.0 + rank, 5.0 - rank])
        results[rank] = (b0, b1, covered, t, {b: o.tolist() for b, o in outs.items()})
    finally:
        dist.destroy_process_group()


def test_two_rank_sharding_and_max_timing():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, results), nprocs=2, join=True,
                       start_method="spawn")
    r0, r1 = results[0], results[1]
    assert (r0[0], r0[1], r1[0], r1[1]) == (0, 1, 1, 3)
    assert r0[2] == [1.0, 1.0, 1.0]
    assert r0[3] == r1[3] == [11.0, 5.0]
    # shards agree with a single-process run of the same units
    import oracle as O
    import synthetic as S
    kv = S.make_kv(3, 1, 768, seed=0)
    q = S.make_queries(kv, 4, seed=1).double().numpy()
    for r in (r0, r1):
        for b, o in r[4].items():
            idx = O.build_index_head(kv.K[b, 0].double().numpy(), kv.V[b, 0].double().numpy(),
                                     None, iters=2)
            k_r, k_e = O.default_budgets(idx["C"])
            ref = O.tripartite_attention(q[b, :4], idx, k_r, k_e)["out"]
            np.testing.assert_array_equal(np.array(o), ref)


@pytest.mark.parametrize("n,w", [(1, 1), (7, 3), (64, 8), (5, 8)])
def test_shard_range_partitions(n, w):
    seen = []
    for r in range(w):
        a, b = shard_range(n, r, w)
        seen.extend(range(a, b))
        assert 0 <= b - a - n // w <= 1
    assert seen == list(range(n))
