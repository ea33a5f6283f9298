"""Multi-GPU plumbing of the wave-index path: one process per GPU.

The path is data parallel over independent units (sequence, KV head); no
step exchanges data between units, so a multi-GPU run gives each rank a
contiguous share of the units (or, for the benchmark, a full replica of the
workload) and needs collectives only for timing: the step time of a run is
the maximum over ranks.
"""
from __future__ import annotations

import torch


def shard_range(n_units: int, rank: int, world: int) -> tuple[int, int]:
    """[begin, end) of the units owned by `rank`: contiguous, disjoint,
    covering [0, n_units), sizes differing by at most one."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} of {world}")
    return n_units * rank // world, n_units * (rank + 1) // world


def max_over_ranks(values, device=None) -> list[float]:
    """Element-wise maximum over all ranks (identity without a process group)."""
    vals = [float(v) for v in values]
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def sum_over_ranks(values, device=None) -> list[float]:
    vals = [float(v) for v in values]
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return vals
    t = torch.tensor(vals, dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return t.tolist()
