"""Seeded synthetic inputs shaped like the wave-index workloads.

This module only draws random numbers; it holds none of the method's
arithmetic, so both the oracle side and the CUDA side of every test and
benchmark can take their inputs from it.

Recipe (one independent stream per (sequence, KV head), numpy PCG64 seeded
through ``SeedSequence(seed).spawn``):

* 512 planted centres ~ N(0, I_128);
* key i = centre[c_i] + N(0, 0.3^2) per element, c_i uniform over the centres;
* 8 outlier positions chosen uniformly without replacement over the whole
  context; the key there is multiplied by 4;
* values ~ N(0, 1);
* each query head: 0.7 * centre[uniform] + N(0, 0.3^2);
* query drift between consecutive decode steps: + N(0, 0.05^2) per element;
* k-means seeding: per segment, K_s distinct positions drawn without
  replacement.

Everything is drawn in fp32 and rounded to bf16 (round to nearest even) by
``torch.Tensor.to(torch.bfloat16)``; the bf16 tensors are the inputs of both
sides.  The planted component of every key is returned too, so a valid index
can be formed without running k-means (used for large decode parity cases).
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

N_CENTRES = 512
KEY_NOISE = 0.3
N_OUTLIERS = 8
OUTLIER_SCALE = 4.0
QUERY_CENTRE_WEIGHT = 0.7
QUERY_NOISE = 0.3
QUERY_DRIFT = 0.05


@dataclasses.dataclass
class KVHeads:
    """Keys/values for B sequences x H_kv heads, bf16 on the host."""

    K: torch.Tensor          # bf16 [B][H_kv][N][d]
    V: torch.Tensor          # bf16 [B][H_kv][N][d]
    component: np.ndarray    # int32 [B][H_kv][N]  planted centre of each key
    centres: np.ndarray      # fp32 [B][H_kv][N_CENTRES][d]


def _streams(seed: int, n: int) -> list[np.random.Generator]:
    return [np.random.Generator(np.random.PCG64(s))
            for s in np.random.SeedSequence(seed).spawn(n)]


def make_kv(batch: int, num_kv_heads: int, seq_len: int, head_dim: int = 128,
            seed: int = 0, n_centres: int = N_CENTRES) -> KVHeads:
    """Mixture-of-Gaussians keys with outliers, Gaussian values."""
    B, H, N, d = batch, num_kv_heads, seq_len, head_dim
    K = torch.empty((B, H, N, d), dtype=torch.bfloat16)
    V = torch.empty((B, H, N, d), dtype=torch.bfloat16)
    comp = np.empty((B, H, N), dtype=np.int32)
    centres = np.empty((B, H, n_centres, d), dtype=np.float32)
    for u, rng in enumerate(_streams(seed, B * H)):
        b, h = divmod(u, H)
        c = rng.standard_normal((n_centres, d), dtype=np.float32)
        lab = rng.integers(0, n_centres, size=N, dtype=np.int64)
        k = c[lab]
        k += KEY_NOISE * rng.standard_normal((N, d), dtype=np.float32)
        n_out = min(N_OUTLIERS, N)
        if n_out:
            pos = rng.choice(N, size=n_out, replace=False)
            k[pos] *= OUTLIER_SCALE
        v = rng.standard_normal((N, d), dtype=np.float32)
        K[b, h] = torch.from_numpy(k).to(torch.bfloat16)
        V[b, h] = torch.from_numpy(v).to(torch.bfloat16)
        comp[b, h] = lab.astype(np.int32)
        centres[b, h] = c
    return KVHeads(K=K, V=V, component=comp, centres=centres)


def make_queries(kv: KVHeads, group_size: int, seed: int = 1) -> torch.Tensor:
    """One decode query per q head: bf16 [B][H_kv*G][d].

    Query head h_q belongs to KV head h_q // G (consecutive q heads share a
    KV head)."""
    B, H, n_c, d = kv.centres.shape
    q = np.empty((B, H * group_size, d), dtype=np.float32)
    for u, rng in enumerate(_streams(seed, B * H)):
        b, h = divmod(u, H)
        for g in range(group_size):
            j = int(rng.integers(0, n_c))
            q[b, h * group_size + g] = (QUERY_CENTRE_WEIGHT * kv.centres[b, h, j]
                                        + QUERY_NOISE * rng.standard_normal(d, dtype=np.float32))
    return torch.from_numpy(q).to(torch.bfloat16)


def drift_queries(q: torch.Tensor, steps: int, seed: int = 2) -> list[torch.Tensor]:
    """Queries for `steps` consecutive decode steps, each the previous one plus
    N(0, 0.05^2) noise (the first step is `q` itself)."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed)))
    cur = q.float().numpy().copy()
    out = [q.clone()]
    for _ in range(steps - 1):
        cur = cur + QUERY_DRIFT * rng.standard_normal(cur.shape, dtype=np.float32)
        out.append(torch.from_numpy(cur).to(torch.bfloat16))
    return out


def init_positions(segment_lengths: list[int], clusters: list[int], batch: int,
                   num_kv_heads: int, seed: int = 3) -> np.ndarray:
    """Seeded k-means seeding: for every (sequence, head, segment), K_s
    distinct positions in [0, L_s) drawn without replacement, in draw order.

    Returns int32 [B][H_kv][sum(K_s)]."""
    C = int(sum(clusters))
    out = np.empty((batch, num_kv_heads, C), dtype=np.int32)
    for u, rng in enumerate(_streams(seed, batch * num_kv_heads)):
        b, h = divmod(u, num_kv_heads)
        base = 0
        for L, k in zip(segment_lengths, clusters):
            out[b, h, base:base + k] = rng.choice(L, size=k, replace=False)
            base += k
    return out


@dataclasses.dataclass
class DeviceKV:
    """Keys/values drawn on a device (large benchmark workloads)."""

    K: torch.Tensor          # bf16 [B][H_kv][N][d]
    V: torch.Tensor          # bf16 [B][H_kv][N][d]
    centres: torch.Tensor    # fp32 [B][H_kv][N_CENTRES][d]


def make_kv_device(batch: int, num_kv_heads: int, seq_len: int, device, head_dim: int = 128,
                   seed: int = 0, n_centres: int = N_CENTRES) -> DeviceKV:
    """The recipe of `make_kv` drawn with torch's generator on `device`, one
    generator per (sequence, KV head) seeded ``seed * 1_000_003 + unit``.  Same
    distributions, different numbers than `make_kv` (which draws on the host
    with numpy); used where only the shape and statistics of the workload
    matter (throughput), so multi-GB inputs take milliseconds to draw."""
    B, H, N, d = batch, num_kv_heads, seq_len, head_dim
    K = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=device)
    V = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=device)
    centres = torch.empty((B, H, n_centres, d), dtype=torch.float32, device=device)
    for u in range(B * H):
        b, h = divmod(u, H)
        g = torch.Generator(device=device)
        g.manual_seed(seed * 1_000_003 + u)
        c = torch.randn((n_centres, d), generator=g, device=device)
        lab = torch.randint(0, n_centres, (N,), generator=g, device=device)
        k = c[lab] + KEY_NOISE * torch.randn((N, d), generator=g, device=device)
        n_out = min(N_OUTLIERS, N)
        if n_out:
            pos = torch.randperm(N, generator=g, device=device)[:n_out]
            k[pos] *= OUTLIER_SCALE
        K[b, h] = k.to(torch.bfloat16)
        V[b, h] = torch.randn((N, d), generator=g, device=device).to(torch.bfloat16)
        centres[b, h] = c
    return DeviceKV(K=K, V=V, centres=centres)


def make_queries_device(kv: DeviceKV, group_size: int, seed: int = 1) -> torch.Tensor:
    """Queries of the `make_queries` recipe from a DeviceKV: bf16 [B][H_kv*G][d]."""
    B, H, n_c, d = kv.centres.shape
    g = torch.Generator(device=kv.centres.device)
    g.manual_seed(seed)
    j = torch.randint(0, n_c, (B, H, group_size), generator=g, device=kv.centres.device)
    sel = torch.gather(kv.centres, 2, j[..., None].expand(B, H, group_size, d))
    q = QUERY_CENTRE_WEIGHT * sel + QUERY_NOISE * torch.randn(
        sel.shape, generator=g, device=kv.centres.device)
    return q.reshape(B, H * group_size, d).to(torch.bfloat16)


def drift_queries_device(q: torch.Tensor, steps: int, seed: int = 2) -> list[torch.Tensor]:
    """`drift_queries` drawn on q's device."""
    g = torch.Generator(device=q.device)
    g.manual_seed(seed)
    cur = q.float()
    out = [q.clone()]
    for _ in range(steps - 1):
        cur = cur + QUERY_DRIFT * torch.randn(cur.shape, generator=g, device=q.device)
        out.append(cur.to(torch.bfloat16))
    return out
