"""Helpers shared by the tests: oracle index <-> device tensors, id comparison
with the tie tolerance, and standard configurations."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle as O
import synthetic as S

# Parity bars (spec tolerances).
OUT_TOL = 2e-2        # max-abs error <= OUT_TOL * ||o_oracle||_2 per query head
ID_TIE_TOL = 1e-4     # selection mismatches only between keys this close (absolute)
ASSIGN_AGREE = 0.999  # k-means assignments identical
OBJ_RTOL = 1e-3       # k-means objective


def oracle_index_heads(kv: S.KVHeads, cfg_iters=None, init_pos=None, use_labels=False,
                       seg_len=8192, clusters=512):
    """Oracle index for every (b, h): k-means (iters given) or planted labels."""
    B, H, N, d = kv.K.shape
    heads = []
    for b in range(B):
        row = []
        for h in range(H):
            Kh = kv.K[b, h].double().numpy()
            Vh = kv.V[b, h].double().numpy()
            if use_labels:
                m0, M = O.middle_range(N)
                comp = kv.component[b, h, m0:m0 + M].astype(np.int64)
                # planted component, folded into each segment's cluster range
                lab = np.empty(M, dtype=np.int64)
                for start, L, Ks in O.segments(M, seg_len, clusters):
                    lab[start:start + L] = comp[start:start + L] % Ks
                row.append(O.index_from_labels(Kh, Vh, lab, seg_len, clusters))
            else:
                ip = None if init_pos is None else init_pos[b, h]
                row.append(O.build_index_head(Kh, Vh, ip, iters=cfg_iters, seg_len=seg_len,
                                              clusters_per_seg=clusters))
        heads.append(row)
    return heads


def oracle_index_unit(kv: S.KVHeads, b: int, h: int, seg_len=8192, clusters=512):
    """Oracle index of one (sequence, KV head) from the generator's planted
    labels (folded into each segment's cluster range)."""
    N = kv.K.shape[2]
    Kh = kv.K[b, h].double().numpy()
    Vh = kv.V[b, h].double().numpy()
    m0, M = O.middle_range(N)
    comp = kv.component[b, h, m0:m0 + M].astype(np.int64)
    lab = np.empty(M, dtype=np.int64)
    for start, L, Ks in O.segments(M, seg_len, clusters):
        lab[start:start + L] = comp[start:start + L] % Ks
    return O.index_from_labels(Kh, Vh, lab, seg_len, clusters)


def put_unit(idx, b: int, h: int, o) -> None:
    """Writes one unit of an oracle index into a device Index."""
    g = idx.geom
    if g.middle:
        idx.Kp[b, h] = torch.from_numpy(o["Kp"]).to(torch.bfloat16)
        idx.Vp[b, h] = torch.from_numpy(o["Vp"]).to(torch.bfloat16)
        idx.perm[b, h] = torch.from_numpy(o["perm"].astype(np.int32))
        idx.centroid[b, h] = torch.from_numpy(o["centroid"]).to(torch.bfloat16)
        idx.counts[b, h] = torch.from_numpy(o["counts"].astype(np.int32))
        idx.vsum[b, h] = torch.from_numpy(o["vsum"]).float()
    idx.offsets[b, h] = torch.from_numpy(o["offsets"].astype(np.int32))
    idx.Ks[b, h] = torch.from_numpy(o["Ks"]).to(torch.bfloat16)
    idx.Vs[b, h] = torch.from_numpy(o["Vs"]).to(torch.bfloat16)


def consumed_unit(o):
    """One unit of the oracle index as the device holds it (vsum in fp32)."""
    o2 = dict(o)
    o2["vsum"] = o["vsum"].astype(np.float32).astype(np.float64)
    return o2


def to_device_index(R, cfg, heads, device):
    """Device Index holding the oracle's index (bf16 / fp32 / int32 exactly as
    the library stores them)."""
    idx = R.Index.empty(cfg, device, labels=False, objective=False)
    B, H = cfg.batch, cfg.num_kv_heads
    g = idx.geom
    for b in range(B):
        for h in range(H):
            o = heads[b][h]
            if g.middle:
                idx.Kp[b, h] = torch.from_numpy(o["Kp"]).to(torch.bfloat16)
                idx.Vp[b, h] = torch.from_numpy(o["Vp"]).to(torch.bfloat16)
                idx.perm[b, h] = torch.from_numpy(o["perm"].astype(np.int32))
                idx.centroid[b, h] = torch.from_numpy(o["centroid"]).to(torch.bfloat16)
                idx.counts[b, h] = torch.from_numpy(o["counts"].astype(np.int32))
                idx.vsum[b, h] = torch.from_numpy(o["vsum"]).float()
            idx.offsets[b, h] = torch.from_numpy(o["offsets"].astype(np.int32))
            idx.Ks[b, h] = torch.from_numpy(o["Ks"]).to(torch.bfloat16)
            idx.Vs[b, h] = torch.from_numpy(o["Vs"]).to(torch.bfloat16)
    return idx


def as_consumed(heads):
    """The oracle's index with vsum rounded to fp32, exactly what the device
    index holds, so both sides decode the same numbers."""
    out = []
    for row in heads:
        r2 = []
        for o in row:
            o2 = dict(o)
            o2["vsum"] = o["vsum"].astype(np.float32).astype(np.float64)
            r2.append(o2)
        out.append(r2)
    return out


def compare_selection(sel_gpu, ora, k_r, k_e, q, heads, G):
    """Selection ids: bit-exact except for ties within ID_TIE_TOL in score.
    Returns the number of tolerated mismatches."""
    tolerated = 0
    B, H = len(heads), len(heads[0])
    for b in range(B):
        for h in range(H):
            o = heads[b][h]
            C = o["C"]
            kr = min(k_r, C)
            ke = min(k_e, C - kr)
            s = (q[b, h * G:(h + 1) * G].double().numpy() @ o["centroid"].T) / math.sqrt(128)
            r = np.where(o["counts"] > 0, s.sum(0), -np.inf)
            order = np.lexsort((np.arange(C), -r))
            Rg = sel_gpu[b, h, :k_r].cpu().numpy()
            Eg = sel_gpu[b, h, k_r:k_r + k_e].cpu().numpy()
            assert (Rg[kr:] == -1).all() and (Eg[ke:] == -1).all()
            Rg, Eg = Rg[:kr], Eg[:ke]
            assert (np.diff(Rg) > 0).all() and (np.diff(Eg) > 0).all(), "ids not sorted"
            Ro, Eo = ora["R"][b][h], ora["E"][b][h]
            for got, want, k in ((set(Rg), set(Ro), kr), (set(Rg) | set(Eg), set(Ro) | set(Eo), kr + ke)):
                diff = got ^ want
                if diff and k > 0:
                    t = r[order[k - 1]]
                    tol = ID_TIE_TOL if np.isfinite(t) else 0.0
                    for c in diff:
                        assert abs(r[c] - t) <= tol or (r[c] == t), \
                            f"(b={b},h={h}) cluster {c} r={r[c]} vs boundary {t}"
                    tolerated += len(diff)
    return tolerated


def compare_output(out_gpu, out_ora):
    o = out_gpu.float().cpu().numpy().astype(np.float64)
    ref = np.asarray(out_ora)
    err = np.abs(o - ref).max(axis=-1)
    norm = np.linalg.norm(ref, axis=-1)
    worst = float((err / np.maximum(norm, 1e-30)).max())
    assert (err <= OUT_TOL * norm).all(), f"max err / ||o|| = {worst}"
    return worst
