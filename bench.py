#!/usr/bin/env python
"""Benchmark of the wave-index decode path on B200.

Headline: decode-attention steps/s at 128K context on the Llama-3.1-8B
geometry (batch 1, 32 query heads, 8 KV heads, head_dim 128, sixteen 8K
segments of 512 clusters; retrieval 147 and estimation 1884 clusters per KV
head), with HBM GB/s of the dominant kernel against the measured copy
bandwidth, and the segmented k-means build (8 KV heads x 128K tokens, 10
iterations) in key vectors clustered per second.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One JSON line is printed by rank 0.  Multi-GPU: one process per GPU under
torchrun; every rank runs an independent replica of the workload (the
path shards by sequence and KV head with no exchange), timing is the max
over ranks.  `--impl reference` times the fp64 CPU oracle on the host cores.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic as S  # noqa: E402

METRIC = "decode-attention steps/sec and HBM GB/s at 128K ctx (frac of peak); k-means tok/s"
UNIT = "steps/s"
B, H, G, N = 1, 8, 4, 131072
LAYERS = 32
WORKLOAD = "llama3.1-8b decode, 128K context, batch 1, 32 q / 8 kv heads, d 128"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), \
            float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1400.0, 1590.0, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle samples during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, local_rank: int):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        self.gpu = vis.split(",")[local_rank].strip() if vis else str(local_rank)
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.15)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.05)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
                power.append(float(parts[3]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(sm), "reasons": sorted(reasons)}


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def _traffic_from_profiles(kernel_src: str):
    """DRAM bytes per launch recorded by an ncu capture of the current kernel
    source (null when the kernel changed since)."""
    sha = hashlib.sha256(open(kernel_src, "rb").read()).hexdigest()[:16]
    for fn in sorted(os.listdir(os.path.join(ROOT, "profiles"))):
        if not fn.endswith(".md"):
            continue
        text = open(os.path.join(ROOT, "profiles", fn), encoding="utf-8").read()
        m = re.search(r"traffic_bytes_per_launch:\s*(\d+)\s+source_sha256_16:\s*([0-9a-f]{16})", text)
        if m and m.group(2) == sha:
            return int(m.group(1)), sha
    return None, sha


def _segment_sizes(geom, seg_len=8192, clusters=512):
    """(tokens, clusters) of each 8K segment of the middle tokens, from the
    library's own geometry (the seeded initial positions need them)."""
    M = geom.middle
    return [(min(seg_len, M - s * seg_len), min(clusters, M - s * seg_len))
            for s in range(geom.num_segments)]


# --------------------------------------------------------------------- ours
def run_ours(args, ws_n, rank, local):
    import kv_cache_vector_segmented_b200 as R
    from kv_cache_vector_segmented_b200.shard import max_over_ranks

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    hbm_peak, tf_sus, tf_burst, peak_kind = _peaks()
    cfg = R.IndexConfig.make(B, H, G, N, iters=10)
    geom = R.geometry(cfg)
    dcfg = R.default_budgets(geom.clusters)

    # ---- inputs: one 128K-token layer, seeded per rank
    kv = S.make_kv(B, H, N, seed=1000 * rank)
    M = geom.middle
    segs = _segment_sizes(geom)
    ip = S.init_positions([L for L, _ in segs], [k for _, k in segs], B, H, seed=1000 * rank + 3)
    Kd, Vd = kv.K.to(dev), kv.V.to(dev)
    ipd = torch.from_numpy(ip).to(dev)

    # ---- k-means build (config: 8 KV heads x 128K, 8K segments x 512, T=10)
    base = R.build_index(Kd, Vd, cfg, init_pos=ipd)
    torch.cuda.synchronize()
    assert R.read_device_status(base._build_ws) == 0
    build_ws = base._build_ws
    kms = []
    for _ in range(3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        R.build_index(Kd, Vd, cfg, init_pos=ipd, out=base, workspace=build_ws)
        e1.record()
        torch.cuda.synchronize()
        kms.append(e0.elapsed_time(e1))
    build_ms = statistics.median(kms)
    assign_flop = 2.0 * H * M * 512 * 128 * 10

    # ---- 32 layer instances (distinct memory, so L2 cannot hold a cycle)
    def clone_index(ix):
        f = {k: getattr(ix, k) for k in ("Kp", "Vp", "perm", "centroid", "counts", "offsets",
                                           "vsum", "Ks", "Vs")}
        return R.Index(cfg=cfg, geom=geom, **{k: v.clone() for k, v in f.items()})

    layers = [clone_index(base) for _ in range(LAYERS)]
    del Kd, Vd
    qs = [S.make_queries(kv, G, seed=1000 * rank + 10 + i).to(dev) for i in range(LAYERS)]
    wsb = R.decode_workspace_bytes(cfg, dcfg)
    wss = [R.alloc_workspace(wsb, dev) for _ in range(LAYERS)]
    outs = [torch.empty((B, H * G, 128), dtype=torch.bfloat16, device=dev) for _ in range(LAYERS)]
    lses = [torch.empty((B, H * G), dtype=torch.float32, device=dev) for _ in range(LAYERS)]
    sels = [torch.empty((B, H, dcfg.k_retrieval + dcfg.k_estimation), dtype=torch.int32,
                        device=dev) for _ in range(LAYERS)]
    rrows = [torch.empty((B, H, dcfg.k_retrieval + 1), dtype=torch.int32, device=dev)
             for _ in range(LAYERS)]

    def step(i):
        R.decode(qs[i], layers[i], dcfg, workspace=wss[i], out=outs[i], lse=lses[i])

    def sel_call(i):
        R.select_clusters(qs[i], layers[i], dcfg, wss[i], sel=sels[i], retr_rows=rrows[i])

    def att_call(i):
        R.attend_selected(qs[i], layers[i], dcfg, wss[i], out=outs[i], lse=lses[i])

    for i in range(max(args.warmup, 3)):
        step(i % LAYERS)
    for i in range(LAYERS):
        sel_call(i)
    torch.cuda.synchronize()
    for i in range(LAYERS):
        assert R.read_device_status(wss[i]) == 0

    # ---- algorithmic bytes of each step, from the realised selections
    counts = base.counts.cpu().numpy().astype(np.int64)
    C, k_r, k_e = geom.clusters, dcfg.k_retrieval, dcfg.k_estimation
    # step: what any implementation must move (centroids, sizes, steady and
    # retrieval K/V rows, value sums of live estimation clusters, offsets of
    # R, selected ids, q in, out and lse out); per call: the call's own
    # interface traffic, including the scores the select call hands over.
    bytes_sel, bytes_att, step_bytes = [], [], []
    for i in range(LAYERS):
        sel = sels[i].cpu().numpy()
        rr = rrows[i].cpu().numpy()
        b_sel = b_att = b_step = 0
        for h in range(H):
            T_R = int(rr[0, h, -1])
            E = sel[0, h, k_r:k_r + k_e]
            E = E[E >= 0]
            live_E = int((counts[0, h, E] > 0).sum())
            kv_rows = (geom.steady + T_R) * 128 * 2 * 2
            b_step += C * 128 * 2 + C * 4 + kv_rows + live_E * 128 * 4 + (k_r + k_e) * 4 + \
                k_r * 4 + G * 128 * 2 * 2 + G * 4
            b_sel += C * 128 * 2 + C * 4 + G * 128 * 2 + (G + 1) * C * 4 + \
                (k_r + k_e) * 4 + (k_r + 1) * 4
            b_att += kv_rows + live_E * 128 * 4 + (k_r + k_e) * 4 + (k_r + 1) * 4 + k_r * 4 + \
                k_e * 4 + G * k_e * 4 + G * 128 * 2 * 2 + G * 4
        bytes_sel.append(b_sel)
        bytes_att.append(b_att)
        step_bytes.append(b_step)

    # ---- CUDA graphs: the timed loop replays captured decode calls
    stream = torch.cuda.Stream(dev)
    K = args.steps

    def capture(fn, idxs):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in idxs:
                fn(i)
        return g

    torch.cuda.synchronize()
    g_full = capture(step, range(LAYERS))
    g_rem = capture(step, range(K % LAYERS)) if K % LAYERS else None
    g_sel = capture(sel_call, range(LAYERS))
    g_att = capture(att_call, range(LAYERS))
    for _ in range(2):
        g_full.replay()
    torch.cuda.synchronize()

    def timed(fn):
        if ws_n > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            fn()
            e1.record(stream)
        torch.cuda.synchronize()
        if ws_n > 1:
            torch.distributed.barrier()
        return e0.elapsed_time(e1)

    def main_loop():
        for _ in range(K // LAYERS):
            g_full.replay()
        if g_rem is not None:
            g_rem.replay()

    clocks = ClockSampler(local)
    clocks.start()
    ms = timed(main_loop)
    clk = clocks.stop()
    # per-call timings for the roofline (same graphs, rotating layers)
    reps = max(1, min(200, (K + LAYERS - 1) // LAYERS))
    ms_sel = timed(lambda: [g_sel.replay() for _ in range(reps)]) / (reps * LAYERS)
    ms_att = timed(lambda: [g_att.replay() for _ in range(reps)]) / (reps * LAYERS)

    ms, ms_sel, ms_att, build_ms = max_over_ranks([ms, ms_sel, ms_att, build_ms], dev)

    # ---- end to end through the public API: pinned H2D of q, D2H of the output
    q_host = [qs[i].cpu().pin_memory() for i in range(LAYERS)]
    o_host = torch.empty((B, H * G, 128), dtype=torch.bfloat16).pin_memory()
    q_dev = torch.empty_like(qs[0])
    k_e2e = min(K, 2000)

    def e2e_loop():
        for i in range(k_e2e):
            j = i % LAYERS
            q_dev.copy_(q_host[j], non_blocking=True)
            R.decode(q_dev, layers[j], dcfg, workspace=wss[j], out=outs[j], lse=lses[j])
            o_host.copy_(outs[j], non_blocking=True)
            torch.cuda.current_stream().synchronize()

    for i in range(3):
        q_dev.copy_(q_host[i], non_blocking=True)
        R.decode(q_dev, layers[i], dcfg, workspace=wss[i], out=outs[i], lse=lses[i])
        o_host.copy_(outs[i], non_blocking=True)
        torch.cuda.current_stream().synchronize()
    ms_e2e = max_over_ranks([timed(e2e_loop)], dev)[0]

    ms_per_step = ms / K
    value = K * ws_n / (ms / 1e3)
    mean_bytes = float(np.mean(step_bytes))
    gbs_sel = float(np.mean(bytes_sel)) / (ms_sel * 1e-3) / 1e9
    gbs_att = float(np.mean(bytes_att)) / (ms_att * 1e-3) / 1e9
    # one decode_kernel launch (cooperative, S1-S6) plus a small memset node
    # (status word and counters) per decode step: the step time is an upper
    # bound on the kernel's duration
    dominant = ("decode_kernel (S1-S6, one cooperative launch per step)",
                mean_bytes / (ms_per_step * 1e-3) / 1e9, ms_per_step, mean_bytes)
    traffic, sha = _traffic_from_profiles(os.path.join(ROOT, "kv_cache_vector_segmented_b200",
                                                       "csrc", "decode.cu"))
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws_n, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16 data, fp32 math",
        "data": "synthetic (seeded mixture-of-Gaussians keys, Gaussian values; the pages' "
                "RULER/LongBench/NIAH workloads are not in this container)",
        "config": {"workload": WORKLOAD, "global_batch": B * ws_n, "seq_len": N,
                   "kv_heads": H, "q_heads": H * G, "head_dim": 128, "clusters_per_head": C,
                   "k_retrieval": k_r, "k_estimation": k_e, "parallelism": f"replicas x{ws_n}",
                   "l2": f"rotating {LAYERS} layer instances, {LAYERS * mean_bytes / 1e6:.0f} MB "
                         "touched per cycle (> 126 MB L2)",
                   "timing": "CUDA graphs of decode calls, CUDA events on the launch stream"},
        "step_bytes": mean_bytes,
        "step_gbs": mean_bytes / (ms_per_step * 1e-3) / 1e9,
        "roofline": {"bound": "hbm", "kernel": dominant[0], "achieved": dominant[1],
                     "peak": hbm_peak, "unit": "GB/s", "frac": dominant[1] / hbm_peak,
                     "peak_kind": peak_kind, "bytes_per_launch": dominant[3],
                     "us_per_launch": dominant[2] * 1e3, "traffic": traffic,
                     "frac_of_8tbs": dominant[1] / 8000.0},
        "split_calls": {"select_us": ms_sel * 1e3, "select_gbs": gbs_sel,
                        "attend_us": ms_att * 1e3, "attend_gbs": gbs_att},
        "kmeans": {"tok_per_s": H * M / (build_ms * 1e-3), "ms_per_build": build_ms,
                   "iters": 10, "segments_per_head": len(segs), "clusters_per_segment": 512,
                   "assign_tflops_lower_bound": assign_flop / (build_ms * 1e-3) / 1e12,
                   "assign_frac_of_sustained_bf16": assign_flop / (build_ms * 1e-3) / 1e12 / tf_sus},
        "clocks": clk,
        "e2e": {"value": k_e2e * ws_n / (ms_e2e / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": B * H * G * 128 * 2,
                "d2h_bytes_per_step": B * H * G * 128 * 2, "steps": k_e2e},
        "gpu_launches": K,
    }
    if rank == 0 and ws_n == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(kv, budget_s=20.0)
    del g_full, g_rem, g_sel, g_att
    return res


# --------------------------------------------------------------------- oracle
def _oracle_index(kv, heads):
    import oracle as O
    out = []
    m0, M = O.middle_range(N)
    for h in heads:
        comp = kv.component[0, h, m0:m0 + M].astype(np.int64) % 512
        out.append(O.index_from_labels(kv.K[0, h].double().numpy(), kv.V[0, h].double().numpy(),
                                       comp))
    return out


def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([p.get("num_threads", 1) for p in threadpool_info()] or [1])
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(kv, budget_s=20.0):
    """The oracle, as it stands, on the host cores: decode of sampled KV heads
    (scaled to one 8-head step) and k-means of one segment."""
    import oracle as O
    t0 = time.time()
    heads = [0, 1]
    idx = _oracle_index(kv, heads)
    q = S.make_queries(kv, G, seed=10).double().numpy()
    k_r, k_e = O.default_budgets(idx[0]["C"])
    per_head = []
    while time.time() - t0 < budget_s * 0.5 or len(per_head) < 2:
        for j, h in enumerate(heads):
            s = time.perf_counter()
            O.tripartite_attention(q[0, h * G:(h + 1) * G], idx[j], k_r, k_e)
            per_head.append(time.perf_counter() - s)
        if len(per_head) >= 40:
            break
    step_s = float(np.median(per_head)) * H
    m0, M = O.middle_range(N)
    X = kv.K[0, 0, m0:m0 + 8192].double().numpy()
    init = np.random.default_rng(0).choice(8192, 512, replace=False)
    s = time.perf_counter()
    O.kmeans(X, init, 10)
    km_s = time.perf_counter() - s
    return {"value": 1.0 / step_s, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
            "sample": f"{len(per_head)} single-KV-head decodes (heads 0-1 of 8, 4 q heads each, "
                      f"147+1884 clusters) scaled x8 to one step; k-means: 1 segment of 8192 "
                      f"keys x 512 clusters x 10 iterations",
            "kmeans_tok_per_s": 8192 / km_s, "host_cpu_count": os.cpu_count()}


def run_reference(args, ws_n, rank):
    """The fp64 CPU oracle timed on the host cores, same workload and metric."""
    import oracle as O
    kv = S.make_kv(B, H, N, seed=0)
    q = S.make_queries(kv, G, seed=10).double().numpy()
    # heads per step so that (warmup + steps) steps fit in about two minutes
    t0 = time.perf_counter()
    idx0 = _oracle_index(kv, [0])
    k_r, k_e = O.default_budgets(idx0[0]["C"])
    s = time.perf_counter()
    O.tripartite_attention(q[0, 0:G], idx0[0], k_r, k_e)
    t_head = max(time.perf_counter() - s, 1e-4)
    total = args.steps + args.warmup
    n_heads = int(max(1, min(H, 120.0 / (total * t_head))))
    idx = idx0 + (_oracle_index(kv, list(range(1, n_heads))) if n_heads > 1 else [])
    times = []
    for it in range(total):
        s = time.perf_counter()
        for h in range(n_heads):
            O.tripartite_attention(q[0, h * G:(h + 1) * G], idx[h], k_r, k_e)
        el = (time.perf_counter() - s) * H / n_heads
        if it >= args.warmup:
            times.append(el)
    step_s = float(np.mean(times))
    v = 1.0 / step_s
    sample = f"{n_heads} of {H} KV heads per step (4 q heads each), time scaled x{H / n_heads:g}"
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": ws_n,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD, "global_batch": B, "seq_len": N},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "setup_s": time.perf_counter() - t0 - sum(times)}


def run_profile_case():
    """Small case for an ncu capture of the two kernels of the path: one
    128K-token layer of the benchmark geometry (about 1.1 GB on the device),
    one index build (10 k-means iterations) and 6 decode calls."""
    import kv_cache_vector_segmented_b200 as R
    dev = torch.device("cuda", 0)
    cfg = R.IndexConfig.make(B, H, G, N, iters=10)
    kv = S.make_kv(B, H, N, seed=0)
    segs = _segment_sizes(R.geometry(cfg))
    ip = S.init_positions([L for L, _ in segs], [k for _, k in segs], B, H, seed=3)
    idx = R.build_index(kv.K.to(dev), kv.V.to(dev), cfg, init_pos=torch.from_numpy(ip).to(dev))
    q = S.make_queries(kv, G, seed=10).to(dev)
    dcfg = R.default_budgets(idx.geom.clusters)
    ws = R.alloc_workspace(R.decode_workspace_bytes(cfg, dcfg), dev)
    for _ in range(6):
        R.decode(q, idx, dcfg, workspace=ws)
    torch.cuda.synchronize()
    assert R.read_device_status(ws) == 0
    print("profile case done", flush=True)


def run_cfg5():
    """Llama3-8B-1048K geometry, batch 1, 1M-token context: K/V rows in pinned
    host memory, a GPU block cache of 5 % of each head's 2 KB blocks (LRU),
    64 decode steps with drifting queries.  Each step: selection on the
    device, the cache plan on the host, the gather of hits (cache) and misses
    (host) into the execution buffer, admission of the misses, attention.
    Wall-clock per step (the host plan and the step's sync are part of the
    synchronous access path); the gather of the fetch list is also timed
    with CUDA events for the host-link rate."""
    import kv_cache_vector_segmented_b200 as R
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    B5, H5, G5, N5 = 1, 8, 4, 1 << 20
    steps, warm = 64, 3
    cfg = R.IndexConfig.make(B5, H5, G5, N5, iters=10)
    geom = R.geometry(cfg)
    kv = S.make_kv(B5, H5, N5, seed=0)
    segs = _segment_sizes(geom)
    ip = S.init_positions([L for L, _ in segs], [k for _, k in segs], B5, H5, seed=3)
    idx = R.build_index(kv.K.to(dev), kv.V.to(dev), cfg, init_pos=torch.from_numpy(ip).to(dev))
    torch.cuda.synchronize()
    del kv.K, kv.V  # the host copy that matters from here on is the permuted one
    C = geom.clusters
    d = R.default_budgets(C)
    k_r = d.k_retrieval
    hK = idx.Kp.cpu().pin_memory()
    hV = idx.Vp.cpu().pin_memory()
    counts = idx.counts.cpu().numpy().reshape(B5 * H5, C)
    offsets = idx.offsets.cpu().numpy().reshape(B5 * H5, C + 1)
    br = 8
    blocks = (counts.astype(np.int64) + br - 1) // br
    cache = R.BlockCache(B5 * H5, max(1, int(0.05 * blocks.sum(axis=1).max())), br)
    cK = torch.zeros((B5, H5, cache.pool_rows, 128), dtype=torch.bfloat16, device=dev)
    cV = torch.zeros_like(cK)
    exec_rows = int(R.max_retrieval_rows(counts, k_r).max())
    eK = torch.empty((B5, H5, exec_rows, 128), dtype=torch.bfloat16, device=dev)
    eV = torch.empty_like(eK)
    ws = R.alloc_workspace(R.decode_workspace_bytes(cfg, d), dev)
    gws = R.alloc_workspace(256, dev)
    out = torch.empty((B5, H5 * G5, 128), dtype=torch.bfloat16, device=dev)
    qs = [q.contiguous().to(dev) for q in
          S.drift_queries(S.make_queries(kv, G5, seed=52), warm + steps, seed=53)]
    hit_rows = miss_rows = 0
    gather_ms = 0.0
    t0 = time.perf_counter()
    for i, qd in enumerate(qs):
        if i == warm:
            torch.cuda.synchronize()
            hit_rows = miss_rows = 0
            gather_ms = 0.0
            t0 = time.perf_counter()
        sel, _ = R.select_clusters(qd, idx, d, ws)
        # only the retrieval ids (the first k_r of each unit) go back to the host
        sel_r = sel.reshape(B5 * H5, -1)[:, :k_r].cpu().numpy()
        fetch, admit, st = cache.plan(sel_r, k_r, counts, offsets)
        hit_rows += st["hit_rows"]
        miss_rows += st["miss_rows"]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        fd = torch.from_numpy(fetch).to(dev)
        e0.record()
        R.gather_blocks(fd, hK, hV, eK, eV, gws, cK, cV)
        e1.record()
        R.gather_blocks(torch.from_numpy(admit).to(dev), hK, hV, eK, eV, gws, cK, cV)
        R.attend_selected(qd, idx, d, ws, exec_K=eK, exec_V=eV, out=out)
        e1.synchronize()
        gather_ms += e0.elapsed_time(e1)
    torch.cuda.synchronize()
    wall_s = time.perf_counter() - t0
    status = max(R.read_device_status(ws), R.read_device_status(gws))
    cache.close()
    host_bytes = miss_rows * 2 * 128 * 2  # K and V rows of the misses, bf16
    return {
        "leg": "config 5", "metric": "decode steps/s with K/V in host memory", "unit": "steps/s",
        "value": steps / wall_s, "ms_per_step": 1e3 * wall_s / steps, "steps": steps,
        "warmup": warm, "n_gpus": 1, "data": "synthetic",
        "config": {"workload": "llama3-8b-1048k decode, 1M context, batch 1, 32 q / 8 kv heads, "
                               "K/V rows in pinned host memory, 5 % LRU block cache per head",
                   "clusters_per_head": C, "k_retrieval": k_r, "k_estimation": d.k_estimation,
                   "cache_blocks_per_head": cache.cfg.blocks_per_unit, "exec_rows": exec_rows,
                   "timing": "wall clock per step, host plan and the step's device sync "
                             "included; fetch gather by CUDA events"},
        "hit_rate_rows": hit_rows / max(1, hit_rows + miss_rows),
        "host_bytes_per_step": host_bytes / steps,
        "fetch_gather_ms_per_step": gather_ms / steps,
        "host_link_gbs": host_bytes / max(1e-9, gather_ms * 1e-3) / 1e9,
        "device_status": int(status),
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=6400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ncu-case", action="store_true",
                    help="run only the small case used for ncu captures")
    ap.add_argument("--cfg5", action="store_true",
                    help="run only the 1M-token host-memory leg (block cache, gather, "
                         "attention) and print its own JSON line")
    args = ap.parse_args()
    if args.ncu_case:
        run_profile_case()
        return
    if args.cfg5:
        print(json.dumps(run_cfg5()), flush=True)
        return
    if args.warmup < 3:
        args.warmup = 3
    ws_n, rank, local = _dist()
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, ws_n, rank)), flush=True)
        return
    if ws_n > 1:
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    res = run_ours(args, ws_n, rank, local)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if ws_n > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
