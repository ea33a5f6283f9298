#!/usr/bin/env python
"""Benchmark of the wave-index decode path on B200.

Headline: decode-attention steps/s at 128K context on the Llama-3.1-8B
geometry (batch 1, 32 query heads, 8 KV heads, head_dim 128, sixteen 8K
segments of 512 clusters; retrieval 147 and estimation 1884 clusters per KV
head), with HBM GB/s of the dominant kernel against the measured copy
bandwidth, and the segmented k-means build (8 KV heads x 128K tokens, 10
iterations) in key vectors clustered per second.  At one GPU the line also
carries the other workloads, each with its own clock record:
  config1   one KV head, 8K context: single-step latency;
  config4   Qwen2.5-7B geometry, batch 16 x 128K, 32 drifting steps;
  config5   Llama3-8B-1048K geometry, 1M context, K/V in pinned host memory
            behind a 5 % LRU block cache, 64 steps, synchronous and
            asynchronous cache update.

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
MIN_TIMED_MS = 200.0  # the K-step timed region is repeated until this much device time


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


def _code_sha16(path: str) -> str:
    """First 16 hex digits of the sha256 of a source file's code: text after
    // (outside string literals) and blank lines dropped, so an edit of the
    comments alone keeps the value."""
    out = []
    for line in open(path, encoding="utf-8"):
        code, quoted, i = [], False, 0
        while i < len(line):
            c = line[i]
            if c == '"' and (i == 0 or line[i - 1] != "\\"):
                quoted = not quoted
            if not quoted and line.startswith("//", i):
                break
            code.append(c)
            i += 1
        t = "".join(code).strip()
        if t:
            out.append(t)
    return hashlib.sha256("\n".join(out).encode()).hexdigest()[:16]


def _traffic_from_profiles(kernel_src: str, kernel: str):
    """DRAM bytes per launch recorded by an ncu capture of `kernel` from the
    current kernel code (null when the code changed since)."""
    sha = _code_sha16(kernel_src)
    pat = re.compile(r"traffic_bytes_per_launch:\s*(\d+)\s+code_sha256_16:\s*([0-9a-f]{16})")
    for fn in sorted(os.listdir(os.path.join(ROOT, "profiles"))):
        if not (fn.startswith(kernel) and fn.endswith(".md")):
            continue
        text = open(os.path.join(ROOT, "profiles", fn), encoding="utf-8").read()
        for m in pat.finditer(text):
            if m.group(2) == sha:
                return int(m.group(1)), sha
    return None, sha


def _segment_sizes(geom, seg_len=8192, clusters=512):
    """(tokens, clusters) of each 8K segment of the middle tokens, from the
    library's own geometry (the seeded initial positions need them)."""
    M = geom.middle
    return [(min(seg_len, M - s * seg_len), min(clusters, M - s * seg_len))
            for s in range(geom.num_segments)]


def headline_config(ws_n, C, k_r, k_e):
    """The headline workload's config keys, printed alike by both arms."""
    return {"workload": WORKLOAD, "global_batch": B * ws_n, "seq_len": N, "kv_heads": H,
            "q_heads": H * G, "head_dim": 128, "clusters_per_head": C, "k_retrieval": k_r,
            "k_estimation": k_e, "parallelism": f"replicas x{ws_n}"}


def step_bytes(counts, sel, rr, C, k_r, k_e, steady, G_):
    """Algorithmic bytes of one decode step, from its realised selection:
    what any implementation must move (centroids and sizes of every cluster,
    steady and retrieval K/V rows, value sums of live estimation clusters,
    offsets of R, the selected ids, q in, out and lse out), summed over the
    (sequence, KV head) units.  counts int [U][C]; sel int [U][k_r + k_e];
    rr int [U][k_r + 1] (retrieval-row prefix)."""
    total = 0
    for u in range(counts.shape[0]):
        T_R = int(rr[u, -1])
        E = sel[u, k_r:k_r + k_e]
        E = E[E >= 0]
        live_E = int((counts[u, E] > 0).sum())
        total += C * 128 * 2 + C * 4 + (steady + T_R) * 128 * 2 * 2 + live_E * 128 * 4 + \
            (k_r + k_e) * 4 + k_r * 4 + G_ * 128 * 2 * 2 + G_ * 4
    return total


def timed_region(fn, ws_n, stream, min_ms=MIN_TIMED_MS, max_reps=200):
    """Device time of fn() (one K-step region), bracketed by a barrier and a
    synchronize on both sides and timed with CUDA events on `stream`;
    repeated until min_ms of device time (at most max_reps times).  Returns
    (median ms, every sample)."""
    samples = []
    while True:
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
        samples.append(e0.elapsed_time(e1))
        # every rank takes the same number of repetitions (decided on rank 0's clock)
        stop = sum(samples) >= min_ms or len(samples) >= max_reps
        if ws_n > 1:
            t = torch.tensor([1 if stop else 0], device=torch.cuda.current_device())
            torch.distributed.broadcast(t, 0)
            stop = bool(t.item())
        if stop:
            return statistics.median(samples), samples


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
    for _ in range(5):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        R.build_index(Kd, Vd, cfg, init_pos=ipd, out=base, workspace=build_ws)
        e1.record()
        torch.cuda.synchronize()
        kms.append(e0.elapsed_time(e1))
    build_ms = statistics.median(kms)
    assign_flop = 2.0 * H * M * 512 * 128 * 10
    prefill = (build_beside_prefill(R, Kd, Vd, cfg, ipd, base, build_ws, dev)
               if ws_n == 1 and not args.headline_only else None)

    # ---- 32 layer instances (distinct memory, so L2 cannot hold a cycle)
    def clone_index(ix):
        f = {k: getattr(ix, k) for k in ("Kp", "Vp", "perm", "centroid", "counts", "offsets",
                                           "vsum", "Ks", "Vs")}
        return R.Index(cfg=cfg, geom=geom, **{k: v.clone() for k, v in f.items()})

    layers = [clone_index(base) for _ in range(LAYERS)]
    del Kd, Vd
    qs = [S.make_queries(kv, G, seed=1000 * rank + 10 + i).to(dev) for i in range(LAYERS)]
    decs = [R.Decoder(layers[i], dcfg) for i in range(LAYERS)]
    sels = [torch.empty((B, H, dcfg.k_retrieval + dcfg.k_estimation), dtype=torch.int32,
                        device=dev) for _ in range(LAYERS)]
    rrows = [torch.empty((B, H, dcfg.k_retrieval + 1), dtype=torch.int32, device=dev)
             for _ in range(LAYERS)]

    def step(i):
        decs[i](qs[i])

    def sel_call(i):
        R.select_clusters(qs[i], layers[i], dcfg, decs[i].ws, sel=sels[i], retr_rows=rrows[i])

    def att_call(i):
        R.attend_selected(qs[i], layers[i], dcfg, decs[i].ws, out=decs[i].out, lse=decs[i].lse)

    for i in range(max(args.warmup, 3)):
        step(i % LAYERS)
    for i in range(LAYERS):
        sel_call(i)
    torch.cuda.synchronize()
    for i in range(LAYERS):
        assert R.read_device_status(decs[i].ws) == 0

    # ---- algorithmic bytes of each step, from the realised selections
    counts = base.counts.cpu().numpy().astype(np.int64).reshape(B * H, -1)
    C, k_r, k_e = geom.clusters, dcfg.k_retrieval, dcfg.k_estimation
    step_b, bytes_sel, bytes_att = [], [], []
    for i in range(LAYERS):
        sel = sels[i].cpu().numpy().reshape(B * H, -1)
        rr = rrows[i].cpu().numpy().reshape(B * H, -1)
        step_b.append(step_bytes(counts, sel, rr, C, k_r, k_e, geom.steady, G))
        # per split call: its own interface traffic, including the scores the
        # select call hands over
        kv_b = sum((geom.steady + int(rr[u, -1])) * 128 * 2 * 2 for u in range(B * H))
        live = sum(int((counts[u, sel[u, k_r:][sel[u, k_r:] >= 0]] > 0).sum())
                   for u in range(B * H))
        bytes_sel.append(B * H * (C * 128 * 2 + C * 4 + G * 128 * 2 + (G + 1) * C * 4 +
                                  (k_r + k_e) * 4 + (k_r + 1) * 4))
        bytes_att.append(kv_b + live * 128 * 4 + B * H * ((k_r + k_e) * 4 + (k_r + 1) * 4 +
                                                          k_r * 4 + k_e * 4 + G * k_e * 4 +
                                                          G * 128 * 2 * 2 + G * 4))

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

    def main_loop():
        for _ in range(K // LAYERS):
            g_full.replay()
        if g_rem is not None:
            g_rem.replay()

    clocks = ClockSampler(local)
    clocks.start()
    ms, ms_samples = timed_region(main_loop, ws_n, stream)
    clk = clocks.stop()
    # per-call timings for the split calls (same graphs, rotating layers)
    ms_sel = timed_region(lambda: g_sel.replay(), ws_n, stream, min_ms=50)[0] / LAYERS
    ms_att = timed_region(lambda: g_att.replay(), ws_n, stream, min_ms=50)[0] / LAYERS

    ms, ms_sel, ms_att, build_ms = max_over_ranks([ms, ms_sel, ms_att, build_ms], dev)

    # ---- end to end through the public API: pinned H2D of q, D2H of the output
    q_host = [qs[i].cpu().pin_memory() for i in range(LAYERS)]
    o_host = torch.empty((B, H * G, 128), dtype=torch.bfloat16).pin_memory()
    k_e2e = min(max(K, 1000), 4000)
    cur = torch.cuda.current_stream(dev)

    def e2e_loop():
        # one public call per step: the query's H2D copy, the step, the
        # output's D2H copy and the wait for it (ri_decode_attention_host)
        for i in range(k_e2e):
            j = i % LAYERS
            decs[j].step_host(q_host[j], o_host, cur)

    for i in range(3):
        decs[i].step_host(q_host[i], o_host, cur)
    ms_e2e = max_over_ranks([timed_region(e2e_loop, ws_n, cur, min_ms=0)[0]], dev)[0]

    ms_per_step = ms / K
    value = K * ws_n / (ms / 1e3)
    mean_bytes = float(np.mean(step_b))
    gbs_sel = float(np.mean(bytes_sel)) / (ms_sel * 1e-3) / 1e9
    gbs_att = float(np.mean(bytes_att)) / (ms_att * 1e-3) / 1e9
    # one decode_kernel launch (S1-S6) per decode step and nothing else: the
    # step time is the kernel's duration plus the gap between graph nodes
    achieved = mean_bytes / (ms_per_step * 1e-3) / 1e9
    traffic, sha = _traffic_from_profiles(os.path.join(ROOT, "kv_cache_vector_segmented_b200",
                                                       "csrc", "decode.cu"), "decode_kernel")
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws_n, "steps": K,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16 data, fp32 math",
        "data": "synthetic (seeded mixture-of-Gaussians keys, Gaussian values; the pages' "
                "RULER/LongBench/NIAH workloads are not in this container)",
        "config": headline_config(ws_n, C, k_r, k_e),
        "timing": {"l2": f"rotating {LAYERS} layer instances, {LAYERS * mean_bytes / 1e6:.0f} MB "
                         "touched per cycle (> 126 MB L2)",
                   "method": "CUDA graphs of decode calls, CUDA events on the launch stream; "
                             f"the {K}-step region timed {len(ms_samples)} times, median",
                   "region_ms_samples": [round(x, 4) for x in ms_samples[:50]]},
        "step_bytes": mean_bytes,
        "step_gbs": achieved,
        "roofline": {"bound": "hbm", "kernel": "decode_kernel (S1-S6, one launch per step: "
                                               "a thread-block cluster per (sequence, KV head))",
                     "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
                     "frac": achieved / hbm_peak, "peak_kind": peak_kind,
                     "bytes_per_launch": mean_bytes, "us_per_launch": ms_per_step * 1e3,
                     "traffic": traffic, "frac_of_8tbs": achieved / 8000.0},
        "split_calls": {"select_us": ms_sel * 1e3, "select_gbs": gbs_sel,
                        "attend_us": ms_att * 1e3, "attend_gbs": gbs_att},
        "kmeans": {"tok_per_s": H * M / (build_ms * 1e-3), "ms_per_build": build_ms,
                   "iters": 10, "segments_per_head": len(segs), "clusters_per_segment": 512,
                   "assign_tflops_lower_bound": assign_flop / (build_ms * 1e-3) / 1e12,
                   "assign_frac_of_sustained_bf16": assign_flop / (build_ms * 1e-3) / 1e12 / tf_sus,
                   "beside_prefill": prefill},
        "clocks": clk,
        "e2e": {"value": k_e2e * ws_n / (ms_e2e / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": B * H * G * 128 * 2,
                "d2h_bytes_per_step": B * H * G * 128 * 2, "steps": k_e2e,
                "call": "Decoder.step_host (ri_decode_attention_host): pinned q H2D, the "
                        "step, out D2H and the stream wait inside one call per step"},
        "gpu_launches": K,
    }
    del g_full, g_rem, g_sel, g_att, layers, decs
    torch.cuda.empty_cache()
    if rank == 0 and ws_n == 1 and not args.headline_only:
        res["config1"] = run_config1(dev, hbm_peak, local)
        torch.cuda.empty_cache()
        res["config4"] = run_config4(dev, hbm_peak, local)
        torch.cuda.empty_cache()
        res["config5"] = run_config5(dev, local)
        torch.cuda.empty_cache()
    if rank == 0 and ws_n == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(kv, budget_s=20.0)
    return res


# ------------------------------------------------------------ build and prefill
def build_beside_prefill(R, Kd, Vd, cfg, ipd, base, build_ws, dev):
    """The index build next to the prefill it belongs to: causal attention of
    the same layer (32 query heads on 8 KV heads, 128K tokens, torch's SDPA
    flash kernel, a library call used only as the yardstick) timed alone,
    the build alone, and both at once on two streams; and the build with 16K
    segments (512 clusters each).  CUDA events; medians of 3."""
    Bq, Hq, Nq = cfg.batch, cfg.num_kv_heads * cfg.group_size, cfg.seq_len
    g = torch.Generator(device=dev)
    g.manual_seed(5)
    q = torch.randn((Bq, Hq, Nq, 128), generator=g, device=dev).to(torch.bfloat16)
    k = Kd.repeat_interleave(cfg.group_size, dim=1)
    v = Vd.repeat_interleave(cfg.group_size, dim=1)
    s_pre, s_bld = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def prefill():
        torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)

    def build():
        R.build_index(Kd, Vd, cfg, init_pos=ipd, out=base, workspace=build_ws)

    def timed(fns):
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e0.record()
        ends = []
        for st, fn in fns:
            st.wait_event(e0)
            with torch.cuda.stream(st):
                fn()
                e = torch.cuda.Event(enable_timing=True)
                e.record(st)
                ends.append(e)
        torch.cuda.synchronize()
        return max(e0.elapsed_time(e) for e in ends)

    timed([(s_pre, prefill)])  # warm-up (SDPA's first call)
    t_pre = statistics.median(timed([(s_pre, prefill)]) for _ in range(3))
    t_bld = statistics.median(timed([(s_bld, build)]) for _ in range(3))
    t_both = statistics.median(timed([(s_pre, prefill), (s_bld, build)]) for _ in range(3))
    assert R.read_device_status(build_ws) == 0
    del q, k, v
    cfg16 = R.IndexConfig.make(cfg.batch, cfg.num_kv_heads, cfg.group_size, cfg.seq_len,
                               seg_len=16384, clusters_per_seg=512, iters=cfg.iters)
    segs16 = _segment_sizes(R.geometry(cfg16), seg_len=16384)
    ip16 = S.init_positions([L for L, _ in segs16], [kk for _, kk in segs16], cfg.batch,
                            cfg.num_kv_heads, seed=7)
    ip16 = torch.from_numpy(ip16).to(dev)
    idx16 = R.build_index(Kd, Vd, cfg16, init_pos=ip16)
    t16 = []
    for _ in range(3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        R.build_index(Kd, Vd, cfg16, init_pos=ip16, out=idx16, workspace=idx16._build_ws)
        e1.record()
        torch.cuda.synchronize()
        t16.append(e0.elapsed_time(e1))
    assert R.read_device_status(idx16._build_ws) == 0
    del idx16
    return {"prefill_attention_ms": t_pre, "build_ms": t_bld, "both_on_two_streams_ms": t_both,
            "build_share_of_prefill_attention": t_bld / t_pre,
            "added_by_build_when_overlapped_ms": t_both - t_pre,
            "build_seg16k_ms": statistics.median(t16), "seg16k_clusters_per_segment": 512,
            "prefill": "causal SDPA (flash), 32 q heads x 128K tokens x d 128, bf16, one layer"}


# ------------------------------------------------------------ other workloads
def _build_for(R, dev, Bc, Hc, Gc, Nc, seed, host_gen=False):
    """A k-means index (10 iterations, seeded initial positions) of a seeded
    workload; returns (index, kv) with kv drawn on the host (small cases) or
    on the device."""
    cfg = R.IndexConfig.make(Bc, Hc, Gc, Nc, iters=10)
    geom = R.geometry(cfg)
    segs = _segment_sizes(geom)
    ip = S.init_positions([L for L, _ in segs], [k for _, k in segs], Bc, Hc, seed=seed + 3)
    if host_gen:
        kv = S.make_kv(Bc, Hc, Nc, seed=seed)
        Kd, Vd = kv.K.to(dev), kv.V.to(dev)
    else:
        kv = S.make_kv_device(Bc, Hc, Nc, dev, seed=seed)
        Kd, Vd = kv.K, kv.V
    idx = R.build_index(Kd, Vd, cfg, init_pos=torch.from_numpy(ip).to(dev))
    torch.cuda.synchronize()
    assert R.read_device_status(idx._build_ws) == 0
    idx._build_ws = None
    if not host_gen:
        kv.K = kv.V = None
    return idx, kv


def run_config1(dev, hbm_peak, local):
    """One KV head (GQA 4), 8K context, one 8K segment of 512 clusters: the
    latency of one decode step.  512 index instances rotate so the cycle
    touches more than L2 holds."""
    import kv_cache_vector_segmented_b200 as R
    n_inst, G1 = 512, 4
    idx, kv = _build_for(R, dev, 1, 1, G1, 8192, seed=0, host_gen=True)
    geom = idx.geom
    d = R.default_budgets(geom.clusters)
    f = {k: getattr(idx, k) for k in ("Kp", "Vp", "perm", "centroid", "counts", "offsets",
                                       "vsum", "Ks", "Vs")}
    insts = [R.Index(cfg=idx.cfg, geom=geom, **{k: v.clone() for k, v in f.items()})
             for _ in range(n_inst)]
    q = S.make_queries(kv, G1, seed=1).to(dev)
    decs = [R.Decoder(x, d) for x in insts]
    sel, rr = R.select_clusters(q, insts[0], d, decs[0].ws)
    counts = idx.counts.cpu().numpy().reshape(1, -1)
    sb = step_bytes(counts, sel.cpu().numpy().reshape(1, -1), rr.cpu().numpy().reshape(1, -1),
                    geom.clusters, d.k_retrieval, d.k_estimation, geom.steady, G1)
    stream = torch.cuda.Stream(dev)
    for x in decs[:3]:
        x(q)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for x in decs:
            x(q, stream)
    g.replay()
    torch.cuda.synchronize()
    assert all(R.read_device_status(x.ws) == 0 for x in decs[:4])
    clocks = ClockSampler(local)
    clocks.start()
    ms, samples = timed_region(lambda: g.replay(), 1, stream, min_ms=100)
    clk = clocks.stop()
    us = ms * 1e3 / n_inst
    del g
    return {"workload": "1 kv head (GQA 4), 8K context, one segment of 512 clusters, "
                        f"k_r {d.k_retrieval}, k_e {d.k_estimation}",
            "us_per_step": us, "steps_per_s": 1e6 / us, "bytes_per_step": sb,
            "gbs": sb / (us * 1e-6) / 1e9, "frac_of_hbm": sb / (us * 1e-6) / 1e9 / hbm_peak,
            "timing": f"CUDA graph of {n_inst} decode calls on {n_inst} index instances "
                      f"({n_inst * sb / 1e6:.0f} MB per cycle), median of {len(samples)}",
            "clocks": clk}


def run_config4(dev, hbm_peak, local):
    """Qwen2.5-7B geometry, batched decode: batch 16 x 4 KV heads x GQA 7,
    128K context, 32 consecutive steps with queries drifting N(0, 0.05^2)."""
    import kv_cache_vector_segmented_b200 as R
    B4, H4, G4, N4, steps = 16, 4, 7, 131072, 32
    idx, kv = _build_for(R, dev, B4, H4, G4, N4, seed=41)
    geom = idx.geom
    d = R.default_budgets(geom.clusters)
    qs = S.drift_queries_device(S.make_queries_device(kv, G4, seed=42), steps, seed=43)
    dec = R.Decoder(idx, d)
    counts = idx.counts.cpu().numpy().reshape(B4 * H4, -1)
    sb = []
    for q in qs:
        sel, rr = R.select_clusters(q, idx, d, dec.ws)
        sb.append(step_bytes(counts, sel.cpu().numpy().reshape(B4 * H4, -1),
                             rr.cpu().numpy().reshape(B4 * H4, -1), geom.clusters,
                             d.k_retrieval, d.k_estimation, geom.steady, G4))
    mean_b = float(np.mean(sb))
    stream = torch.cuda.Stream(dev)
    for q in qs[:3]:
        dec(q)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for q in qs:
            dec(q, stream)
    g.replay()
    torch.cuda.synchronize()
    assert R.read_device_status(dec.ws) == 0
    clocks = ClockSampler(local)
    clocks.start()
    ms, samples = timed_region(lambda: g.replay(), 1, stream, min_ms=200)
    clk = clocks.stop()
    us = ms * 1e3 / steps
    del g
    return {"workload": "qwen2.5-7b batched decode, batch 16 x 128K, 28 q / 4 kv heads, "
                        f"{geom.clusters} clusters per head, k_r {d.k_retrieval}, "
                        f"k_e {d.k_estimation}, 32 drifting steps",
            "us_per_step": us, "steps_per_s": 1e6 / us, "tokens_per_s": B4 * 1e6 / us,
            "bytes_per_step": mean_b, "gbs": mean_b / (us * 1e-6) / 1e9,
            "frac_of_hbm": mean_b / (us * 1e-6) / 1e9 / hbm_peak,
            "timing": f"CUDA graph of the 32 steps (one decode_kernel launch each; "
                      f"{mean_b / 1e6:.0f} MB per step > L2), median of {len(samples)}",
            "data": "synthetic, drawn on the device (same recipe as the host generator)",
            "clocks": clk}


def _cfg5_mode(R, dev, local, idx, d, hK, hV, counts, offsets, qs, warm, mode):
    """One pass of the 1M-token host-memory workload with a fresh cache:
    `mode` "sync" (ri_cache_plan between select and gather) or "async" (cache
    worker: lookup on the critical path, LRU update and admit copies on a
    host thread and a side stream)."""
    units, k_r, br = counts.shape[0], d.k_retrieval, 8
    blocks = (counts.astype(np.int64) + br - 1) // br
    cap = max(1, int(0.05 * blocks.sum(axis=1).max()))
    cache = R.BlockCache(units, cap, br)
    shp = (idx.cfg.batch, idx.cfg.num_kv_heads)
    cK = torch.zeros((*shp, cache.pool_rows, 128), dtype=torch.bfloat16, device=dev)
    cV = torch.zeros_like(cK)
    exec_rows = int(R.max_retrieval_rows(counts, k_r).max())
    eK = torch.empty((*shp, exec_rows, 128), dtype=torch.bfloat16, device=dev)
    eV = torch.empty_like(eK)
    ws = R.alloc_workspace(R.decode_workspace_bytes(idx.cfg, d), dev)
    gws = R.alloc_workspace(256, dev)
    out = torch.empty((idx.cfg.batch, idx.cfg.num_kv_heads * idx.cfg.group_size, 128),
                      dtype=torch.bfloat16, device=dev)
    sel_host = torch.empty((units, k_r), dtype=torch.int32).pin_memory()
    sel_np = sel_host.numpy()
    stream = torch.cuda.current_stream(dev)
    worker = None
    if mode == "async":
        wgws = R.alloc_workspace(256, dev)
        worker = R.CacheWorker(cache, host_K=hK, host_V=hV, cache_K=cK, cache_V=cV, exec_K=eK,
                               exec_V=eV, gather_workspace=wgws)
    else:  # pinned staging of the two copy lists, so their H2D copies do not block
        cap_l = units * exec_rows
        stage = torch.empty((2, cap_l, 6), dtype=torch.int32).pin_memory()
        stage_d = torch.empty((2, cap_l, 6), dtype=torch.int32, device=dev)
    t_cache, t_wait, t_upd, gather_ms = [], [], [], 0.0
    hit_rows = miss_rows = rows_req = blocks_req = 0
    t0 = time.perf_counter()
    for i, qd in enumerate(qs):
        if i == warm:
            torch.cuda.synchronize()
            t_cache, t_wait, t_upd, gather_ms = [], [], [], 0.0
            hit_rows = miss_rows = rows_req = blocks_req = 0
            t0 = time.perf_counter()
        sel, _ = R.select_clusters(qd, idx, d, ws)
        sel_host.copy_(sel.reshape(units, -1)[:, :k_r])  # waits for the selection
        nreq = counts[np.arange(units)[:, None], np.maximum(sel_np, 0)] * (sel_np >= 0)
        rows_req += int(nreq.sum())
        blocks_req += int(((nreq + br - 1) // br).sum())
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if worker is None:
            s0 = time.perf_counter()
            fetch, admit, st = cache.plan(sel_np, k_r, counts, offsets)
            t_cache.append(time.perf_counter() - s0)
            nf, na = len(fetch), len(admit)
            stage[0, :nf].numpy()[:] = fetch
            stage[1, :na].numpy()[:] = admit
            stage_d[0, :nf].copy_(stage[0, :nf], non_blocking=True)
            stage_d[1, :na].copy_(stage[1, :na], non_blocking=True)
            e0.record(stream)
            R.gather_blocks(stage_d[0, :nf], hK, hV, eK, eV, gws, cK, cV,
                            shape=R.gather_shape(int((fetch[:, 1] == R.SRC_HOST).sum()), nf))
            e1.record(stream)
            R.gather_blocks(stage_d[1, :na], hK, hV, eK, eV, gws, cK, cV,
                            shape=R.gather_shape(0, na))
        else:
            s0 = time.perf_counter()
            worker.wait()            # the previous update, normally already applied
            s1 = time.perf_counter()
            fl, st = worker.lookup(sel_np, k_r, counts, offsets, stream)
            s2 = time.perf_counter()
            fd = worker.fetch_to_device(stream)
            e0.record(stream)
            R.gather_blocks(fd, hK, hV, eK, eV, gws, cK, cV,
                            shape=R.gather_shape(int((fl[:, 1] == R.SRC_HOST).sum()), len(fl)))
            e1.record(stream)
            s3 = time.perf_counter()
            worker.update_async(stream)
            s4 = time.perf_counter()
            t_wait.append(s1 - s0)
            t_cache.append(s2 - s1)
            t_upd.append(s4 - s3)
        hit_rows += st["hit_rows"]
        miss_rows += st["miss_rows"]
        R.attend_selected(qd, idx, d, ws, exec_K=eK, exec_V=eV, out=out)
        e1.synchronize()
        gather_ms += e0.elapsed_time(e1)
    torch.cuda.synchronize()
    wall_s = time.perf_counter() - t0
    steps = len(qs) - warm
    status = max(R.read_device_status(ws), R.read_device_status(gws))
    if worker is not None:
        worker.close()
        torch.cuda.synchronize()
        status = max(status, R.read_device_status(wgws))
    cache.validate()
    cache.close()
    host_bytes = miss_rows * 2 * 128 * 2  # K and V rows of the misses, bf16
    res = {"steps_per_s": steps / wall_s, "ms_per_step": 1e3 * wall_s / steps,
           "hit_rate_rows": hit_rows / max(1, hit_rows + miss_rows),
           "host_bytes_per_step": host_bytes / steps,
           "fetch_gather_ms_per_step": gather_ms / steps,
           "host_link_gbs": host_bytes / max(1e-9, gather_ms * 1e-3) / 1e9,
           "fragment_rows_skipped_frac": 1.0 - rows_req / max(1, br * blocks_req),
           "device_status": int(status)}
    if worker is None:
        res["plan_us_median"] = 1e6 * statistics.median(t_cache)
    else:
        res["lookup_us_median"] = 1e6 * statistics.median(t_cache)
        res["wait_for_update_us_median"] = 1e6 * statistics.median(t_wait)
        res["update_handoff_us_median"] = 1e6 * statistics.median(t_upd)
        res["update_cost_on_critical_path_us"] = 1e6 * (statistics.median(t_wait) +
                                                         statistics.median(t_upd))
    return res, {"cache_blocks_per_head": cap, "exec_rows": exec_rows}


def run_config5(dev, local):
    """Llama3-8B-1048K geometry, batch 1, 1M-token context: K/V rows in pinned
    host memory, a GPU block cache of 5 % of each head's 2 KB blocks (LRU),
    64 decode steps with drifting queries, once with the synchronous cache
    plan and once with the asynchronous update.  Wall clock per step (the
    host's part of the step is on its critical path); the fetch gather is
    also timed with CUDA events for the host-link rate."""
    import kv_cache_vector_segmented_b200 as R
    B5, H5, G5, N5, steps, warm = 1, 8, 4, 1 << 20, 64, 3
    idx, kv = _build_for(R, dev, B5, H5, G5, N5, seed=51)
    C = idx.geom.clusters
    d = R.default_budgets(C)
    hK = idx.Kp.cpu().pin_memory()
    hV = idx.Vp.cpu().pin_memory()
    counts = idx.counts.cpu().numpy().reshape(B5 * H5, C)
    offsets = idx.offsets.cpu().numpy().reshape(B5 * H5, C + 1)
    qs = S.drift_queries_device(S.make_queries_device(kv, G5, seed=52), warm + steps, seed=53)
    out = {"workload": "llama3-8b-1048k decode, 1M context, batch 1, 32 q / 8 kv heads, "
                       "K/V rows in pinned host memory, 5 % LRU block cache per head",
           "clusters_per_head": C, "k_retrieval": d.k_retrieval, "k_estimation": d.k_estimation,
           "steps": steps, "warmup": warm,
           "timing": "wall clock per step (selection, its D2H, the cache step on the host, "
                     "gathers, attention); fetch gather by CUDA events",
           "data": "synthetic, drawn on the device; queries drift N(0, 0.05^2) per step"}
    for mode in ("sync", "async"):
        clocks = ClockSampler(local)
        clocks.start()
        r, geo = _cfg5_mode(R, dev, local, idx, d, hK, hV, counts, offsets, qs, warm, mode)
        r["clocks"] = clocks.stop()
        out[mode] = r
        out.update(geo)
        torch.cuda.empty_cache()
    return out


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


def _oracle_decode_sample(idx, q, heads, budget_s, max_n=40):
    """Per-head decode times of the oracle over `heads`, for about budget_s."""
    import oracle as O
    k_r, k_e = O.default_budgets(idx[0]["C"])
    per_head = []
    t0 = time.time()
    while time.time() - t0 < budget_s or len(per_head) < 2:
        for j, h in enumerate(heads):
            s = time.perf_counter()
            O.tripartite_attention(q[0, h * G:(h + 1) * G], idx[j], k_r, k_e)
            per_head.append(time.perf_counter() - s)
        if len(per_head) >= max_n:
            break
    return per_head


def cpu_baseline(kv, budget_s=20.0):
    """The oracle, as it stands, on the host cores: decode of sampled KV heads
    (scaled to one 8-head step) with numpy's BLAS on every core and on one
    thread, and k-means of one segment (all cores)."""
    import oracle as O
    heads = [0, 1]
    idx = _oracle_index(kv, heads)
    q = S.make_queries(kv, G, seed=10).double().numpy()
    per_head = _oracle_decode_sample(idx, q, heads, budget_s * 0.35)
    step_s = float(np.median(per_head)) * H
    single = None
    try:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=1):
            ph1 = _oracle_decode_sample(idx, q, heads, budget_s * 0.35)
        single = {"value": 1.0 / (float(np.median(ph1)) * H), "unit": UNIT, "cores": 1,
                  "sample": f"{len(ph1)} single-KV-head decodes, scaled x8"}
    except Exception as e:  # threadpoolctl missing: say so
        single = {"unavailable": f"threadpoolctl: {e}"}
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
            "single_thread": single,
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
    C = idx0[0]["C"]
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": ws_n,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": headline_config(ws_n, C, k_r, k_e),
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": _blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "setup_s": time.perf_counter() - t0 - sum(times)}


def run_profile_case(which):
    """Small cases for ncu captures.  "decode": one 128K-token layer of the
    headline geometry (about 1.1 GB on the device), one index build (10
    k-means iterations) and 6 decode calls.  "gather": the 1M-token host
    memory workload at 2 KV heads, 6 steps of select / plan / gather /
    attend (the fetch and admit copies are gather_kernel launches)."""
    import kv_cache_vector_segmented_b200 as R
    dev = torch.device("cuda", 0)
    if which == "decode":
        cfg = R.IndexConfig.make(B, H, G, N, iters=10)
        kv = S.make_kv(B, H, N, seed=0)
        segs = _segment_sizes(R.geometry(cfg))
        ip = S.init_positions([L for L, _ in segs], [k for _, k in segs], B, H, seed=3)
        idx = R.build_index(kv.K.to(dev), kv.V.to(dev), cfg,
                            init_pos=torch.from_numpy(ip).to(dev))
        q = S.make_queries(kv, G, seed=10).to(dev)
        dcfg = R.default_budgets(idx.geom.clusters)
        ws = R.alloc_workspace(R.decode_workspace_bytes(cfg, dcfg), dev)
        for _ in range(6):
            R.decode(q, idx, dcfg, workspace=ws)
        torch.cuda.synchronize()
        assert R.read_device_status(ws) == 0
    else:
        idx, kv = _build_for(R, dev, 1, 2, 4, 1 << 20, seed=51)
        C = idx.geom.clusters
        d = R.default_budgets(C)
        hK, hV = idx.Kp.cpu().pin_memory(), idx.Vp.cpu().pin_memory()
        counts = idx.counts.cpu().numpy().reshape(2, C)
        offsets = idx.offsets.cpu().numpy().reshape(2, C + 1)
        qs = S.drift_queries_device(S.make_queries_device(kv, 4, seed=52), 6, seed=53)
        r, _ = _cfg5_mode(R, dev, 0, idx, d, hK, hV, counts, offsets, qs, 1, "sync")
        assert r["device_status"] == 0
    print(f"profile case {which} done", flush=True)


def run_gather_shapes():
    """Launch-shape sweep of the gather kernel (threads per block x blocks per
    SM) for four copy lists on the 1M-context geometry (8 units): 16-row
    copies from pinned host memory (cache misses), 16-row copies of which 2 %
    are misses (the host-memory workload's usual mix), and 8-row and 16-row
    copies from the device block pool (cache hits).  CUDA events, median of
    5."""
    import kv_cache_vector_segmented_b200 as R
    dev = torch.device("cuda", 0)
    U, M, POOL, EXE = 8, 131072, 65536, 65536
    g = torch.Generator()
    g.manual_seed(9)
    hK = torch.randn((1, U, M, 128), generator=g).to(torch.bfloat16).pin_memory()
    hV = torch.randn((1, U, M, 128), generator=g).to(torch.bfloat16).pin_memory()
    cK = torch.randn((1, U, POOL, 128), device=dev).to(torch.bfloat16)
    cV = torch.randn_like(cK)
    eK = torch.empty((1, U, EXE, 128), dtype=torch.bfloat16, device=dev)
    eV = torch.empty_like(eK)
    ws = R.alloc_workspace(256, dev)
    rng = np.random.default_rng(0)

    def copy_list(host_frac, n_per_unit, rows):
        out = []
        for u in range(U):
            dst = rng.permutation(EXE // rows)[:n_per_unit] * rows
            hsrc = rng.integers(0, M - rows, n_per_unit)
            csrc = rng.permutation(POOL // rows)[:n_per_unit] * rows
            host = rng.random(n_per_unit) < host_frac
            out += [(u, R.SRC_HOST if h else R.SRC_CACHE, int(a if h else c), R.DST_EXEC, int(b),
                     rows) for h, a, c, b in zip(host, hsrc, csrc, dst)]
        return torch.tensor(out, dtype=torch.int32, device=dev)

    lists = {"host_16rows": copy_list(1.0, 400, 16),
             "mixed_16rows_2pct_host": copy_list(0.02, 2000, 16),
             "device_8rows": copy_list(0.0, 4000, 8),
             "device_16rows": copy_list(0.0, 2000, 16)}
    res = {}
    for name, d in lists.items():
        row = {}
        for threads in (64, 128, 256, 512):
            for bps in (1, 2, 4, 8, 16, 32):
                if threads * bps > 2048:
                    continue
                for _ in range(2):
                    R.gather_blocks(d, hK, hV, eK, eV, ws, cK, cV, shape=(threads, bps))
                ts = []
                for _ in range(5):
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record()
                    R.gather_blocks(d, hK, hV, eK, eV, ws, cK, cV, shape=(threads, bps))
                    e1.record()
                    torch.cuda.synchronize()
                    ts.append(e0.elapsed_time(e1) * 1e3)
                row[f"{threads}x{bps}"] = round(float(np.median(ts)), 1)
        host = int(d[:, 1].eq(R.SRC_HOST).sum().item())
        chosen = R.gather_shape(host, d.shape[0])
        res[name] = {"copies": int(d.shape[0]), "us_by_threads_x_blocks_per_sm": row,
                     "best": min(row, key=row.get), "chosen": f"{chosen[0]}x{chosen[1]}"}
    assert R.read_device_status(ws) == 0
    return {"leg": "gather launch shapes", "unit": "us per launch", "lists": res}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=6400)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the config1 / config4 / config5 legs")
    ap.add_argument("--ncu-case", choices=["decode", "gather"], default=None,
                    help="run only the small case used for ncu captures")
    ap.add_argument("--gather-shapes", action="store_true",
                    help="run only the launch-shape sweep of the gather kernel")
    args = ap.parse_args()
    if args.ncu_case:
        run_profile_case(args.ncu_case)
        return
    if args.gather_shapes:
        print(json.dumps(run_gather_shapes()), flush=True)
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
