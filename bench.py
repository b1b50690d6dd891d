#!/usr/bin/env python
"""Benchmark of the SparsePR attention call on one B200 per rank.

A step is one whole SparsePR call (partition, routing, block-sparse attention, probe
rows, fit, apply) on the video-DiT 720p-like workload: 40 heads x 75,600 tokens
(21x45x80 grid), head dim 128, bf16, synthetic seeded latents.  Each rank runs its own
independent call (weak scaling, no data-path collective).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Rank 0 prints one JSON line.  ``--impl reference`` times the fp64 CPU oracle on a
bounded sample of the same workload instead (the reference arm).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SparsePR ms/call & eff. TFLOP/s at 22% pair density; mean rel-L2 err vs dense"
UNIT = "TFLOP/s (dense-equivalent, 4*d*N^2*H per call)"

# DRAM bytes per launch of the dominant kernel from an ncu capture of the same kernel
# build (profiles/attn_tc_kernel_video_4h.md: 301.4 MB on 4 heads), scaled by heads to
# the 40-head launch; None whenever that kernel has changed since the capture.
DOMINANT_TRAFFIC_BYTES = 3.014e9
E2E_GROUPS = 4  # head groups of the host entry point (copies of one overlap the compute of the next)


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", default="video")
    ap.add_argument("--heads", type=int, default=0, help="override the head count (profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the oracle's CPU timing (profiling runs; cpu_baseline is then null)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--study", choices=["ablation", "probe-budget", "routing"], default=None,
                    help="error studies instead of the timed run (one JSON line per variant)")
    return ap.parse_args()


def workload(args):
    from synthetic import CONFIGS
    w = CONFIGS[args.config]
    if args.heads:
        w = w.with_(heads=args.heads)
    return w


def config_block(w, args):
    t, y, x = w.grid
    return {"workload": f"{w.name}: {w.heads} heads x {w.n_tokens} tokens ({t}x{y}x{x} grid), d={w.head_dim}, "
                        f"{w.dtype}, B={w.block}, S={w.n_sampled}, P={w.n_probe}, density={w.density}, "
                        f"lambda={w.ridge_lambda}, r={w.rank}, T={w.kmeans_iters}",
            "batch": w.batch, "heads": w.heads, "tokens": w.n_tokens, "head_dim": w.head_dim,
            "parallelism": f"independent call per rank x{args.gpus}", "seed": args.seed,
            "l2": "inputs (3 x 774 MB bf16) larger than the 126 MB L2; no flush needed"}


def dense_flops(w):
    return 4.0 * w.head_dim * float(w.n_tokens) ** 2 * w.heads * w.batch


def max_over_ranks(seconds, world, device=None):
    """The job's time: the slowest rank's (an all-reduce MAX over the process group);
    the value itself on one rank."""
    if world == 1:
        return seconds
    import torch
    import torch.distributed as dist
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step, world, steps, seconds):
    """Whole-job aggregate (weak scaling): every rank processes the same per-step work,
    so the job's units are units x ranks x steps over the slowest rank's time."""
    return units_per_rank_step * world * steps / seconds


# ------------------------------------------------------------------- CPU oracle sample

def oracle_sample(w, seed=0):
    """Time the fp64 oracle's stages on one head of the workload restricted to its
    first frame and extrapolate to the full call by each stage's cost order.
    Returns (seconds per full call, description, threads)."""
    import numpy as np

    from oracle import sparsepr_oracle as O
    from synthetic import make_inputs
    t_frames, gy, gx = w.grid
    sub = w.with_(grid=(1, gy, gx), heads=1)
    q, k, v = make_inputs(sub, seed)
    q, k, v = (x[0, 0].double().numpy() for x in (q, k, v))
    n_s, n = sub.n_tokens, w.n_tokens
    tau = 1.0 / math.sqrt(w.head_dim)
    s_count = min(w.n_sampled, n_s)
    tm = {}
    t0 = time.perf_counter()
    part = O.partition(q, k, tau, w.block, s_count, w.kmeans_iters)
    tm["partition"] = time.perf_counter() - t0
    kk = O.route_k(n_s, w.block, w.density, w.n_probe)
    t0 = time.perf_counter()
    routes = O.route(part["block_scores"], kk)
    tm["route"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    s = O.sparse_attention(q, k, v, tau, part["key_labels"], part["query_labels"], routes)
    tm["sparse"] = time.perf_counter() - t0
    pidx = O.midpoint_stride(n_s, w.n_probe)
    t0 = time.perf_counter()
    d_probe = O.dense_attention_rows(q, k, v, tau, pidx)
    tm["probes"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    fit = O.fit_residual(s[pidx], d_probe, w.ridge_lambda, w.rank)
    tm["fit"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.apply_residual(s, fit["M"], fit["beta"], pidx, d_probe)
    tm["apply"] = time.perf_counter() - t0
    r = n / n_s
    # partition: N*G*dims with G ~ N and dims S (keys) / G (queries) -> between N^2 and N^3;
    # take N^2 (keys dominate at S fixed).  sparse ~ N*k*B ~ N^2.  probes ~ P*N.  apply ~ N.
    scale = {"partition": r * r, "route": r * r, "sparse": r * r, "probes": r, "fit": 1.0, "apply": r}
    per_head = sum(tm[x] * scale[x] for x in tm)
    full = per_head * w.heads * w.batch
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        threads = 1
    desc = (f"fp64 oracle, 1 head, first frame ({n_s} tokens, S={s_count}, P={w.n_probe}); stage times "
            + ", ".join(f"{x} {tm[x]:.2f}s" for x in tm)
            + f"; extrapolated per stage (partition, route, sparse x(N/n)^2; probes, apply x N/n; fit x1) "
              f"and x{w.heads * w.batch} heads")
    return full, desc, threads


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    times = []
    desc = threads = None
    for i in range(args.warmup + args.steps):
        full, desc, threads = oracle_sample(w, args.seed)
        if i >= args.warmup:
            times.append(full)
    sec = statistics.mean(times)
    value = dense_flops(w) / sec / 1e12
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config_block(w, args),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------- GPU helpers

class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index):
        import torch
        self.proc = None
        self.sel = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.sel = ["-i", uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"]
        except Exception:
            self.sel = []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", *self.sel, f"--query-gpu={','.join(self.FIELDS)}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in out.strip().splitlines():
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[3:]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return float(pk["bf16_tflops_sustained"]), "measured (cuBLAS bf16, sustained)"
    except Exception:
        return 1400.0, "fallback (1.4 PFLOP/s sustained bf16)"


def run_ours(args, w):
    import torch
    import torch.distributed as dist

    import free_block_sparse_response_b200 as spr
    from free_block_sparse_response_b200.build import build
    from synthetic import make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if rank == 0:
        build()
    if world > 1:
        dist.barrier()
    spr.lib()

    cpu_base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu_sec, cpu_desc, cpu_threads = oracle_sample(w, args.seed)
        cpu_base = {"value": dense_flops(w) / cpu_sec / 1e12, "unit": UNIT, "cores": cpu_threads,
                    "kind": "oracle", "sample": cpu_desc}

    q_h, k_h, v_h = make_inputs(w, args.seed + rank)
    q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
    bt, h, n, d = q.shape
    sc = spr.SparsePRConfig(block=w.block, n_sampled=w.n_sampled, n_probe=w.n_probe, kmeans_iters=w.kmeans_iters,
                            rank=w.rank, density=w.density, ridge_lambda=w.ridge_lambda)
    ws = spr.new_workspace(bt, h, n, d, sc, dev)
    o = torch.empty_like(q)
    fused = spr.fused_supported(q, sc)
    # probe-first order with the correction fused into the attention kernel (the call
    # spr.attention makes for this shape); the unfused order otherwise
    stages = (["partition", "route", "probe_dense", "fit_residual", "sparse_attn_apply"] if fused else
              ["partition", "route", "sparse_attn", "probe_dense", "fit_residual", "apply_residual"])

    def step(record=None):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(stages) + 1)] if record is not None else None
        mark = (lambda i: ev[i].record()) if ev else (lambda i: None)
        mark(0)
        part = spr.partition(q, k, sc, ws)
        mark(1)
        rt, kk, pairs = spr.route(part, n, sc, ws)
        mark(2)
        pidx = spr.probe_rows(n, sc.n_probe, bt, h, dev)
        if fused:
            p_out, p_sparse = spr.probe_dense(q, k, v, pidx, part, rt, kk, sc, ws)
            mark(3)
            m, beta = spr.fit_residual(p_sparse, p_out, sc, ws)
            mark(4)
            spr.sparse_attn_apply(q, k, v, part, rt, kk, sc, m, beta, pidx, p_out, ws, out=o)
            mark(5)
        else:
            s_out = spr.sparse_attn(q, k, v, part, rt, kk, sc, ws=ws)
            mark(3)
            p_out, p_sparse = spr.probe_dense(q, k, v, pidx, part, rt, kk, sc, ws)
            mark(4)
            m, beta = spr.fit_residual(p_sparse, p_out, sc, ws)
            mark(5)
            spr.apply_residual(s_out, m, beta, pidx, p_out, out_dtype=q.dtype, out=o)
            mark(6)
        if ev:
            record.append(ev)
        return {"part": part, "route": rt, "pidx": pidx, "pairs": pairs, "k": kk}

    for _ in range(args.warmup):
        step()
    spr.check(ws)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = ClockSampler(local)
    clocks.start()
    launches0 = spr.launch_count()
    events = []
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    spr.kernel_timing_read()  # forget pairs from before the timed region
    spr.kernel_timing(True)   # event pair around each attention kernel launch
    t_start.record()
    for _ in range(args.steps):
        last = step(events)
    t_end.record()
    torch.cuda.synchronize()
    spr.kernel_timing(False)
    attn_kernel_ms, attn_kernel_n = spr.kernel_timing_read()
    launches = spr.launch_count() - launches0
    clk = clocks.stop()
    spr.check(ws)
    elapsed = max_over_ranks(t_start.elapsed_time(t_end) / 1e3, world, dev)
    if world > 1:
        dist.barrier()
    ms_step = elapsed / args.steps * 1e3
    stage_ms = {s: statistics.mean(e[i].elapsed_time(e[i + 1]) for e in events) for i, s in enumerate(stages)}
    step_ms = [round(e[0].elapsed_time(e[-1]), 3) for e in events]  # per timed step, first stage to last

    # ---- dominant kernel roofline (block-sparse attention: 4*d flops per routed pair)
    pairs = last["pairs"].to(torch.float64).sum().item()
    sparse_pairs = pairs - float(w.n_probe) * n * h * bt
    sparse_flops = 4.0 * d * sparse_pairs
    # the attention kernel's own launches, timed by the library's event pairs on the
    # launch stream (the stage also holds the copy of K and V into group order)
    t_sparse = attn_kernel_ms / max(attn_kernel_n, 1) / 1e3
    peak, peak_src = measured_peak()
    achieved = sparse_flops / t_sparse / 1e12 if t_sparse > 0 else None
    kname = ("attn_tc_kernel<false, true> (block-sparse attention + fused correction, tcgen05)" if fused else
             "attn_tc_kernel<false, false> (block-sparse attention, tcgen05)")
    roofline = {"kernel": kname, "bound": "tensor", "achieved": achieved,
                "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak if achieved is not None else None, "traffic": DOMINANT_TRAFFIC_BYTES if (args.config == "video" and not args.heads and fused) else None,
                "peak_source": peak_src, "kernel_ms": t_sparse * 1e3, "kernel_launches_timed": attn_kernel_n,
                "per_launch_flops": sparse_flops}
    if attn_kernel_n == 0:  # shapes outside the tensor-core kernel (fp32, d = 64, B = 64)
        roofline["note"] = "no tensor-core attention launch in this configuration"

    # ---- e2e through host buffers (pinned), copies inside the timed region: the library's
    # host entry point, heads in groups whose copies overlap the neighbouring groups' compute
    qp, kp, vp = (t.contiguous().pin_memory() for t in (q_h, k_h, v_h))
    op = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    groups = min(E2E_GROUPS, bt * h)
    ws_host = spr.host_workspace(qp, sc, groups, device=dev)
    spr.attention_host(qp, kp, vp, sc, out=op, groups=groups, ws=ws_host)
    torch.cuda.synchronize()
    spr.check(ws_host)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        spr.attention_host(qp, kp, vp, sc, out=op, groups=groups, ws=ws_host)
    e1.record()
    torch.cuda.synchronize()
    spr.check(ws_host)
    del ws_host
    e2e_s = max_over_ranks(e0.elapsed_time(e1) / 1e3, world, dev)
    h2d = sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h))
    d2h = o.numel() * o.element_size()

    # ---- dense comparators and the error metric (outside the timed regions)
    # the uncorrected sparse output of the last timed call's decisions (metric only)
    s_last = spr.sparse_attn(q, k, v, last["part"], last["route"], last["k"], sc, ws=ws)
    dense = torch.empty(bt, h, n, d, dtype=torch.float32, device=dev)
    spr.dense_attn(q, k, v, block=w.block, out=dense)
    torch.cuda.synchronize()
    de0, de1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    de0.record()
    for _ in range(2):
        spr.dense_attn(q, k, v, block=w.block, out=dense)
    de1.record()
    torch.cuda.synchronize()
    dense_ms = de0.elapsed_time(de1) / 2
    sdpa_ms = None
    try:
        import torch.nn.functional as F
        F.scaled_dot_product_attention(q, k, v)
        torch.cuda.synchronize()
        se0, se1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        se0.record()
        for _ in range(2):
            F.scaled_dot_product_attention(q, k, v)
        se1.record()
        torch.cuda.synchronize()
        sdpa_ms = se0.elapsed_time(se1) / 2
    except Exception:
        sdpa_ms = None
    pidx = spr.probe_rows(n, sc.n_probe, bt, h, dev)
    err = spr.row_errors(o, dense, pidx)
    err_s = spr.row_errors(s_last, dense, pidx)

    def summary(e):
        means, p99s = [], []
        for hh in range(h):
            x = e[0, hh]
            x = x[~torch.isnan(x)]
            xs, _ = torch.sort(x)
            means.append(float(xs.double().mean()))
            p99s.append(float(xs[max(math.ceil(0.99 * xs.numel()) - 1, 0)]))
        return statistics.mean(means), statistics.mean(p99s)

    err_mean, err_p99 = summary(err)
    s_mean, s_p99 = summary(err_s)
    spr.check(ws)

    value = job_throughput(dense_flops(w), world, args.steps, elapsed) / 1e12
    e2e_value = job_throughput(dense_flops(w), world, args.steps, e2e_s) / 1e12
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded video-token latents)",
                "config": config_block(w, args),
                "err": {"mean_rel_l2_unprobed": err_mean, "p99_rel_l2_unprobed": err_p99,
                        "uncorrected_sparse_mean": s_mean, "uncorrected_sparse_p99": s_p99,
                        "reference": "same-family dense attention, fp32 output"},
                "density": pairs / (float(n) ** 2 * h * bt), "k": last["k"],
                "stage_ms": stage_ms, "step_ms": step_ms, "dense_ms": dense_ms, "sdpa_ms": sdpa_ms,
                "speedup_vs_dense": dense_ms / ms_step,
                "roofline": roofline, "cpu_baseline": cpu_base,
                "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                        "ms_per_step": e2e_s / args.steps * 1e3, "api": "sparsepr_attention_host",
                        "head_groups": groups},
                "gpu_launches": launches, "clocks": clk}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ------------------------------------------------------------------- error studies

def _gpu_modules():
    import torch
    import free_block_sparse_response_b200 as spr
    return torch, spr


def _err_summary(e):
    """Head-averaged mean and p99 of the per-row errors (NaN rows = probe rows skipped)."""
    torch, _ = _gpu_modules()
    means, p99s = [], []
    for b in range(e.shape[0]):
        for hh in range(e.shape[1]):
            x = e[b, hh]
            x = x[~torch.isnan(x)]
            xs, _ = torch.sort(x)
            means.append(float(xs.double().mean()))
            p99s.append(float(xs[max(math.ceil(0.99 * xs.numel()) - 1, 0)]))
    return statistics.mean(means), statistics.mean(p99s)


def _study_inputs(args, w):
    from synthetic import make_inputs
    torch, spr = _gpu_modules()
    dev = torch.device("cuda", 0)
    q, k, v = (t.to(dev) for t in make_inputs(w, args.seed))
    bt, h, n, d = q.shape
    dense = torch.empty(bt, h, n, d, dtype=torch.float32, device=dev)
    spr.dense_attn(q, k, v, block=w.block, out=dense)
    return q, k, v, dense


def _uncorrected(q, k, v, cfg, ws):
    """Block-sparse output without residual correction, its k from the pair budget
    without probe rows (equal executed-pair density to the corrected call)."""
    _, spr = _gpu_modules()
    n = q.shape[2]
    cfg0 = dataclasses.replace(cfg, n_probe=0)
    part = spr.partition(q, k, cfg0, ws)
    rt, kk, pairs = spr.route(part, n, cfg0, ws)
    return spr.sparse_attn(q, k, v, part, rt, kk, cfg0, ws=ws), kk, pairs


def run_study_ablation(args, w):
    """Error of the semantic baseline and of each SparsePR component against the
    same-family dense output: semantic partition without correction (the comparator
    of the pages' error reduction), semantic partition + probe fit, Response-Coupled
    Partitioning without correction, and the full method.  Errors over the rows that
    are not probe rows of the full method; equal executed-pair density throughout."""
    _, spr = _gpu_modules()
    q, k, v, dense = _study_inputs(args, w)
    bt, h, n, d = q.shape
    base = spr.SparsePRConfig(block=w.block, n_sampled=w.n_sampled, n_probe=w.n_probe, kmeans_iters=w.kmeans_iters,
                              rank=w.rank, density=w.density, ridge_lambda=w.ridge_lambda)
    ws = spr.new_workspace(bt, h, n, d, base, q.device)
    pidx = spr.probe_rows(n, w.n_probe, bt, h, q.device)
    rows = []
    for mode, name in ((spr.PARTITION_SEMANTIC, "semantic"), (spr.PARTITION_RESPONSE, "response-coupled")):
        cfg = dataclasses.replace(base, partition_mode=mode)
        s, kk0, pairs0 = _uncorrected(q, k, v, cfg, ws)
        m, p = _err_summary(spr.row_errors(s, dense, pidx))
        rows.append({"variant": f"{name} partition, no correction", "mean_rel_l2": m, "p99_rel_l2": p, "k": kk0,
                     "density": float(pairs0.double().sum()) / (float(n) ** 2 * h * bt)})
        o, parts = spr.attention(q, k, v, cfg, ws=ws, return_parts=True)
        m, p = _err_summary(spr.row_errors(o, dense, pidx))
        rows.append({"variant": f"{name} partition + probe-fitted correction", "mean_rel_l2": m, "p99_rel_l2": p,
                     "k": parts["k"],
                     "density": float(parts["executed_pairs"].double().sum()) / (float(n) ** 2 * h * bt)})
    spr.check(ws)
    ref = rows[0]["mean_rel_l2"]
    for r in rows:
        r["mean_error_reduction_vs_semantic_uncorrected"] = 1.0 - r["mean_rel_l2"] / ref
        r.update({"study": "ablation", "workload": config_block(w, args)["workload"], "seed": args.seed,
                  "reference": "same-family dense attention, fp32 output"})
        print(json.dumps(r), flush=True)


def run_study_probe_budget(args, w):
    """Mean and p99 unprobed-row error against the probe budget P (k re-derived from
    the pair budget for each P), with the uncorrected output at the same density."""
    _, spr = _gpu_modules()
    q, k, v, dense = _study_inputs(args, w)
    bt, h, n, d = q.shape
    for P in (32, 64, 128, 256, 512):
        cfg = spr.SparsePRConfig(block=w.block, n_sampled=w.n_sampled, n_probe=P, kmeans_iters=w.kmeans_iters,
                                 rank=w.rank, density=w.density, ridge_lambda=w.ridge_lambda)
        ws = spr.new_workspace(bt, h, n, d, cfg, q.device)
        pidx = spr.probe_rows(n, P, bt, h, q.device)
        o, parts = spr.attention(q, k, v, cfg, ws=ws, return_parts=True, fused=False)
        m, p = _err_summary(spr.row_errors(o, dense, pidx))
        mu, pu = _err_summary(spr.row_errors(parts["S"], dense, pidx))
        spr.check(ws)
        print(json.dumps({"study": "probe-budget", "workload": config_block(w, args)["workload"], "P": P,
                          "k": parts["k"], "density": float(parts["executed_pairs"].double().sum()) /
                          (float(n) ** 2 * h * bt), "mean_rel_l2": m, "p99_rel_l2": p,
                          "uncorrected_mean_rel_l2": mu, "uncorrected_p99_rel_l2": pu,
                          "mean_error_reduction": 1.0 - m / mu, "seed": args.seed}), flush=True)
        del ws


def run_study_routing(args, w):
    """Error of the three block-routing score readings (centroid, size-corrected, LSE)
    under the two splits of the pair budget (uniform k per block; one budget per head
    spent on the best pairs), with and without the probe-fitted correction, and the
    device time of one whole call (the default fused order) for each."""
    torch, spr = _gpu_modules()
    q, k, v, dense = _study_inputs(args, w)
    bt, h, n, d = q.shape
    for budget, bname in ((spr.BUDGET_UNIFORM, "uniform"), (spr.BUDGET_GLOBAL, "global")):
        for mode, name in ((spr.ROUTE_CENTROID, "centroid"), (spr.ROUTE_SIZE_CORRECTED, "size-corrected"),
                           (spr.ROUTE_LSE, "lse")):
            cfg = spr.SparsePRConfig(block=w.block, n_sampled=w.n_sampled, n_probe=w.n_probe,
                                     kmeans_iters=w.kmeans_iters, rank=w.rank, density=w.density,
                                     ridge_lambda=w.ridge_lambda, route_scores=mode, route_budget=budget)
            ws = spr.new_workspace(bt, h, n, d, cfg, q.device)
            pidx = spr.probe_rows(n, w.n_probe, bt, h, q.device)
            o, parts = spr.attention(q, k, v, cfg, ws=ws, return_parts=True, fused=False)
            m, p = _err_summary(spr.row_errors(o, dense, pidx))
            mu, pu = _err_summary(spr.row_errors(parts["S"], dense, pidx))
            spr.check(ws)
            del o, parts
            spr.attention(q, k, v, cfg, ws=ws)  # warm
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            spr.attention(q, k, v, cfg, ws=ws)
            e1.record()
            torch.cuda.synchronize()
            spr.check(ws)
            pairs = spr.route(spr.partition(q, k, cfg, ws), n, cfg, ws)[2]
            print(json.dumps({"study": "routing", "scores": name, "budget": bname,
                              "workload": config_block(w, args)["workload"],
                              "density": float(pairs.double().sum()) / (float(n) ** 2 * h * bt),
                              "mean_rel_l2": m, "p99_rel_l2": p, "uncorrected_mean_rel_l2": mu,
                              "uncorrected_p99_rel_l2": pu, "call_ms": e0.elapsed_time(e1), "seed": args.seed}),
                  flush=True)
            del ws


def main():
    args = parse_args()
    w = workload(args)
    if args.study == "ablation":
        run_study_ablation(args, w)
    elif args.study == "probe-budget":
        run_study_probe_budget(args, w)
    elif args.study == "routing":
        run_study_routing(args, w)
    elif args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
