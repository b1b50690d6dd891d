#!/usr/bin/env python
"""Benchmark of the SparsePR attention call on one B200 per rank.

A step is one whole SparsePR call (partition, routing, block-sparse attention, probe
rows, fit, apply) on the video-DiT 720p-like workload: 40 heads x 75,600 tokens
(21x45x80 grid), head dim 128, bf16, synthetic seeded latents.  On N GPUs the call's
heads are split into N contiguous slices, one per rank (heads are independent problems:
no data-path collective; the output stays sharded by head, as in head-parallel DiTs);
the call's time is the slowest rank's (strong scaling).  ``--scaling weak`` instead
gives every rank a whole call of its own.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

``--gpus N`` without a torchrun environment re-launches itself under
``torch.distributed.run`` with N ranks.  Rank 0 prints one JSON line.
``--impl reference`` times the fp64 CPU oracle on a bounded sample of the same
workload instead (the reference arm; rank 0 only).
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
    ap.add_argument("--scaling", choices=["strong", "weak"], default="strong",
                    help="strong: one call's heads split over the ranks; weak: a whole call per rank")
    return ap.parse_args()


def workload(args):
    from synthetic import CONFIGS
    w = CONFIGS[args.config]
    if args.heads:
        w = w.with_(heads=args.heads)
    return w


def head_slice(heads, world, rank):
    """Contiguous heads [lo, hi) of `rank` when one call's heads are split over `world`
    ranks; slice sizes differ by at most one."""
    if not 1 <= world <= heads or not 0 <= rank < world:
        raise ValueError(f"cannot split {heads} heads over {world} ranks (rank {rank})")
    return heads * rank // world, heads * (rank + 1) // world


def parallelism(w, world, scaling):
    if scaling == "weak":
        return f"independent call per rank x{world}"
    sizes = [hi - lo for lo, hi in (head_slice(w.heads, world, r) for r in range(world))]
    return f"heads split over {world} rank(s), contiguous slices of {sizes} heads"


def config_block(w, args, world=1):
    t, y, x = w.grid
    return {"workload": f"{w.name}: {w.heads} heads x {w.n_tokens} tokens ({t}x{y}x{x} grid), d={w.head_dim}, "
                        f"{w.dtype}, B={w.block}, S={w.n_sampled}, P={w.n_probe}, density={w.density}, "
                        f"lambda={w.ridge_lambda}, r={w.rank}, T={w.kmeans_iters}",
            "batch": w.batch, "heads": w.heads, "tokens": w.n_tokens, "head_dim": w.head_dim,
            "parallelism": parallelism(w, world, args.scaling), "seed": args.seed,
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


def sum_over_ranks(value, world, device=None):
    """Sum of a per-rank number over the process group (the value itself on one rank)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def gather_head_stats(stats, world):
    """Per-head statistics of every rank's slice, concatenated in head order (ranks hold
    contiguous slices in rank order); outside the timed region."""
    if world == 1:
        return list(stats)
    import torch.distributed as dist
    parts = [None] * world
    dist.all_gather_object(parts, list(stats))
    return [x for part in parts for x in part]


# ------------------------------------------------------------------- CPU oracle sample

def oracle_inputs(w, seed=0):
    """The first head of the seeded workload as fp64 arrays (the oracle's inputs)."""
    from synthetic import make_inputs
    q, k, v = make_inputs(w, seed, heads=1)
    return tuple(x[0, 0].double().numpy() for x in (q, k, v))


def oracle_sample(w, seed=0, group_sample=16, block_div=64, inputs=None):
    """Time the fp64 oracle on one FULL head of the workload, stage by stage, and scale
    to the whole call.  Every scale factor counts identical units of work:

    * the k-means distances loop over the groups, each group's pass the same full-size
      work (all N rows): timed on `group_sample` evenly spaced groups, scaled by G / that;
    * the sparse attention loops over query blocks of equal work: timed on 1/block_div
      of the blocks, scaled by N / their rows;
    * the profiles, group means, capacity fill, coordinates, routing, probe rows, fit and
      apply run in full (the fill on a full-size distance matrix formed outside the
      timed region; only its shape and values matter to the fill's cost);
    * one k-means iteration per side is timed and counted T times;
    * heads are independent problems: x heads.
    Returns (seconds per full call, description, threads)."""
    import numpy as np

    from oracle import sparsepr_oracle as O
    q, k, v = oracle_inputs(w, seed) if inputs is None else inputs
    n, B, T = w.n_tokens, w.block, w.kmeans_iters
    G = O.n_groups(n, B)
    tau = 1.0 / math.sqrt(w.head_dim)
    rng = np.random.default_rng(seed)
    gsel = np.unique(np.linspace(0, G - 1, min(group_sample, G)).astype(np.int64))
    tm = {}

    def timed(name, fn, scale=1.0):
        t0 = time.perf_counter()
        out = fn()
        tm[name] = tm.get(name, 0.0) + (time.perf_counter() - t0) * scale
        return out

    def fill_input(x, cent):   # the full fp32 distance matrix the fill takes (untimed)
        return ((x * x).sum(1)[:, None] - 2.0 * (x @ cent.T) + (cent * cent).sum(1)[None, :]).astype(np.float32)

    def kmeans_side(name, x):
        labels = timed(f"{name} k-means", lambda: O.chunk_labels(n, B))
        cent = timed(f"{name} k-means", lambda: O.group_means(x, labels, G))
        if T == 0:
            return labels
        O.squared_distances(x, cent[gsel[:2]])   # untimed: the first large allocations of a process are slower
        timed(f"{name} k-means", lambda: O.squared_distances(x, cent[gsel]), G / gsel.size * T)
        d32 = fill_input(x, cent)
        labels = timed(f"{name} k-means", lambda: O.fill(d32, B), T)
        timed(f"{name} k-means", lambda: O.group_means(x, labels, G, previous=cent), T)
        return labels

    sidx = O.midpoint_stride(n, w.n_sampled)
    prof = timed("key k-means", lambda: O.key_response_profiles(q, k, sidx, tau))
    kl = kmeans_side("key", prof)
    mu = timed("query k-means", lambda: O.group_means(k, kl, G))
    coords = timed("query k-means", lambda: tau * (q @ mu.T))
    ql = kmeans_side("query", coords)
    scores = timed("route", lambda: O.group_means(coords, ql, G).astype(np.float32))
    kk = O.route_k(n, B, w.density, w.n_probe)
    routes = timed("route", lambda: O.route(scores, kk))
    blocks = np.sort(rng.choice(G, max(G // block_div, 1), replace=False))
    brows = np.flatnonzero(np.isin(ql, blocks))
    s_rows = timed("sparse", lambda: O.sparse_attention(q[brows], k, v, tau, kl, ql[brows], routes),
                   n / max(brows.size, 1))
    pidx = O.midpoint_stride(n, w.n_probe)
    d_probe = timed("probes", lambda: O.dense_attention_rows(q, k, v, tau, pidx))
    # the fit takes the probe rows' sparse outputs (computed untimed; the sampled
    # attention above already counts their cost within the rows' share)
    s_probe = O.sparse_attention(q[pidx], k, v, tau, kl, ql[pidx], routes)
    fit = timed("fit", lambda: O.fit_residual(s_probe, d_probe, w.ridge_lambda, w.rank))
    s_full = np.zeros((n, w.head_dim))
    s_full[brows] = s_rows
    timed("apply", lambda: O.apply_residual(s_full, fit["M"], fit["beta"], pidx, d_probe))
    per_head = sum(tm.values())
    full = per_head * w.heads * w.batch
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        threads = 1
    desc = (f"fp64 oracle on one full head ({n} tokens, G={G}, S={w.n_sampled}, P={w.n_probe}, T={T}); "
            f"k-means distances timed on {gsel.size} of the {G} groups (each a full pass over the rows) and "
            f"scaled by G/{gsel.size}, sparse attention on 1/{block_div} of the query blocks scaled by rows, "
            f"one k-means iteration per side x T, the rest in full; "
            f"per-head stage seconds " + ", ".join(f"{x} {tm[x]:.1f}" for x in tm)
            + f"; x{w.heads * w.batch} heads (independent problems)")
    return full, desc, threads


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    times = []
    desc = threads = None
    inputs = oracle_inputs(w, args.seed)
    for i in range(args.warmup + args.steps):
        full, desc, threads = oracle_sample(w, args.seed, inputs=inputs)
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
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: the SparsePR call needs a CUDA device (none visible); "
                         "the CPU oracle is timed with --impl reference")
    strong = args.scaling == "strong"
    lo, hi = head_slice(w.heads, world, rank) if strong else (0, w.heads)
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

    if strong:   # this rank's contiguous head slice of the one seeded call
        q_h, k_h, v_h = (t[:, lo:hi].contiguous() for t in make_inputs(w, args.seed, heads=hi))
    else:        # a whole call of its own
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
                "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak if achieved is not None else None, "traffic": (DOMINANT_TRAFFIC_BYTES * (hi - lo) / w.heads
                            if (args.config == "video" and not args.heads and fused) else None),
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
    h2d = sum_over_ranks(float(sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h))), world, dev)
    d2h = sum_over_ranks(float(o.numel() * o.element_size()), world, dev)

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
    dense_ms = max_over_ranks(de0.elapsed_time(de1) / 2, world, dev)
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
        sdpa_ms = float("nan")
    sdpa_ms = max_over_ranks(sdpa_ms, world, dev)   # every rank takes the collective
    sdpa_ms = None if math.isnan(sdpa_ms) else sdpa_ms
    pidx = spr.probe_rows(n, sc.n_probe, bt, h, dev)
    err = spr.row_errors(o, dense, pidx)
    err_s = spr.row_errors(s_last, dense, pidx)

    def per_head(e):
        """(mean, nearest-rank p99) of every head's unprobed-row errors on this rank."""
        out = []
        for hh in range(h):
            x = e[0, hh]
            x = x[~torch.isnan(x)]
            xs, _ = torch.sort(x)
            out.append((float(xs.double().mean()), float(xs[max(math.ceil(0.99 * xs.numel()) - 1, 0)])))
        return out

    def summary(stats):
        return statistics.mean(m for m, _ in stats), statistics.mean(p for _, p in stats)

    err_mean, err_p99 = summary(gather_head_stats(per_head(err), world))
    s_mean, s_p99 = summary(gather_head_stats(per_head(err_s), world))
    spr.check(ws)
    pairs_all = sum_over_ranks(pairs, world, dev)
    heads_all = w.heads * (world if not strong else 1)

    # strong: the ranks together make one call; weak: one call per rank
    calls = 1 if strong else world
    value = job_throughput(dense_flops(w), calls, args.steps, elapsed) / 1e12
    e2e_value = job_throughput(dense_flops(w), calls, args.steps, e2e_s) / 1e12
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": args.scaling,
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded video-token latents)",
                "config": config_block(w, args, world),
                "err": {"mean_rel_l2_unprobed": err_mean, "p99_rel_l2_unprobed": err_p99,
                        "uncorrected_sparse_mean": s_mean, "uncorrected_sparse_p99": s_p99,
                        "reference": "same-family dense attention, fp32 output"},
                "density": pairs_all / (float(n) ** 2 * heads_all * bt), "k": last["k"],
                "stage_ms": stage_ms, "step_ms": step_ms, "rank0_heads": [lo, hi],
                "dense_ms": dense_ms, "sdpa_ms": sdpa_ms,
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
    the pair budget for each P), with the uncorrected output at the same density, under
    the two readings of the ridge scale: lambda absolute (on a Gram whose weights sum to
    P), and lambda relative to tr(X_c^T W X_c) / d (RIDGE_RELATIVE); the partition,
    routes, probe rows and sparse output are shared, only the fit and apply differ."""
    torch, spr = _gpu_modules()
    q, k, v, dense = _study_inputs(args, w)
    bt, h, n, d = q.shape
    for P in (32, 64, 128, 256, 512):
        if P > n:
            continue
        cfg = spr.SparsePRConfig(block=w.block, n_sampled=w.n_sampled, n_probe=P, kmeans_iters=w.kmeans_iters,
                                 rank=w.rank, density=w.density, ridge_lambda=w.ridge_lambda)
        ws = spr.new_workspace(bt, h, n, d, cfg, q.device)
        pidx = spr.probe_rows(n, P, bt, h, q.device)
        o, parts = spr.attention(q, k, v, cfg, ws=ws, return_parts=True, fused=False)
        mu, pu = _err_summary(spr.row_errors(parts["S"], dense, pidx))
        for ridge, flag in (("absolute", 0), ("relative", spr.RIDGE_RELATIVE)):
            rcfg = dataclasses.replace(cfg, weight_mode=cfg.weight_mode | flag)
            m_, b_ = spr.fit_residual(parts["probe_sparse"], parts["probe_out"], rcfg, ws)
            o_r = spr.apply_residual(parts["S"], m_, b_, parts["probe_idx"], parts["probe_out"], out_dtype=q.dtype)
            m, p = _err_summary(spr.row_errors(o_r, dense, pidx))
            spr.check(ws)
            print(json.dumps({"study": "probe-budget", "workload": config_block(w, args)["workload"], "P": P,
                              "ridge": ridge, "lambda": w.ridge_lambda,
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


def relaunch_under_torchrun(args):
    """`--gpus N` (N > 1) outside a torchrun environment: run this same command line as N
    ranks of one node (rendezvous on 127.0.0.1); returns their exit status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    args = parse_args()
    w = workload(args)
    world = int(os.environ.get("WORLD_SIZE", "0"))
    if args.impl == "ours" and args.study is None:
        if world == 0 and args.gpus > 1:
            sys.exit(relaunch_under_torchrun(args))
        if world > 1 and world != args.gpus:
            raise SystemExit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}")
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
