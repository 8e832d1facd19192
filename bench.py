#!/usr/bin/env python
"""Benchmark of the Veda-style block-sparse attention hot path on B200.

One step = one full pass of the path over one synthetic layer call:
tile pool + selector projection -> tile scores (tensor cores) + fixed-budget
top-k -> block-sparse attention (the stages veda_attn runs), inputs resident
in HBM.  Default workload: the 1344x768, 24 fps, 5.17 s landscape clip
(31 x 48 x 84 = 124,992 video tokens, 32 heads, head dim 128, tile 128,
90% sparsity = 98 kept tiles, 512 text + 256 audio dense keys), bf16.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   (times the CPU oracle instead)

Prints one JSON line on rank 0.  Multi-GPU (torchrun): by default every rank
runs its own independent layer call (weak scaling); with --split heads the
heads of one call are split into contiguous ranges, one per rank (strong
scaling).  Neither has a data-path collective; the timed region is bracketed
by barriers and the max over ranks is reported.
"""
from __future__ import annotations

import argparse
import atexit
import dataclasses
import datetime
import json
import os
import statistics
import subprocess
import sys
import time
from datetime import timedelta

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "ms per sparse-attn call; kept-block TFLOP/s vs bf16 peak at 90%/95% sparsity"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["veda", "reference"], default="veda")
    ap.add_argument("--workload", default="t2v_5.17s", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--budget", type=int, default=0, help="override the video budget")
    ap.add_argument("--heads", type=int, default=0, help="override the head count (smaller profiling cases)")
    ap.add_argument("--simt", action="store_true", help="use the SIMT attention kernel")
    ap.add_argument("--unfused-selection", action="store_true",
                    help="time the three-kernel selection (fp32 SIMT scores, then the warp-per-row top-k)")
    ap.add_argument("--onchip-selection", action="store_true",
                    help="time the on-chip selection (tensor-core scores recomputed per pass, no score matrix)")
    ap.add_argument("--split", choices=["calls", "heads"], default="calls",
                    help="N GPUs: one independent layer call per GPU (weak scaling), or the heads of one "
                         "call split into N contiguous ranges, no collective (strong scaling)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ncu", action="store_true", help="short run for profiler captures (no extras)")
    ap.add_argument("--dense-queries", type=int, default=0, metavar="ROWS",
                    help="time veda_dense_query_attn instead: ROWS non-video query rows over every key")
    return ap.parse_args()


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) per launch of the
# attention kernel in its current form (L2 evict-last K/V loads, evict-first
# Q loads and O stores), from one ncu capture of 8 of the 32 heads of each
# workload, scaled by the units processed (x4) to the full launch:
#   t2v_5.17s  1.2719 GB read + 0.2537 GB written = 1.5256 GB (8 heads)
#   t2v_14.38s 22.7348 GB read + 0.7642 GB written = 23.4990 GB (8 heads)
# Other workloads have no capture: null.
ATTN_TRAFFIC = {("t2v_5.17s", 32, 98): 1.5256e9 * 4, ("t2v_14.38s", 32, 138): 23.4990e9 * 4}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi samples every 100 ms, started before the warm-up so that it
    is running when the timed region begins; only the samples whose
    timestamps fall inside the timed region (wall clock) are summarised."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.ident = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.ident = None

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.ident:
            cmd += ["-i", self.ident]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        proc = self.proc
        atexit.register(lambda: proc.poll() is None and proc.kill())   # no sampler outlives the run

    def stop(self, t0: float, t1: float):
        """Summary of the samples taken between wall-clock times t0 and t1."""
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        inside = [r for r in rows if t0 <= r[0] <= t1]
        if not inside and rows:   # a region shorter than the sampling period: the nearest sample
            inside = [min(rows, key=lambda r: abs(r[0] - 0.5 * (t0 + t1)))]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({nm for r in inside for nm, val in zip(names, r[3]) if val.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[1] for r in inside) if inside else None,
                "sm_max_mhz": max(r[2] for r in inside) if inside else None,
                "reasons": reasons, "samples": len(inside)}


# ---------------------------------------------------------------------------
# CPU oracle on a bounded sample (the cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------

def oracle_units(w, seed=0):
    """The fixed attention sample of the oracle baseline: at least 64 (b, h,
    query tile) units and at least four per host core, so that every core
    stays busy and the time scales linearly to the full call; the first tile
    and the last (padded) tile are always in it."""
    import numpy as np
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    n = min(w.B * w.H * w.n_q_tiles, max(64, 4 * cores))
    units = [(0, 0, 0), (w.B - 1, w.H - 1, w.n_q_tiles - 1)]
    rng = np.random.default_rng(seed)
    seen = set(units)
    while len(units) < n:
        u = (int(rng.integers(w.B)), int(rng.integers(w.H)), int(rng.integers(w.n_q_tiles)))
        if u not in seen:
            seen.add(u)
            units.append(u)
    return units


def oracle_sample(w, host, units):
    """Time the oracle (fp64 C, OpenMP) on one bounded sample of the call:
    selection (pool -> project -> score -> top-k) of every head in full, and
    attention on the fixed `units`; the attention time is extrapolated
    linearly to all (b, h, query tile) units.  Returns (ms per call, threads,
    description)."""
    import oracle
    oracle.build()
    t0 = time.perf_counter()
    sel = oracle.select_tiles(host, w.T, w.budget_video, w.budget_ref if w.ref_frames else 0)
    t_sel = time.perf_counter() - t0
    t0 = time.perf_counter()
    oracle.attend_units(host, w.T, sel["idx_v"], sel.get("idx_r"), units)
    t_att = time.perf_counter() - t0
    total_units = w.B * w.H * w.n_q_tiles
    ms = (t_sel + t_att * (total_units / len(units))) * 1e3
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    threads = min(int(os.environ.get("OMP_NUM_THREADS", cores)), cores)
    sample = (f"oracle (fp64 C, OpenMP, {threads} threads): selection of all {w.H} heads in full "
              f"({t_sel:.2f} s) and attention on a fixed sample of {len(units)} of {total_units} "
              f"(b, h, query tile) units including the first and the last (padded) tile ({t_att:.2f} s), "
              f"attention extrapolated linearly to one call")
    return ms, threads, sample


def host_copy(g):
    return {k: v.cpu().contiguous() for k, v in g.items()}


# ---------------------------------------------------------------------------

def max_over_ranks(dist, values, device):
    """Element-wise max of a list of floats over all ranks (no-op when not
    distributed)."""
    if dist is None:
        return list(values)
    t = torch.tensor(list(values), device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def head_range(H, n, rank):
    """Heads [h0, h1) of `rank` when the H heads of one call are split into n
    contiguous, near-equal ranges (every head is an independent problem)."""
    return rank * H // n, (rank + 1) * H // n


def head_slice(g, h0, h1):
    """The inputs of heads [h0, h1): strided views of the [B, N, H, d]
    tensors (the library takes any 16-byte strides) and of the [H, d, r]
    selector weights."""
    return {k: (v[h0:h1] if k in ("w_q", "w_k") else v[:, :, h0:h1]) for k, v in g.items()}


def bench_config(w, n, simt=False, split="calls"):
    """The `config` object of the JSON line (identical in both arms)."""
    par = (f"{n} independent layer calls (one per GPU)" if split == "calls" or n == 1 else
           f"the {w.H} heads of one call split over {n} GPUs (contiguous ranges, no collective)")
    return dict(w.describe(), **{
        "kept_tflop_per_call": round(w.kept_flops() / 1e12, 3),
        "parallelism": par,
        "l2": "inputs larger than L2 (Q, K, V of one call exceed 126 MB each)",
        "attention_kernel": "simt" if (simt or w.dtype != "bf16") else "tcgen05",
    })


def make_problem(veda, w, g, simt=False, flags=0):
    return veda.Problem(g["q"], g["k"], g["v"], tile=w.T, r=w.r, budget=w.budget_video,
                        k_ref=g.get("k_ref"), v_ref=g.get("v_ref"),
                        budget_ref=w.budget_ref if "k_ref" in g else 0,
                        k_dense=g.get("k_dense"), v_dense=g.get("v_dense"),
                        flags=(veda.binding.VEDA_FLAG_SIMT_ATTENTION if simt else 0) | flags)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} needs one process per GPU: launch with "
                         f"torch.distributed.run --nproc-per-node {args.gpus} (WORLD_SIZE is {world})")
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        # the CPU oracle: rank 0 alone runs and prints; other ranks do no work
        if rank == 0:
            w = workloads.get(args.workload)
            if args.budget:
                w = w.with_budget(args.budget)
            dev = torch.device("cuda", local) if torch.cuda.is_available() else torch.device("cpu")
            run_reference(args, w, dev, world)
        return
    dist = None
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    w = workloads.get(args.workload)
    if args.budget:
        w = w.with_budget(args.budget)
    if args.heads:
        w = workloads.small(w.name, H=args.heads, budget_video=w.budget_video)
    n = world

    import learned_block_sparse_pool_b200 as veda
    g = workloads.make_inputs(w, device=dev)
    sel_flags = (veda.binding.VEDA_FLAG_UNFUSED_SELECTION if args.unfused_selection else 0) | \
        (veda.binding.VEDA_FLAG_ONCHIP_SELECTION if args.onchip_selection else 0)
    # calls: every rank runs the whole call (n calls per step); heads: every
    # rank runs its head range of the same call (one call per step)
    split = args.split == "heads" and n > 1
    calls_per_step = 1 if split else n
    w_run = w
    if split:
        h0, h1 = head_range(w.H, n, rank)
        g = head_slice(g, h0, h1)
        w_run = dataclasses.replace(w, H=h1 - h0)
    p = make_problem(veda, w_run, g, args.simt, sel_flags)
    ws = veda.workspace(p)
    if args.dense_queries:
        if split:
            raise SystemExit("--dense-queries runs whole calls (--split calls)")
        dense_query_run(args, veda, w, g, p, ws, dev, local, rank, n, dist)
        return
    iv, ir = veda.alloc_indices(p)
    out, _ = veda.alloc_output(p)
    stream = torch.cuda.current_stream(dev)

    # the stages of one call, each bracketed by CUDA events on the launching stream
    if args.unfused_selection:
        stages = [("pool_project", lambda: veda.pool_project(p, g["w_q"], g["w_k"], ws, stream)),
                  ("score", lambda: veda.score_tiles(p, ws, stream)),
                  ("topk", lambda: veda.topk_tiles(p, iv, ir, ws, stream))]
    else:
        stages = [("pool_project", lambda: veda.pool_project(p, g["w_q"], g["w_k"], ws, stream)),
                  ("select", lambda: veda.score_topk_tiles(p, iv, ir, ws, stream))]
    stages.append(("attention", lambda: veda.block_sparse_attn(p, iv, ir, out, None, ws, stream)))
    n_st = len(stages)

    def step(ev):
        for s_i, (_, fn) in enumerate(stages):
            fn()
            ev[s_i + 1].record(stream)

    def events():
        return [torch.cuda.Event(enable_timing=True) for _ in range(n_st + 1)]

    clocks = ClockSampler(local)
    clocks.start()
    for _ in range(args.warmup):
        ev = events()
        ev[0].record(stream)
        step(ev)
    st = veda.check_status(ws, stream)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {veda.status_string(st)}")

    evs = [events() for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    wall0 = time.time()
    t_start.record(stream)
    for k in range(args.steps):
        evs[k][0].record(stream)
        step(evs[k])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    wall1 = time.time()
    clk = clocks.stop(wall0, wall1)
    st = veda.check_status(ws, stream)
    if st != 0:
        raise RuntimeError(f"device status after timing: {veda.status_string(st)}")

    total_ms = t_start.elapsed_time(t_end)
    stage = [[evs[k][s].elapsed_time(evs[k][s + 1]) for k in range(args.steps)] for s in range(n_st)]
    stage_avg = [sum(x) / len(x) for x in stage]
    total_ms, *stage_avg = max_over_ranks(dist, [total_ms] + stage_avg, dev)
    st_ms = {name: stage_avg[i] for i, (name, _) in enumerate(stages)}

    pk, pk_src = peaks()
    # per-GPU work: the whole call, or (heads split) the largest rank's share
    wm = dataclasses.replace(w, H=-(-w.H // n)) if split else w
    attn_s = st_ms["attention"] / 1e3
    flops = wm.kept_flops()
    achieved_tf = flops / attn_s / 1e12
    sustained_tf = pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    burst_tf = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    # the burst figure applies to a timed region of under a few seconds (the
    # clocks stay near their maximum), the sustained one to a longer loop
    long_region = total_ms > 5000.0
    peak_tf = sustained_tf if long_region else burst_tf
    hbm = pk.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    esz = 2 if wm.dtype == "bf16" else 4
    pool_bytes = (2 * wm.n_video + wm.n_ref) * wm.B * wm.H * wm.d * esz
    rows = wm.B * wm.H * wm.n_q_tiles
    selector = {
        "pool_project_gbs": round(pool_bytes / (st_ms["pool_project"] / 1e3) / 1e9, 1),
        "pool_project_frac": round(pool_bytes / (st_ms["pool_project"] / 1e3) / 1e9 / hbm, 4),
        "peak_gbs": hbm, "peak_kind": f"HBM copy ({pk_src})",
    }
    segs = [(wm.n_q_tiles, wm.budget_video)] + ([(wm.n_ref_tiles, wm.budget_ref)] if wm.ref_frames else [])
    score_flop = sum(2.0 * wm.r * rows * nk for nk, _ in segs)
    if args.unfused_selection:
        # a row's scores are read unless every tile is kept; the kept indices are written
        topk_bytes = sum(rows * ((nk * 4 if k < nk else 0) + k * 4) for nk, k in segs)
        selector.update({
            "topk_gbs": round(topk_bytes / (st_ms["topk"] / 1e3) / 1e9, 1),
            "topk_frac": round(topk_bytes / (st_ms["topk"] / 1e3) / 1e9 / hbm, 4),
            "score_kernel": "SIMT fp32 contraction (alu-bound)",
            "score_gflops": round(score_flop / (st_ms["score"] / 1e3) / 1e9, 1),
        })
        launches_per_step = 2 + 2 * len(segs)
    elif args.onchip_selection:
        # one kernel: tensor-core scores recomputed per pass, top-k on chip;
        # reads the bf16 projection planes (k-hat from L2) and writes the kept indices
        sel_bytes = sum(rows * k * 4 for _, k in segs) + 6 * 64 * rows * (1 + len(segs))
        selector.update({
            "select_kernel": "tensor-core scores + on-chip top-k (no score matrix in HBM)",
            "select_ms": round(st_ms["select"], 4),
            "select_algorithmic_bytes": sel_bytes,
            "select_score_gflops": round(score_flop / (st_ms["select"] / 1e3) / 1e9, 1),
        })
        launches_per_step = 3 + sum(1 for nk, k in segs if k < nk)   # + the top-k of rows left over
    else:
        # tensor-core scores written once (exact), then the warp-per-row top-k
        # reads them: planes in, scores out and back in, indices out
        sel_bytes = sum(rows * (2 * nk * 4 + k * 4) for nk, k in segs) + 6 * 64 * rows * (1 + len(segs))
        selector.update({
            "select_kernels": "tensor-core scores to HBM + warp-per-row top-k",
            "select_ms": round(st_ms["select"], 4),
            "select_algorithmic_bytes": sel_bytes,
            "select_gbs": round(sel_bytes / (st_ms["select"] / 1e3) / 1e9, 1),
            "select_frac": round(sel_bytes / (st_ms["select"] / 1e3) / 1e9 / hbm, 4),
            "select_score_gflops": round(score_flop / (st_ms["select"] / 1e3) / 1e9, 1),
        })
        launches_per_step = 3 + len(segs)

    res = {
        "metric": METRIC,
        "value": round(total_ms / args.steps / calls_per_step, 4),
        "unit": "ms",
        "n_gpus": n,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": False,
        "scaling": "strong" if split else "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded; N(0,1) + smooth sinusoid component, shapes of the 1344x768 24 fps clips)",
        "config": bench_config(w, n, args.simt, args.split),
        "kernels_ms": {name: round(v, 4) for name, v in st_ms.items()},
        "roofline": {
            "kernel": "block-sparse attention",
            "bound": "tensor", "achieved": round(achieved_tf, 2), "peak": peak_tf, "unit": "TFLOP/s",
            "frac": round(achieved_tf / peak_tf, 4),
            "traffic": (None if (w.name, w.H, w.budget_video) not in ATTN_TRAFFIC else
                        ATTN_TRAFFIC[(w.name, w.H, w.budget_video)] * wm.H / w.H),
            "peak_kind": (f"bf16 dense, {'sustained' if long_region else 'burst'} ({pk_src}; timed region "
                          f"{total_ms / 1e3:.2f} s)"),
            "frac_of_burst_peak": round(achieved_tf / burst_tf, 4),
            "frac_of_sustained_peak": round(achieved_tf / sustained_tf, 4),
            "algorithmic": f"{flops:.4g} FLOP per launch = 4*T*T*d x kept (b,h,q-tile,k-tile) pairs",
        },
        "selector_hbm": selector,
        "clocks": clk,
        "gpu_launches": launches_per_step * args.steps,
    }

    if not args.ncu and not args.no_e2e:
        res["e2e"] = e2e_run(veda, w_run, g, p, dev, stream, args.steps, calls_per_step, dist, args.simt)
    if not args.ncu and not args.no_cpu_baseline and n == 1 and rank == 0:
        ms, cores, sample = oracle_sample(w, host_copy(g), oracle_units(w))
        res["cpu_baseline"] = {"value": round(ms, 1), "unit": "ms", "cores": cores, "kind": "oracle",
                               "sample": sample}
    if rank == 0:
        print(json.dumps(res), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def dense_query_run(args, veda, w, g, p, ws, dev, local, rank, n, dist):
    """Dense-query rows (text / VLM / audio / reference tokens as queries over
    every key of the problem): one veda_dense_query_attn per step."""
    rows = args.dense_queries
    gen = torch.Generator(device=dev).manual_seed(1000 + w.seed)
    q_rows = torch.randn((w.B, rows, w.H, w.d), generator=gen, device=dev, dtype=torch.float32).to(w.torch_dtype)
    out = torch.empty_like(q_rows)
    stream = torch.cuda.current_stream(dev)
    clocks = ClockSampler(local)
    clocks.start()
    for _ in range(args.warmup):
        veda.dense_query_attn(p, q_rows, out, None, ws, stream)
    st = veda.check_status(ws, stream)
    if st != 0:
        raise RuntimeError(f"device status after warm-up: {veda.status_string(st)}")
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    wall0 = time.time()
    t0.record(stream)
    for _ in range(args.steps):
        veda.dense_query_attn(p, q_rows, out, None, ws, stream)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    clk = clocks.stop(wall0, time.time())
    st = veda.check_status(ws, stream)
    if st != 0:
        raise RuntimeError(f"device status after timing: {veda.status_string(st)}")
    ms, = max_over_ranks(dist, [t0.elapsed_time(t1) / args.steps], dev)
    tiles = w.n_q_tiles + (w.n_ref_tiles if w.n_ref else 0) + w.n_dense_tiles
    flops = 4.0 * w.T * w.T * w.d * w.B * w.H * (-(-rows // w.T)) * tiles
    pk, pk_src = peaks()
    sustained_tf = pk.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    burst_tf = pk.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    long_region = ms * args.steps > 5000.0
    peak_tf = sustained_tf if long_region else burst_tf
    achieved = flops / (ms / 1e3) / 1e12
    res = {
        "metric": "ms per dense-query attention call (non-video query rows over every key)",
        "value": round(ms / n, 4), "unit": "ms", "n_gpus": n, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms, 4), "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic (seeded N(0,1) query rows; the workload's keys)",
        "config": dict(w.describe(), **{"dense_query_rows": rows, "key_tiles_per_query_tile": tiles,
                                        "tflop_per_call": round(flops / 1e12, 4),
                                        "l2": "keys larger than L2 (K, V of one call exceed 126 MB each)"}),
        "roofline": {"kernel": "attention, every key tile", "bound": "tensor", "achieved": round(achieved, 2),
                     "peak": peak_tf, "unit": "TFLOP/s", "frac": round(achieved / peak_tf, 4), "traffic": None,
                     "peak_kind": f"bf16 dense, {'sustained' if long_region else 'burst'} ({pk_src})",
                     "frac_of_burst_peak": round(achieved / burst_tf, 4),
                     "frac_of_sustained_peak": round(achieved / sustained_tf, 4)},
        "clocks": clk,
        "gpu_launches": args.steps,
    }
    if rank == 0:
        print(json.dumps(res), flush=True)
    if dist is not None:
        dist.destroy_process_group()


def e2e_run(veda, w, g, p, dev, stream, steps, calls_per_step, dist, simt, heads_per_group=2):
    """Same metric through the public host-buffer call (veda_attn_host): every
    step takes Q, K, V, the dense and reference keys and the selector weights
    from pinned host memory and returns the attention output to pinned host
    memory; the library pipelines the copies with the compute over groups of
    heads."""
    host = {k: v.cpu().contiguous().pin_memory() for k, v in g.items()}
    ph = make_problem(veda, w, host, simt)
    buf = veda.attn_host_buffer(ph, heads_per_group, dev)
    out_host = torch.empty((w.B, w.n_video, w.H, w.d), dtype=w.torch_dtype, pin_memory=True)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_host.numel() * out_host.element_size()

    def one():
        veda.attn_host(ph, host["w_q"], host["w_k"], None, None, out_host, None, heads_per_group, buf, stream)

    one()
    torch.cuda.synchronize(dev)
    k2 = max(2, min(steps, 5))
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t0.record(stream)
    for _ in range(k2):
        one()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(dist, [t0.elapsed_time(t1)], dev)[0]
    st = veda.check_status(buf, stream)
    if st != 0:
        raise RuntimeError(f"device status after e2e: {veda.status_string(st)}")
    return {"value": round(ms / k2 / calls_per_step, 4), "unit": "ms", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h,
            "steps": k2, "call": f"veda_attn_host (pinned host buffers, {heads_per_group} heads per group)"}


def run_reference(args, w, dev, n):
    """--impl reference: the CPU oracle on the host cores, each step one
    bounded sample of the same workload (the sample and extrapolation of the
    main arm's cpu_baseline), reported as ms per call."""
    g = workloads.make_inputs(w, device=dev)
    host = host_copy(g)
    del g
    units = oracle_units(w)
    for _ in range(args.warmup):
        oracle_sample(w, host, units)
    vals = []
    t_all = time.perf_counter()
    for _ in range(args.steps):
        ms, cores, sample = oracle_sample(w, host, units)
        vals.append(ms)
    wall = time.perf_counter() - t_all
    v = statistics.mean(vals)
    res = {
        "impl": "reference",
        "metric": METRIC, "value": round(v, 1), "unit": "ms", "n_gpus": n, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(wall / args.steps * 1e3, 1), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(w, n, args.simt, args.split),
        "cpu_baseline": {"value": round(v, 1), "unit": "ms", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(v, 1), "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(res), flush=True)


if __name__ == "__main__":
    main()
