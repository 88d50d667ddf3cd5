#!/usr/bin/env python
"""Benchmark of the block-sparse bidirectional attention hot path on B200.

One bench step = one complete denoising run of one attention layer through
the library's step driver (sparsed_run_steps): dense attention for the warm-up
steps, pattern selection (dense pass + block mass + top-k) at the switch and at
anchors, block-sparse attention afterwards. Default workload: c4_64k
(H=32, L=65536, d=128, bq=bk=128, keep 0.10, T=1024, first 20% dense).

Metric: effective TFLOP/s = attention flops of the run / device time, counting
4*L*L*d per head for a dense or selecting step and 4*bq*bk*d per kept block for
a sparse step (the block-mass pass of a selecting step is overhead, not counted).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (launched by torchrun) the layer's heads are split evenly over the
ranks (strong scaling): a uniform budget needs no exchange, an entropy budget
all-gathers the H per-head entropies at each selecting step (NCCL). The time
is the max over ranks and the value the whole layer's flops over that time.
(--path losa runs an independent block per rank.)
--impl reference times the fp64 CPU oracle on this host's cores on a bounded
sample of the same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_bidirectional_select_b200.inputs import (BLOCK_WORKLOADS, WORKLOADS, make_block_inputs,  # noqa: E402
                                                           make_inputs, to_f64)

METRIC = "block-sparse attn effective TFLOP/s & ms/step at 64k, % of B200 bf16 peak"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# NVIDIA's dense bf16 tensor figure for one B200 (the 4.5 PFLOP/s of the spec
# sheet is with 2:4 sparsity); context beside the measured peaks
DATASHEET_BF16_TFLOPS = 2250.0


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------- accounting

def run_accounting(wl, kinds, kv_count_sum):
    """Effective flops of one run and the kernel launches it makes."""
    dense = 4.0 * wl.H * float(wl.L) * float(wl.L) * wl.d
    sparse = 4.0 * wl.bq * wl.bk * wl.d * float(kv_count_sum)
    n_dense = kinds.count(0)
    n_select = kinds.count(1)
    n_sparse = kinds.count(2)
    per_select = 3 + (2 if wl.budget == "entropy" else 0)  # dense, mass, [entropy, budget], top-k
    return dict(flops=(n_dense + n_select) * dense + n_sparse * sparse, dense_flops=dense,
                sparse_flops=sparse, n_dense=n_dense, n_select=n_select, n_sparse=n_sparse,
                launches=n_dense + n_select * per_select + n_sparse)


# ----------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def _gpu_id(self):
        try:
            uuid = torch.cuda.get_device_properties(self.dev).uuid
            s = str(uuid)
            return s if s.startswith("GPU-") else "GPU-" + s
        except Exception:
            return str(self.dev)

    def start(self):
        cmd = ["nvidia-smi", f"--id={self._gpu_id()}", "--query-gpu=" + ",".join(self.FIELDS),
               "--format=csv,noheader,nounits", "-lms", "200"]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        sm, smax, reasons = [], [], set()
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(self.REASONS, parts[3:]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- CPU oracle

def cpu_oracle_sample(wl, q, k, v, budget_s, rng_seed=0):
    """Time the fp64 oracle on sampled (head, query block) tiles of this
    workload: the dense rows of the tile, its block-mass row, its top-k and its
    block-masked rows; extrapolate to the effective TFLOP/s of a full run."""
    import oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    nqb, nkb = -(-wl.L // wl.bq), -(-wl.L // wl.bk)
    kk = O.uniform_keep(nkb, wl.keep)
    rng = np.random.default_rng(rng_seed)
    t_dense = t_mass = t_sparse = 0.0
    n = 0
    heads = {}
    t_start = time.perf_counter()
    while time.perf_counter() - t_start < budget_s and n < 64:
        h = int(rng.integers(wl.H))
        i = int(rng.integers(nqb))
        if h not in heads:
            heads.clear()
            heads[h] = (to_f64(q[h]), to_f64(k[h]), to_f64(v[h]))
        qh, kh, vh = heads[h]
        r0, r1 = i * wl.bq, min((i + 1) * wl.bq, wl.L)
        t0 = time.perf_counter()
        _, lse = O.dense_attention(qh[r0:r1], kh, vh, wl.scale)
        t1 = time.perf_counter()
        lse_full = np.zeros(wl.L)
        lse_full[r0:r1] = lse
        mrow = O.block_mass(qh, kh, wl.scale, lse_full, wl.bq, wl.bk, qblocks=[i])[0]
        sel = O.topk_blocks(mrow, kk)
        t2 = time.perf_counter()
        keys = O.kept_keys(sel, wl.bk, wl.L)
        O.softmax_attention(qh[r0:r1], kh[keys], vh[keys], wl.scale)
        t3 = time.perf_counter()
        t_dense += t1 - t0
        t_mass += t2 - t1
        t_sparse += t3 - t2
        n += 1
    tiles = wl.H * nqb
    kinds = O.schedule(wl.T, wl.warmup_frac, wl.refresh_every)
    acc = run_accounting(wl, kinds, wl.H * nqb * kk)
    step_dense = tiles * t_dense / n
    step_select = tiles * (t_dense + t_mass) / n
    step_sparse = tiles * t_sparse / n
    run_s = acc["n_dense"] * step_dense + acc["n_select"] * step_select + acc["n_sparse"] * step_sparse
    value = acc["flops"] / run_s / 1e12
    sample = (f"{n} (head, query-block) tiles of {wl.name}: fp64 dense rows + block-mass row + top-k + "
              f"masked rows per tile, {t_dense + t_mass + t_sparse:.1f} s of oracle time, "
              f"extrapolated to a full {wl.T}-step run ({tiles} tiles per step)")
    return {"value": value, "unit": UNIT, "cores": int(cores), "kind": "oracle", "sample": sample,
            "ms_per_step_extrapolated": run_s * 1e3}


# ----------------------------------------------------------------- ranks

def head_range(H, world, rank):
    """The heads [h0, h1) of the layer this rank holds: the layer's heads split
    evenly over the ranks in rank order (every head's work is independent; an
    entropy budget only exchanges the per-head entropies)."""
    if H % world:
        raise SystemExit(f"--gpus {world} must divide the {H} heads of the layer")
    n = H // world
    return rank * n, (rank + 1) * n


def reduce_max(x, world, device):
    """Max of a host float over all ranks (identity for one rank)."""
    if world == 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(x, world, device):
    """Sum of a host float over all ranks (identity for one rank)."""
    if world == 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def job_value(layer_flops_per_step, steps, total_ms):
    """Whole-job throughput in TFLOP/s: the layer's flops (all ranks' heads
    together) over the slowest rank's time (strong scaling: the layer is
    fixed, its heads split over the ranks)."""
    return layer_flops_per_step * steps / (total_ms * 1e-3) / 1e12


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    wl = WORKLOADS[args.workload]
    log(f"[reference] generating inputs for {wl.name}")
    q, k, v = make_inputs(wl)
    budget = args.cpu_seconds
    for _ in range(args.warmup):
        cpu_oracle_sample(wl, q, k, v, min(budget, 5.0), rng_seed=99)
    vals, base = [], None
    t0 = time.perf_counter()
    for s in range(args.steps):
        base = cpu_oracle_sample(wl, q, k, v, budget, rng_seed=s)
        vals.append(base["value"])
    wall = time.perf_counter() - t0
    value = statistics.median(vals)
    base = dict(base, value=value)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": base["ms_per_step_extrapolated"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl),
            "cpu_baseline": base,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s_sampling": wall}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------- GPU arm

def workload_config(wl):
    return {"workload": wl.name, "H": wl.H, "L": wl.L, "d": wl.d, "bq": wl.bq, "bk": wl.bk,
            "keep": wl.keep, "budget": wl.budget, "T": wl.T, "warmup_frac": wl.warmup_frac,
            "refresh_every": wl.refresh_every, "inputs": wl.structure,
            "l2": "inputs larger than L2 (Q,K,V %.2f GiB vs 126 MB)" % (3 * wl.H * wl.L * wl.d * 2 / 2**30)}


def event_time(fn, stream, n):
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(n):
        fn()
    e.record(stream)
    e.synchronize()
    return s.elapsed_time(e)


def median_time(fn, stream, reps):
    out = []
    for _ in range(reps):
        out.append(event_time(fn, stream, 1))
    return statistics.median(out)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="c4_64k", choices=sorted(WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--op", choices=["run", "dense", "sparse", "select", "col_sparse", "col_select"],
                    default="run",
                    help="run: the full denoising run (the benchmark); dense/sparse/select and the column "
                         "path's col_sparse/col_select: time one library call alone, K launches after W "
                         "warm-up launches (for profiling)")
    ap.add_argument("--path", choices=["blocks", "columns", "losa"], default="blocks",
                    help="blocks: the block-sparse path (the benchmark); columns: the same denoising run "
                         "with the column-sparse pattern; losa: block-wise generation over a prefix cache "
                         "with active-token reuse (--block-workload)")
    ap.add_argument("--block-workload", default="losa_32k", choices=sorted(BLOCK_WORKLOADS))
    ap.add_argument("--warmup-frac", type=float, default=None,
                    help="override the workload's dense warm-up fraction w (e.g. 0.05: the column or block "
                         "pattern applied from earlier denoising steps)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import block_sparse_bidirectional_select_b200 as sp
    import torch.distributed as dist

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=300))

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x):
        return reduce_max(x, world, dev)

    wl = WORKLOADS[args.workload]
    if args.warmup_frac is not None:
        wl = wl.scaled(warmup_frac=args.warmup_frac)
    if args.op != "run":
        return time_one_op(args, wl, dev, rank)
    if args.path == "columns":
        return run_columns(args, wl, dev, rank, world, barrier, max_over_ranks)
    if args.path == "losa":
        return run_losa(args, dev, rank, world, barrier, max_over_ranks)
    h0, h1 = head_range(wl.H, world, rank)
    log(f"[rank {rank}] inputs for {wl.name}, heads {h0}..{h1 - 1}")
    q_cpu, k_cpu, v_cpu = (t[h0:h1].contiguous() for t in make_inputs(wl))
    q, k, v = (t.to(dev) for t in (q_cpu, k_cpu, v_cpu))
    stream = torch.cuda.current_stream()
    peaks, peak_src = load_peaks()

    H, L, d = h1 - h0, wl.L, wl.d
    wl_local = wl.scaled(H=H)
    ws = torch.empty(sp.run_steps_workspace_bytes(H, L, wl.bq, wl.bk), dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((H, L), dtype=torch.float32, device=dev)
    group = dist.group.WORLD if world > 1 else None

    def one_run(time_steps=False):
        if world > 1:
            # this rank's heads; an entropy budget all-gathers the per-head
            # entropies at every selecting step (the loop's only exchange)
            return sp.run_steps_sharded(q, k, v, wl.T, wl.warmup_frac, keep=wl.keep, budget=wl.budget,
                                        refresh_every=wl.refresh_every, group=group, bq=wl.bq, bk=wl.bk,
                                        out=o, lse=lse, workspace=ws)
        return sp.run_steps(q, k, v, wl.T, wl.warmup_frac, keep=wl.keep, budget=wl.budget,
                            refresh_every=wl.refresh_every, bq=wl.bq, bk=wl.bk, out=o, lse=lse,
                            workspace=ws, time_steps=time_steps)

    log(f"[rank {rank}] warm-up x{args.warmup}")
    for _ in range(args.warmup):
        res = one_run()
    sp.device_check()
    kinds = res.kinds
    kv_sum = int(res.kv_count.sum().item())
    acc = run_accounting(wl_local, kinds, kv_sum)
    layer_flops = reduce_sum(acc["flops"], world, dev)

    # ---------------- timed region: K full runs
    torch.cuda.synchronize()
    barrier()
    clocks = ClockSampler(local)
    clocks.start()
    step_ms = []
    s_ev = torch.cuda.Event(enable_timing=True)
    e_ev = torch.cuda.Event(enable_timing=True)
    s_ev.record(stream)
    for _ in range(args.steps):
        r = one_run(time_steps=world == 1)
        if r.step_ms is not None:
            step_ms.append(r.step_ms)
    e_ev.record(stream)
    e_ev.synchronize()
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    total_ms = max_over_ranks(s_ev.elapsed_time(e_ev))
    sp.device_check()
    ms_per_step = total_ms / args.steps
    value = job_value(layer_flops, args.steps, total_ms)

    per_kind = {0: [], 1: [], 2: []}
    for run in step_ms:
        for kind, ms in zip(kinds, run):
            per_kind[kind].append(ms)
    dense_ms = statistics.mean(per_kind[0]) if per_kind[0] else None
    select_ms = statistics.mean(per_kind[1]) if per_kind[1] else None
    sparse_ms = statistics.mean(per_kind[2]) if per_kind[2] else None

    peak_tc = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    peak_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    time_dense = (acc["n_dense"] * (dense_ms or 0.0))
    time_sparse = (acc["n_sparse"] * (sparse_ms or 0.0))
    dominant = "dense" if time_dense >= time_sparse else "sparse"
    d_ach = acc["dense_flops"] / (dense_ms * 1e-3) / 1e12 if dense_ms else None
    s_ach = acc["sparse_flops"] / (sparse_ms * 1e-3) / 1e12 if sparse_ms else None
    traffic = load_traffic(wl.name)

    def roof(kernel, ach, units):
        return {"kernel": kernel, "bound": "tensor", "achieved": ach, "peak": peak_tc, "unit": "TFLOP/s",
                "frac": (ach / peak_tc) if ach else None,
                "peak_source": f"{peak_src} bf16_tflops_sustained (kernel timed inside the long run)",
                "units_per_launch": units, "traffic": traffic.get(kernel)}

    dense_name = f"attn_fwd_kernel<{d},{wl.bk},dense>"
    sparse_name = f"attn_list_kernel<{d},{wl.bk}>"
    roof_dense = roof(dense_name, d_ach, f"{H}x{L}x{L} score tiles, 4*H*L^2*d flops")
    roof_sparse = roof(sparse_name, s_ach, f"{kv_sum} kept blocks, 4*bq*bk*d flops each")
    roofline = roof_dense if dominant == "dense" else roof_sparse

    # ---------------- single-kernel timings (context)
    extra = {}
    if res.kv_idx is not None and acc["n_sparse"] > 0:
        fn = lambda: sp.block_sparse_attn(q, k, v, res.kv_idx, res.kv_count, bq=wl.bq, bk=wl.bk, out=o, lse=lse)
        fn()
        ms = median_time(fn, stream, 20)
        tf = acc["sparse_flops"] / (ms * 1e-3) / 1e12
        extra["block_sparse_attn"] = {"ms": ms, "tflops": tf, "frac_of_peak_burst": tf / peak_burst,
                                      "peak_burst": peak_burst, "kept_blocks": kv_sum,
                                      "frac_of_datasheet_dense_bf16": tf / DATASHEET_BF16_TFLOPS}
    fn = lambda: sp.dense_attn(q, k, v, bq=wl.bq, bk=wl.bk, out=o, lse=lse)
    fn()
    ms = median_time(fn, stream, 3)
    extra["dense_attn"] = {"ms": ms, "tflops": acc["dense_flops"] / (ms * 1e-3) / 1e12}
    try:
        import torch.nn.functional as F
        q4, k4, v4 = (t.unsqueeze(0) for t in (q, k, v))
        fn = lambda: F.scaled_dot_product_attention(q4, k4, v4)
        fn()
        ms = median_time(fn, stream, 3)
        extra["torch_sdpa_dense"] = {"ms": ms, "tflops": acc["dense_flops"] / (ms * 1e-3) / 1e12}
    except Exception as ex:  # context only
        extra["torch_sdpa_dense"] = {"error": str(ex)[:200]}
    sp.device_check()

    # ---------------- end to end through the public API with host buffers
    e2e = None
    if not args.skip_e2e:
        qh, kh, vh = (t.pin_memory() for t in (q_cpu, k_cpu, v_cpu))
        oh = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        lh = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
        qd, kd, vd = (torch.empty_like(t) for t in (q, k, v))

        def e2e_run():
            qd.copy_(qh, non_blocking=True)
            kd.copy_(kh, non_blocking=True)
            vd.copy_(vh, non_blocking=True)
            if world > 1:
                sp.run_steps_sharded(qd, kd, vd, wl.T, wl.warmup_frac, keep=wl.keep, budget=wl.budget,
                                     refresh_every=wl.refresh_every, group=group, bq=wl.bq, bk=wl.bk, out=o,
                                     lse=lse, workspace=ws)
            else:
                sp.run_steps(qd, kd, vd, wl.T, wl.warmup_frac, keep=wl.keep, budget=wl.budget,
                             refresh_every=wl.refresh_every, bq=wl.bq, bk=wl.bk, out=o, lse=lse, workspace=ws)
            oh.copy_(o, non_blocking=True)
            lh.copy_(lse, non_blocking=True)

        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(event_time(e2e_run, stream, args.steps))
        torch.cuda.synchronize()
        bi = 3 * q.numel() * q.element_size()
        bo = o.numel() * o.element_size() + lse.numel() * lse.element_size()
        e2e = {"value": job_value(layer_flops, args.steps, e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo, "ms_per_step": e2e_ms / args.steps}

    cpu = None
    if rank == 0 and world == 1 and not args.skip_cpu:
        log("[rank 0] timing the CPU oracle on a bounded sample")
        cpu = cpu_oracle_sample(wl, q_cpu, k_cpu, v_cpu, args.cpu_seconds)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(workload_config(wl), parallelism=f"heads x{world}" if world > 1 else "single",
                       step="one complete T-step denoising run of the layer"),
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": acc["launches"] * args.steps,
        "clocks": clk,
        "pct_of_peak": {"value_vs_burst": value / world / peak_burst, "value_vs_sustained": value / world / peak_tc,
                        "value_vs_datasheet_dense_bf16": value / world / DATASHEET_BF16_TFLOPS,
                        "peak_source": peak_src},
        # per GPU and per GHz of the median SM clock sampled in the timed
        # region: the run's throughput with the power-capped clock divided out
        "tflops_per_gpu_per_ghz": (value / world / (clk["sm_mhz"] / 1000.0)) if clk.get("sm_mhz") else None,
        "ms_per_denoise_step": ms_per_step / wl.T,
        "steps_breakdown": {"dense_ms": dense_ms, "select_ms": select_ms, "sparse_ms": sparse_ms,
                            "n_dense": acc["n_dense"], "n_select": acc["n_select"], "n_sparse": acc["n_sparse"]},
        "roofline_sparse": roof_sparse, "roofline_dense": roof_dense,
        **extra,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def time_one_op(args, wl, dev, rank):
    """Time one library call alone (dense_attn, block_sparse_attn with the
    pattern select_pattern picks, or select_pattern) on one GPU."""
    import block_sparse_bidirectional_select_b200 as sp
    q, k, v = (t.to(dev) for t in make_inputs(wl))
    stream = torch.cuda.current_stream()
    o = torch.empty_like(q)
    lse = torch.empty((wl.H, wl.L), dtype=torch.float32, device=dev)
    dense_flops = 4.0 * wl.H * float(wl.L) * float(wl.L) * wl.d
    if args.op == "dense":
        fn = lambda: sp.dense_attn(q, k, v, bq=wl.bq, bk=wl.bk, out=o, lse=lse)
        flops = dense_flops
    elif args.op == "select":
        ws = torch.empty(sp.workspace_bytes(wl.H, wl.L, wl.bq, wl.bk), dtype=torch.uint8, device=dev)
        fn = lambda: sp.select_pattern(q, k, v, keep=wl.keep, budget=wl.budget, bq=wl.bq, bk=wl.bk,
                                       workspace=ws)
        flops = dense_flops
    elif args.op == "col_select":
        kc = sp.column_keep(wl.L, wl.keep)
        ws = torch.empty(sp.column_workspace_bytes(wl.H, wl.L, wl.d, kc), dtype=torch.uint8, device=dev)
        fn = lambda: sp.select_columns(q, k, v, keep=wl.keep, bq=wl.bq, bk=wl.bk, workspace=ws)
        flops = dense_flops
    elif args.op == "col_sparse":
        pat = sp.select_columns(q, k, v, keep=wl.keep, bq=wl.bq, bk=wl.bk)
        kc = pat.cols.shape[1]
        ws = torch.empty(sp.column_workspace_bytes(wl.H, wl.L, wl.d, kc), dtype=torch.uint8, device=dev)
        fn = lambda: sp.column_sparse_attn(q, k, v, pat.cols, bq=wl.bq, bk=wl.bk, out=o, lse=lse, workspace=ws)
        flops = 4.0 * wl.H * float(wl.L) * kc * wl.d
    else:
        pat = sp.select_pattern(q, k, v, keep=wl.keep, budget=wl.budget, bq=wl.bq, bk=wl.bk)
        fn = lambda: sp.block_sparse_attn(q, k, v, pat.kv_idx, pat.kv_count, bq=wl.bq, bk=wl.bk, out=o, lse=lse)
        flops = 4.0 * wl.bq * wl.bk * wl.d * float(pat.kv_count.sum().item())
    for _ in range(args.warmup):
        fn()
    sp.device_check()
    torch.cuda.synchronize()
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    times = [event_time(fn, stream, 1) for _ in range(args.steps)]
    clk = clocks.stop()
    sp.device_check()
    ms = statistics.median(times)
    if rank == 0:
        print(json.dumps({"op": args.op, "workload": wl.name, "launches": args.steps, "ms_median": ms,
                          "ms_all": times, "tflops": flops / (ms * 1e-3) / 1e12, "clocks": clk}), flush=True)
    return 0


def run_columns(args, wl, dev, rank, world, barrier, max_over_ranks):
    """The same denoising run with the column-sparse pattern (PulseCol): dense
    warm-up, column selection at the switch, attention over the kept columns.
    Effective flops count 4*L*kc*d per head for a sparse step."""
    import block_sparse_bidirectional_select_b200 as sp
    h0, h1 = head_range(wl.H, world, rank)  # this rank's heads of the layer (no exchange: columns are per head)
    q, k, v = (t[h0:h1].contiguous().to(dev) for t in make_inputs(wl))
    stream = torch.cuda.current_stream()
    H, L, d = h1 - h0, wl.L, wl.d
    kc = sp.column_keep(L, wl.keep)
    ws = torch.empty(sp.column_workspace_bytes(H, L, d, kc), dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((H, L), dtype=torch.float32, device=dev)

    def one_run(time_steps=False):
        return sp.run_steps_columns(q, k, v, wl.T, wl.warmup_frac, keep=wl.keep,
                                    refresh_every=wl.refresh_every, bq=wl.bq, bk=wl.bk, out=o, lse=lse,
                                    workspace=ws, time_steps=time_steps)

    for _ in range(args.warmup):
        res = one_run()
    sp.device_check()
    kinds = res.kinds
    n_dense, n_select, n_sparse = kinds.count(0), kinds.count(1), kinds.count(2)
    dense = 4.0 * H * float(L) * float(L) * d
    sparse = 4.0 * H * float(L) * kc * d
    flops = (n_dense + n_select) * dense + n_sparse * sparse
    torch.cuda.synchronize()
    barrier()
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    s_ev = torch.cuda.Event(enable_timing=True)
    e_ev = torch.cuda.Event(enable_timing=True)
    step_ms = []
    s_ev.record(stream)
    for _ in range(args.steps):
        step_ms.append(one_run(time_steps=True).step_ms)
    e_ev.record(stream)
    e_ev.synchronize()
    barrier()
    clk = clocks.stop()
    total_ms = max_over_ranks(s_ev.elapsed_time(e_ev))
    sp.device_check()
    per_kind = {0: [], 1: [], 2: []}
    for run in step_ms:
        for kind, ms in zip(kinds, run):
            per_kind[kind].append(ms)
    mean = lambda x: statistics.mean(x) if x else None
    fn = lambda: sp.column_sparse_attn(q, k, v, res.kv_idx, bq=wl.bq, bk=wl.bk, out=o, lse=lse, workspace=ws)
    fn()
    ms_alone = median_time(fn, stream, 20)
    peaks, peak_src = load_peaks()
    peak_burst = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    layer_flops = reduce_sum(flops, world, dev)
    line = {"metric": "column-sparse attn effective TFLOP/s & ms/step at 64k", "value":
            job_value(layer_flops, args.steps, total_ms), "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": total_ms / args.steps, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(workload_config(wl), path="columns", kept_columns_per_head=kc,
                           parallelism=f"heads x{world}" if world > 1 else "single",
                           step="one complete T-step denoising run of the layer"),
            "ms_per_denoise_step": total_ms / args.steps / wl.T,
            "steps_breakdown": {"dense_ms": mean(per_kind[0]), "select_ms": mean(per_kind[1]),
                                "sparse_ms": mean(per_kind[2]), "n_dense": n_dense, "n_select": n_select,
                                "n_sparse": n_sparse},
            "column_sparse_attn": {"ms": ms_alone, "tflops": sparse / (ms_alone * 1e-3) / 1e12,
                                   "frac_of_peak_burst": sparse / (ms_alone * 1e-3) / 1e12 / peak_burst,
                                   "peak_source": peak_src},
            "gpu_launches": (n_dense + 3 * n_select + 2 * n_sparse) * args.steps, "clocks": clk}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def losa_bytes(wl, union_counts):
    """Algorithmic HBM bytes of one block run: the first step reads the whole
    prefix K and V; a later step reads the K and V rows of its heads' unions;
    every step reads the block's Q, K, V (and the previous Q) and writes O and
    LSE. union_counts: [T, H] blocks per head (step 0: all)."""
    row = wl.d * 2
    full = 2 * wl.H * wl.P * row
    blk = wl.H * wl.B * (4 * row + 4)
    per_step = [full + blk]
    for t in range(1, union_counts.shape[0]):
        keys = float(union_counts[t].sum()) * wl.bk  # a ragged last prefix block counts whole
        per_step.append(2 * keys * row + blk + wl.H * wl.B * row)
    return per_step


def run_losa(args, dev, rank, world, barrier, max_over_ranks):
    """Block-wise generation (LoSA page, section 3): one bench step is one
    block's T denoising steps through sparsed_losa_block -- a dense first step
    over the whole prefix (and the per-token selection), then steps in which
    only the active tokens attend to the union of their blocks. The path is
    bound by HBM reads of the prefix cache: value = algorithmic bytes of the
    run / device time (GB/s). The L2 is flushed before every timed run."""
    import block_sparse_bidirectional_select_b200 as sp
    wl = BLOCK_WORKLOADS[args.block_workload]
    k_pre, v_pre, qs, ks, vs = (t.to(dev) for t in make_block_inputs(wl.scaled(seed=wl.seed + 7919 * rank)))
    stream = torch.cuda.current_stream()
    splits = sp.losa_splits(wl.H, wl.B, wl.P, wl.bq, wl.bk)
    ws = torch.empty(sp.losa_workspace_bytes(wl.H, wl.B, wl.P, wl.d, wl.bq, wl.bk, splits), dtype=torch.uint8,
                     device=dev)
    out = torch.empty_like(qs)
    lse = torch.empty((wl.T, wl.H, wl.B), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def one_run():
        return sp.losa_block(qs, ks, vs, k_pre, v_pre, n_sel=wl.n_sel, tau=wl.tau, bq=wl.bq, bk=wl.bk,
                             splits=splits, out=out, lse=lse, workspace=ws)

    for _ in range(args.warmup):
        res = one_run()
    sp.device_check()
    ucount = res.union_count.cpu().numpy()
    n_active = res.active.cpu().numpy().sum(axis=1)
    per_step_bytes = losa_bytes(wl, ucount)
    run_bytes = float(sum(per_step_bytes))
    # the block run captured once in a CUDA graph (the library's side stream
    # joins the capture through its fork / join events) and replayed: a later
    # step is a handful of short dependent kernels, whose launch gaps the
    # graph removes
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        one_run()
    graph.replay()
    torch.cuda.synchronize()
    sp.device_check()

    def timed(fn):
        total = 0.0
        for _ in range(args.steps):
            flush.zero_()
            s_ev = torch.cuda.Event(enable_timing=True)
            e_ev = torch.cuda.Event(enable_timing=True)
            s_ev.record(stream)
            fn()
            e_ev.record(stream)
            e_ev.synchronize()
            total += s_ev.elapsed_time(e_ev)
        return total

    torch.cuda.synchronize()
    barrier()
    clocks = ClockSampler(dev.index or 0)
    clocks.start()
    total = timed(graph.replay)
    barrier()
    clk = clocks.stop()
    total_ms = max_over_ranks(total)
    eager_ms = max_over_ranks(timed(one_run))
    sp.device_check()
    # the first (dense) step alone: 8 calls back to back (the GPU, not the
    # host, sets the pace: each reads the whole 0.5 GB prefix) between two
    # events; a later step's time is the rest of the block run over its T-1
    # steps (the C driver enqueues them back to back)
    flush.zero_()
    s_ev = torch.cuda.Event(enable_timing=True)
    e_ev = torch.cuda.Event(enable_timing=True)
    n_first = 8
    s_ev.record(stream)
    for _ in range(n_first):
        sp.losa_init(qs[0], ks[0], vs[0], k_pre, v_pre, n_sel=wl.n_sel, bq=wl.bq, bk=wl.bk, splits=splits,
                     workspace=ws)
    e_ev.record(stream)
    e_ev.synchronize()
    sp.device_check()
    first_ms = s_ev.elapsed_time(e_ev) / n_first
    block_ms = total_ms / args.steps
    peaks, peak_src = load_peaks()
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    gbs = run_bytes * args.steps * world / (total_ms * 1e-3) / 1e9
    step_ms = (block_ms - first_ms) / (wl.T - 1) if wl.T > 1 else None
    step_bytes = statistics.mean(per_step_bytes[1:]) if wl.T > 1 else None
    nkb = -(-wl.P // wl.bk)
    line = {"metric": "block-wise generation with active-token reuse: HBM GB/s of a block's steps",
            "value": gbs, "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "H": wl.H, "prefix": wl.P, "block": wl.B, "d": wl.d, "bq": wl.bq,
                       "bk": wl.bk, "blocks_per_token": wl.n_sel, "T": wl.T, "tau": wl.tau, "splits": splits,
                       "l2": "flushed before every timed run",
                       "parallelism": f"independent blocks x{world}" if world > 1 else "single"},
            "ms_per_denoise_step": total_ms / args.steps / wl.T,
            "first_step_ms": first_ms, "later_step_ms": step_ms,
            "timing": "block run replayed from a CUDA graph; eager launches beside it",
            "ms_per_step_eager": eager_ms / args.steps,
            "later_step_ms_eager": (eager_ms / args.steps - first_ms) / (wl.T - 1) if wl.T > 1 else None,
            "active_tokens_per_step": float(n_active[1:].mean()) if wl.T > 1 else None,
            "union_blocks_per_head": float(ucount[1:].mean()) if wl.T > 1 else None,
            "prefix_density": float(ucount[1:].mean()) / nkb if wl.T > 1 else None,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm, "unit": "GB/s", "frac": gbs / hbm,
                         "traffic": load_traffic(wl.name, "losa_kernels_sha256", LOSA_KERNEL_FILES).get("block_run"),
                         "traffic_unit": "DRAM bytes of one block run (its launches summed, ncu, caches flushed "
                                         "before each launch)",
                         "peak_source": peak_src},
            "later_step_roofline": None if step_ms is None else
            {"bound": "hbm", "achieved": step_bytes / (step_ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
             "frac": step_bytes / (step_ms * 1e-3) / 1e9 / hbm, "bytes": step_bytes},
            "first_step_roofline": {"bound": "hbm", "achieved": per_step_bytes[0] / (first_ms * 1e-3) / 1e9,
                                    "peak": hbm, "unit": "GB/s",
                                    "frac": per_step_bytes[0] / (first_ms * 1e-3) / 1e9 / hbm,
                                    "bytes": per_step_bytes[0]},
            "gpu_launches": (6 + 5 * (wl.T - 1) + 2) * args.steps, "clocks": clk}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def code_signature(src):
    """The kernel source without comments and blank lines: traffic figures
    stay valid across edits of the comments only."""
    lines = []
    for line in src.splitlines():
        code = line.split("//", 1)[0].strip()
        if code:
            lines.append(code)
    return "\n".join(lines)


ATTN_KERNEL_FILES = ("attn_kernel.cuh", "attn_list_kernel.cuh")
LOSA_KERNEL_FILES = ATTN_KERNEL_FILES + ("losa_kernels.cuh",)


def kernel_signature(files=ATTN_KERNEL_FILES):
    """sha256 of the kernels' code (comments and blank lines removed): by
    default the dense two-tile kernel and the block-sparse one-tile kernel;
    with LOSA_KERNEL_FILES also the block-wise path's own kernels."""
    import hashlib
    csrc = os.path.join(ROOT, "block_sparse_bidirectional_select_b200", "csrc")
    parts = []
    for name in files:
        with open(os.path.join(csrc, name)) as f:
            parts.append(code_signature(f.read()))
    return hashlib.sha256("\n".join(parts).encode()).hexdigest()


def load_traffic(workload, sha_key="attn_kernels_sha256", files=ATTN_KERNEL_FILES):
    """DRAM bytes from the committed ncu capture (profiles/traffic.json), used
    only while the kernels' source is the one that was captured: per launch
    of the attention kernels, or (sha_key "losa_kernels_sha256") per block
    run of the block-wise path."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        sha = kernel_signature(files)
    except (OSError, ValueError):
        return {}
    if t.get(sha_key) != sha:
        return {}
    return t.get(workload, {})


if __name__ == "__main__":
    sys.exit(main())
