#!/usr/bin/env python
"""Benchmark of the fused softmax cross-entropy hot path on B200.

One step = one forward and one backward pass over one batch of synthetic,
seeded input already resident in HBM (the row path: online log-sum-exp
forward, then the VJP from the saved lse; the fused-linear path: forward and
backward of Z = H W^T without storing Z). Default workload: 1,048,576 rows x
128 classes, fp32 logits ~N(0,1), 10% of targets at ignore_index=-100,
label smoothing 0.1.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload c2] [--also LIST]
    python bench.py --impl reference ...   (the float64 CPU oracle, timed)

Prints one JSON line (rank 0). With the default headline (c2) the line also
carries, under "workloads", the same measurements for every other workload
(c1, c3a, c3b, c4a, c4b, c5, soft, kl), each with its rates, roofline,
clocks and end-to-end rate; --also chooses them ("none" for the headline
alone). For N > 1 it is launched with torchrun, one rank per GPU; every rank
processes its own batch (rows are independent, no data-path collective), the
device time is the max over ranks and the value is the bytes of all ranks over
that time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from softmax_cross_entropy_lse_b200 import sharding  # noqa: E402
from softmax_cross_entropy_lse_b200 import workloads as wl  # noqa: E402

METRIC = "CE fwd and fwd+bwd GB/s and rows/s vs HBM roofline; fused-linear TFLOP/s"

# The pages' own numbers (Apple M5 Pro, MLX PR #4776 Benchmarks table, fix
# column): forward + backward milliseconds for the same shape and dtype.
# Another machine's numbers: context, not the target.
PAGE_FWD_BWD_MS = {"c2": 6.364, "c3a": 6.073, "c3b": 7.263}

ROW_WORKLOADS = {
    "c1": dict(desc="4096 x 1024 fp32 rows ~N(0,1), uniform targets", dt="f32", eps=0.0),
    "c2": dict(desc="1,048,576 x 128 fp32 rows ~N(0,1), 10% ignore_index=-100, label smoothing 0.1",
               dt="f32", eps=wl.C2_EPS),
    "c3a": dict(desc="8192 x 32000 bf16 rows ~N(0, std 2), bf16 dlogits", dt="bf16", eps=0.0),
    "c3b": dict(desc="2048 x 151,936 bf16 rows ~N(0, std 2), bf16 dlogits", dt="bf16", eps=0.0),
    "c4a": dict(desc="view x[:, :-1] of a (10, 119, 151,936) fp32 tensor vs t[:, 1:]", dt="f32",
                eps=0.0),
    "c4b": dict(desc="(2^27 + 2^20) x 8 fp32 rows ~N(0,1)", dt="f32", eps=0.0),
}


# Data-sheet peaks, reported beside the measured ones: HBM3e 8 TB/s and
# 2.25 PFLOP/s dense bf16 for one B200.
SPEC_HBM_GBS = 8000.0
SPEC_BF16_TFLOPS = 2250.0


def roofline(bound, kernel, achieved, peak, peak_src, traffic, algorithmic=None):
    """The roofline object of a JSON line: the fraction of the measured peak
    (the copy or GEMM rate measured on this machine's B200s) and, beside it, the
    fraction of the data-sheet peak."""
    spec = SPEC_HBM_GBS if bound == "hbm" else SPEC_BF16_TFLOPS
    r = {"bound": bound, "kernel": kernel, "achieved": round(achieved, 2), "peak": peak,
         "unit": "GB/s" if bound == "hbm" else "TFLOP/s", "frac": round(achieved / peak, 4),
         "traffic": traffic, "peak_source": peak_src, "spec_peak": spec,
         "frac_of_spec": round(achieved / spec, 4)}
    if algorithmic is not None:
        r["algorithmic_bytes_per_launch" if bound == "hbm" else "algorithmic_flop_per_launch"] = \
            algorithmic
    return r


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0), \
            d.get("bf16_tflops_sustained", 1400.0), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# Source files each pass's kernels are built from (the shared device code,
# the launch interface, the planner and the pass's own file).
PASS_SOURCES = {
    "forward": ["ce_rows_fwd.cu", "ce_device.cuh", "ce_launch.h", "ce_api.cu", "ce_sm100.cuh"],
    "backward": ["ce_rows_bwd.cu", "ce_device.cuh", "ce_launch.h", "ce_api.cu", "ce_sm100.cuh"],
}


def kernel_source_sha(files) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "softmax_cross_entropy_lse_b200", "csrc")
    for f in sorted(files):
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current sources of that pass's kernels (the entry's "sources", else
    PASS_SOURCES); else None."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload, {}).get(kernel)
    if not e:
        return None
    files = e.get("sources") or PASS_SOURCES.get(kernel)
    if not files or e.get("source_sha") != kernel_source_sha(files):
        return None
    return e.get("bytes_per_launch")


# -- clocks during the timed region ---------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = f"/tmp/ce_bench_clocks_{os.getpid()}.csv"

    def __enter__(self):
        try:
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.out.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
                except ValueError:
                    continue
        os.remove(self.path)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v == "Active"})
        loaded = [r for r in rows if r[2] > 200.0] or rows
        return {"sm_mhz": float(np.median([r[0] for r in loaded])),
                "sm_max_mhz": float(max(r[1] for r in rows)), "reasons": reasons,
                "samples": len(rows), "power_w_max": float(max(r[2] for r in rows))}


# -- distributed plumbing (softmax_cross_entropy_lse_b200.sharding) --------------------------------
def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if world > 1 and world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}")
    return sharding.init_from_env("nccl", timeout_s=120)


# -- row workloads ------------------------------------------------------------------------
def make_rows(workload: str, seed: int):
    """Host arrays: (logits storage, float32 values, targets, layout kind)."""
    if workload == "c4a":
        x, t = wl.c4a(seed)
        return x, x, t, "view"
    if workload == "c4b":
        n = (wl.C4B_ROWS + wl.C4B_CHUNK - 1) // wl.C4B_CHUNK
        chunks = [wl.c4b_chunk(k, seed) for k in range(n)]
        z = np.concatenate([c[0] for c in chunks])
        y = np.concatenate([c[1] for c in chunks])
        return z, z, y, "plain"
    gen = {"c1": wl.c1, "c2": wl.c2, "c3a": wl.c3a, "c3b": wl.c3b}.get(workload)
    if gen is None:
        raise SystemExit(f"unknown workload {workload}")
    z, z32, y = gen(seed)
    return z, z32, y, "plain"


def bench_rows(args, rk):
    import torch
    import softmax_cross_entropy_lse_b200 as ce
    world = rk.world
    spec = ROW_WORKLOADS[args.workload]
    dt, eps = spec["dt"], spec["eps"]
    z, z32, y, kind = make_rows(args.workload, seed=rk.rank)
    if args.rows and kind == "plain":  # a smaller batch of the same rows (profiling)
        z, z32, y = z[:args.rows], z32[:args.rows], y[:args.rows]
    dev = torch.device("cuda", torch.cuda.current_device())
    if dt == "bf16":
        z_h = torch.from_numpy(np.ascontiguousarray(z).view(np.int16)).view(torch.bfloat16)
    else:
        z_h = torch.from_numpy(np.ascontiguousarray(z))
    y_h = torch.from_numpy(np.ascontiguousarray(y))
    z_d, y_d = z_h.to(dev), y_h.to(dev)

    def views(zd, yd):
        return (zd[:, :-1], yd[:, 1:]) if kind == "view" else (zd, yd)

    zv, yv = views(z_d, y_d)
    N = zv.numel() // zv.shape[-1]
    V = zv.shape[-1]
    esz = zv.element_size()
    yflat = (y[:, 1:] if kind == "view" else y).reshape(-1)
    # the mean over the global batch: every rank scales by 1 / (rows counted on
    # all ranks), one all-reduce of an integer when the batch is formed
    g = torch.full((1,), sharding.mean_grad_scale(rk, yflat), dtype=torch.float32, device=dev)
    dz = torch.empty(z_d.shape, dtype=z_d.dtype, device=dev)
    dzv = views(dz, y_d)[0]
    ws_bytes = ce.ce_workspace_size(N, V, zv.dtype)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    # L2: a batch larger than L2 is read from HBM every step; a small batch
    # rotates through enough copies that each is evicted before its reuse.
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    nbuf = 1
    if z_d.numel() * esz < 2 * l2:
        nbuf = int(np.ceil(3 * l2 / (z_d.numel() * esz)))
    bufs = [(z_d, y_d, dz)] + [(z_d.clone(), y_d.clone(), torch.empty_like(dz))
                               for _ in range(nbuf - 1)]

    # per-row outputs allocated once per buffer: no allocation in a timed region
    outs = [ce.ForwardResult(*(torch.empty(N, dtype=torch.float32, device=dev) for _ in range(3)),
                             None) for _ in range(nbuf)]

    def fwd(i):
        zb, yb, _ = bufs[i % nbuf]
        zvb, yvb = views(zb, yb)
        return ce.ce_forward(zvb, yvb, eps, -100, workspace=ws, out=outs[i % nbuf])

    def bwd(i, r):
        zb, yb, db = bufs[i % nbuf]
        zvb, yvb = views(zb, yb)
        ce.ce_backward(g, zvb, yvb, r.lse, r.lse_lo, eps, -100, dlogits=views(db, yb)[0])

    def fused(i):
        zb, yb, db = bufs[i % nbuf]
        zvb, yvb = views(zb, yb)
        ce.ce_forward_backward(zvb, yvb, g, eps, -100, dlogits=views(db, yb)[0], workspace=ws,
                               out=outs[i % nbuf])

    fwd_bytes = N * V * esz + 12 * N
    bwd_bytes = 2 * N * V * esz + 12 * N
    step_bytes = fwd_bytes + bwd_bytes
    launches_per_step = (2 if ws_bytes > 0 else 1) + 1

    # A batch that fits in L2 takes microseconds on the device, less than the
    # host needs to issue its calls: its timed loops are captured once as CUDA
    # graphs and replayed, so the device time is what is measured.
    use_graph = nbuf > 1
    fixed = [fwd(i) for i in range(nbuf)]  # saved lse per buffer (backward-only loops)
    torch.cuda.synchronize()
    fixed = [ce.ForwardResult(r.loss, r.lse.clone(), r.lse_lo.clone(), None) for r in fixed]

    def run_loop(kind, steps, ev=None):
        for i in range(steps):
            if ev is not None:
                ev[i][0].record(stream)
            if kind == "fused":
                fused(i)
                continue
            r = fwd(i) if kind in ("step", "fwd") else fixed[i % nbuf]
            if ev is not None:
                ev[i][1].record(stream)
            if kind in ("step", "bwd"):
                bwd(i, r)
            if ev is not None:
                ev[i][2].record(stream)

    def timed(kind, steps):
        """Device ms for `steps` iterations (max over ranks); per-iteration
        events in eager mode."""
        evs = None
        if use_graph:
            gr = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream()
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                run_loop(kind, min(steps, nbuf))
            stream.wait_stream(side)
            with torch.cuda.graph(gr):
                run_loop(kind, steps)
            gr.replay()
        else:
            for i in range(args.warmup):
                run_loop(kind, 1)
            evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        sharding.barrier(rk)
        torch.cuda.synchronize()
        t0.record(stream)
        if use_graph:
            gr.replay()
        else:
            run_loop(kind, steps, evs)
        t1.record(stream)
        torch.cuda.synchronize()
        sharding.barrier(rk)
        return sharding.max_over_ranks(rk, t0.elapsed_time(t1)), evs

    for i in range(args.warmup):
        run_loop("step", 1)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        ms, evs = timed("step", args.steps)
    if use_graph:
        fwd_ms = timed("fwd", args.steps)[0] / args.steps
        bwd_ms = timed("bwd", args.steps)[0] / args.steps
    else:
        fwd_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
        bwd_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))

    # the forward alone, back to back: inside the step the forward also pays for
    # writing back the gradient lines the previous backward left dirty in L2
    fwd_alone_ms = timed("fwd", args.steps)[0] / args.steps if not use_graph else fwd_ms

    # the same step through the fused call (one read of each row that fits on chip)
    fused_ms = timed("fused", args.steps)[0] / args.steps

    # end to end through the public API with host buffers: pinned host inputs
    # copied in, forward + backward, the per-row loss copied out, every step
    z_pin = z_h.pin_memory()
    y_pin = y_h.pin_memory()
    loss_h = torch.empty(N, dtype=torch.float32).pin_memory()

    def e2e_step():
        z_d.copy_(z_pin, non_blocking=True)
        y_d.copy_(y_pin, non_blocking=True)
        zv2, yv2 = views(z_d, y_d)
        r = ce.ce_forward(zv2, yv2, eps, -100, workspace=ws, out=outs[0])
        ce.ce_backward(g, zv2, yv2, r.lse, r.lse_lo, eps, -100, dlogits=dzv)
        loss_h.copy_(r.loss, non_blocking=True)

    e2e_steps = max(2, min(args.steps, 10))
    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    sharding.barrier(rk)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = sharding.max_over_ranks(rk, a.elapsed_time(b)) / e2e_steps
    h2d = z_h.numel() * z_h.element_size() + y_h.numel() * y_h.element_size()
    d2h = 4 * N

    peak_hbm, _, _, peak_src = load_peaks()
    dom, dom_ms, dom_bytes = ("backward", bwd_ms, bwd_bytes) if bwd_ms >= fwd_ms else \
        ("forward", fwd_ms, fwd_bytes)
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    value = world * step_bytes * args.steps / (ms * 1e-3) / 1e9
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5),
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32" if dt == "f32" else "bf16", "data": "synthetic",
        "rows_per_s": round(world * N * args.steps / (ms * 1e-3), 1),
        "fwd_GBs": round(fwd_bytes / (fwd_ms * 1e-3) / 1e9, 2),
        "fwd_rows_per_s": round(N / (fwd_ms * 1e-3), 1),
        "fwd_alone_GBs": round(fwd_bytes / (fwd_alone_ms * 1e-3) / 1e9, 2),
        "bwd_GBs": round(bwd_bytes / (bwd_ms * 1e-3) / 1e9, 2),
        "config": {"workload": f"{args.workload}: {spec['desc']}; forward + backward",
                   "rows": N, "classes": V, "label_smoothing": eps, "ignore_index": -100,
                   "bytes_per_step": step_bytes,
                   "l2": ("inputs larger than L2" if nbuf == 1 else
                          f"{nbuf} rotating input buffers (total larger than L2); "
                          "timed loops captured as CUDA graphs and replayed"),
                   "parallelism": f"rows sharded over {world} rank(s), no data-path collective"},
        "e2e": {"value": round(world * step_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "roofline": roofline("hbm", dom, achieved, peak_hbm, peak_src,
                             recorded_traffic(args.workload, dom), dom_bytes),
    }
    if fused_ms is not None:
        fused_bytes = 2 * N * V * esz + 16 * N
        out["fused"] = {"call": "ce_forward_backward", "ms_per_step": round(fused_ms, 5),
                        "GB/s": round(fused_bytes / (fused_ms * 1e-3) / 1e9, 2),
                        "algorithmic_bytes": fused_bytes,
                        "rows_per_s": round(world * N / (fused_ms * 1e-3), 1),
                        "speedup_vs_separate": round((ms / args.steps) / fused_ms, 3)}
    if args.workload in PAGE_FWD_BWD_MS:
        page_gbs = step_bytes / (PAGE_FWD_BWD_MS[args.workload] * 1e-3) / 1e9
        out["vs_baseline"] = round(value / page_gbs, 2)
        out["vs_apple_m5pro_mlx"] = out["vs_baseline"]
        out["vs_baseline_basis"] = (
            f"value / the pages' Apple M5 Pro MLX rate for this shape ({page_gbs:.1f} GB/s from "
            f"{PAGE_FWD_BWD_MS[args.workload]} ms forward + backward, MLX PR #4776 Benchmarks, "
            "fix column): another machine's number, context only")
    clocks = clk.summary()
    if clocks:
        out["clocks"] = clocks
    return out, (z32, y, eps, kind)


# -- probability (soft) targets --------------------------------------------------------------
SOFT_DESC = ("8192 x 32000 bf16 logits ~N(0, std 2) against bf16 target distributions "
             "(normalised U[0,1) draws), bf16 dlogits; forward + backward")


def soft_inputs(seed: int, N: int = 8192, V: int = 32000):
    rng = np.random.default_rng(seed)
    z, _ = wl.encode(rng.standard_normal((N, V), dtype=np.float32) * 2, "bf16")
    t = rng.random((N, V), dtype=np.float32)
    t /= t.sum(1, keepdims=True)
    t, _ = wl.encode(t, "bf16")
    return z, t


def bench_soft(args, rk):
    import torch
    import softmax_cross_entropy_lse_b200 as ce
    world = rk.world
    z, t = soft_inputs(rk.rank)
    if args.rows:
        z, t = z[:args.rows], t[:args.rows]
    dev = torch.device("cuda", torch.cuda.current_device())
    z_h = torch.from_numpy(np.ascontiguousarray(z).view(np.int16)).view(torch.bfloat16)
    t_h = torch.from_numpy(np.ascontiguousarray(t).view(np.int16)).view(torch.bfloat16)
    z_d, t_d = z_h.to(dev), t_h.to(dev)
    N, V = z_d.shape
    g = torch.full((1,), 1.0 / N, dtype=torch.float32, device=dev)
    dz = torch.empty_like(z_d)
    stream = torch.cuda.current_stream()
    fwd_bytes = N * V * 4 + 16 * N
    bwd_bytes = N * V * 6 + 16 * N
    step_bytes = fwd_bytes + bwd_bytes

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        r = ce.ce_soft_forward(z_d, t_d)
        if ev is not None:
            ev[1].record(stream)
        ce.ce_soft_backward(g, z_d, t_d, r.lse, r.lse_lo, r.target_sum, dlogits=dz)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        sharding.barrier(rk)
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize()
        sharding.barrier(rk)
    ms = sharding.max_over_ranks(rk, t0.elapsed_time(t1))
    fwd_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    bwd_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    # end to end: logits and targets copied in from pinned host memory, loss out
    z_pin, t_pin = z_h.pin_memory(), t_h.pin_memory()
    loss_h = torch.empty(N, dtype=torch.float32).pin_memory()

    def e2e_step():
        z_d.copy_(z_pin, non_blocking=True)
        t_d.copy_(t_pin, non_blocking=True)
        r = ce.ce_soft_forward(z_d, t_d)
        ce.ce_soft_backward(g, z_d, t_d, r.lse, r.lse_lo, r.target_sum, dlogits=dz)
        loss_h.copy_(r.loss, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    sharding.barrier(rk)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(3):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = sharding.max_over_ranks(rk, a.elapsed_time(b)) / 3
    peak_hbm, _, _, peak_src = load_peaks()
    dom, dom_ms, dom_bytes = ("backward", bwd_ms, bwd_bytes) if bwd_ms >= fwd_ms else \
        ("forward", fwd_ms, fwd_bytes)
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    out = {
        "metric": METRIC, "value": round(world * step_bytes * args.steps / (ms * 1e-3) / 1e9, 2),
        "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms / args.steps, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "fwd_GBs": round(fwd_bytes / (fwd_ms * 1e-3) / 1e9, 2),
        "bwd_GBs": round(bwd_bytes / (bwd_ms * 1e-3) / 1e9, 2),
        "config": {"workload": f"soft: {SOFT_DESC}", "rows": N, "classes": V,
                   "bytes_per_step": step_bytes, "l2": "inputs larger than L2",
                   "parallelism": f"rows sharded over {world} rank(s), no data-path collective"},
        "e2e": {"value": round(world * step_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": 2 * N * V * 2, "d2h_bytes_per_step": 4 * N},
        "gpu_launches": 2 * args.steps,
        "roofline": roofline("hbm", dom, achieved, peak_hbm, peak_src,
                             recorded_traffic("soft", dom), dom_bytes),
    }
    clocks = clk.summary()
    if clocks:
        out["clocks"] = clocks
    return out, None


# -- KL divergence of a student from a teacher -------------------------------------------------
KL_DESC = ("512 x 151,936 fp32 student and teacher logits, both ~N(0, 16) "
           "(the shape and draw of the fused KL check in \"One barrier short\"); forward + backward")


def kl_inputs(seed: int, N: int = 512, V: int = 151936):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((N, V), dtype=np.float32) * 4,
            rng.standard_normal((N, V), dtype=np.float32) * 4)


def bench_kl(args, rk):
    import torch
    import softmax_cross_entropy_lse_b200 as ce
    world = rk.world
    q, p = kl_inputs(rk.rank)
    if args.rows:
        q, p = q[:args.rows], p[:args.rows]
    dev = torch.device("cuda", torch.cuda.current_device())
    q_h, p_h = torch.from_numpy(q), torch.from_numpy(p)
    q_d, p_d = q_h.to(dev), p_h.to(dev)
    N, V = q_d.shape
    g = torch.full((1,), 1.0 / N, dtype=torch.float32, device=dev)
    dq = torch.empty_like(q_d)
    stream = torch.cuda.current_stream()
    fwd_bytes = 2 * N * V * 4 + 20 * N
    bwd_bytes = 3 * N * V * 4 + 20 * N
    step_bytes = fwd_bytes + bwd_bytes

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        r = ce.kl_forward(q_d, p_d)
        if ev is not None:
            ev[1].record(stream)
        ce.kl_backward(g, q_d, p_d, r, dstudent=dq)
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        sharding.barrier(rk)
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize()
        sharding.barrier(rk)
    ms = sharding.max_over_ranks(rk, t0.elapsed_time(t1))
    fwd_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    bwd_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    q_pin, p_pin = q_h.pin_memory(), p_h.pin_memory()
    loss_h = torch.empty(N, dtype=torch.float32).pin_memory()

    def e2e_step():
        q_d.copy_(q_pin, non_blocking=True)
        p_d.copy_(p_pin, non_blocking=True)
        r = ce.kl_forward(q_d, p_d)
        ce.kl_backward(g, q_d, p_d, r, dstudent=dq)
        loss_h.copy_(r.loss, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    sharding.barrier(rk)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(3):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = sharding.max_over_ranks(rk, a.elapsed_time(b)) / 3
    peak_hbm, _, _, peak_src = load_peaks()
    dom, dom_ms, dom_bytes = ("backward", bwd_ms, bwd_bytes) if bwd_ms >= fwd_ms else \
        ("forward", fwd_ms, fwd_bytes)
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    out = {
        "metric": METRIC, "value": round(world * step_bytes * args.steps / (ms * 1e-3) / 1e9, 2),
        "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms / args.steps, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "fwd_GBs": round(fwd_bytes / (fwd_ms * 1e-3) / 1e9, 2),
        "bwd_GBs": round(bwd_bytes / (bwd_ms * 1e-3) / 1e9, 2),
        "config": {"workload": f"kl: {KL_DESC}", "rows": N, "classes": V,
                   "bytes_per_step": step_bytes, "l2": "inputs larger than L2",
                   "parallelism": f"rows sharded over {world} rank(s), no data-path collective"},
        "e2e": {"value": round(world * step_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": 2 * N * V * 4, "d2h_bytes_per_step": 4 * N},
        "gpu_launches": 2 * args.steps,
        "roofline": roofline("hbm", dom, achieved, peak_hbm, peak_src,
                             recorded_traffic("kl", dom), dom_bytes),
    }
    clocks = clk.summary()
    if clocks:
        out["clocks"] = clocks
    return out, None


# -- fused-linear workload -------------------------------------------------------------------
def bench_linear(args, rk):
    import torch
    import softmax_cross_entropy_lse_b200 as ce
    world = rk.world
    N, V, D = args.linear_shape
    hb, hf, wb, wf, y = wl.c5(seed=rk.rank, N=N, V=V, D=D)
    dev = torch.device("cuda", torch.cuda.current_device())
    H_h = torch.from_numpy(hb.view(np.int16)).view(torch.bfloat16)
    W_h = torch.from_numpy(wb.view(np.int16)).view(torch.bfloat16)
    y_h = torch.from_numpy(y)
    H, W, yd = H_h.to(dev), W_h.to(dev), y_h.to(dev)
    g = torch.full((1,), sharding.mean_grad_scale(rk, y), dtype=torch.float32, device=dev)
    L = ce.lib()
    ws_f = torch.empty(max(L.linear_ce_workspace_size(N, V, D, 0), 16), dtype=torch.uint8,
                       device=dev)
    ws_b = torch.empty(max(L.linear_ce_backward_workspace_size(N, V, D, 0), 16),
                       dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        loss, lse = ce.linear_ce_forward(H, W, yd, workspace=ws_f)
        if ev is not None:
            ev[1].record(stream)
        ce.linear_ce_backward(g, H, W, yd, lse, workspace=ws_b)
        if ev is not None:
            ev[2].record(stream)

    fwd_flop = 2.0 * N * V * D
    bwd_flop = 3 * fwd_flop
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clk:
        sharding.barrier(rk)
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(args.steps):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize()
        sharding.barrier(rk)
    ms = sharding.max_over_ranks(rk, t0.elapsed_time(t1))
    fwd_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in evs]))
    bwd_ms = float(np.mean([e[1].elapsed_time(e[2]) for e in evs]))
    _, peak_burst, peak_sust, src = load_peaks()
    step_flop = fwd_flop + bwd_flop
    value = world * step_flop * args.steps / (ms * 1e-3) / 1e12
    # e2e: H, W and targets copied in from pinned host memory each step, loss out
    Hp, Wp, yp = H_h.pin_memory(), W_h.pin_memory(), y_h.pin_memory()
    loss_h = torch.empty(N, dtype=torch.float32).pin_memory()

    def e2e_step():
        H.copy_(Hp, non_blocking=True)
        W.copy_(Wp, non_blocking=True)
        yd.copy_(yp, non_blocking=True)
        loss, lse = ce.linear_ce_forward(H, W, yd, workspace=ws_f)
        ce.linear_ce_backward(g, H, W, yd, lse, workspace=ws_b)
        loss_h.copy_(loss, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    sharding.barrier(rk)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(2):
        e2e_step()
    b.record(stream)
    torch.cuda.synchronize()
    e2e_ms = sharding.max_over_ranks(rk, a.elapsed_time(b)) / 2
    dom, dom_ms, dom_flop = ("backward", bwd_ms, bwd_flop) if bwd_ms >= fwd_ms else \
        ("forward", fwd_ms, fwd_flop)
    achieved = dom_flop / (dom_ms * 1e-3) / 1e12
    ws_sizes = {"forward": int(ws_f.numel()), "backward": int(ws_b.numel())}
    del ws_f, ws_b
    dvf = dense_vs_fused(H, W, yd, g, steps=3)
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "fwd_tflops": round(fwd_flop / (fwd_ms * 1e-3) / 1e12, 2), "fwd_ms": round(fwd_ms, 4),
        "bwd_ms": round(bwd_ms, 4),
        "workspace_bytes": ws_sizes,
        "config": {"workload": f"c5: fused linear CE, H ({N}, {D}) bf16 ~N(0,1), W ({V}, {D}) "
                               "bf16 ~N(0, std 0.02), forward + backward (logits recomputed)",
                   "N": N, "V": V, "D": D, "flop_per_step": step_flop,
                   "l2": "operands larger than L2 (W is 1.24 GB)",
                   "parallelism": f"rows sharded over {world} rank(s), no data-path collective"},
        "e2e": {"value": round(world * step_flop / (e2e_ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": (N * D + V * D) * 2 + 4 * N, "d2h_bytes_per_step": 4 * N},
        "gpu_launches": (2 + 3 * ((V + 8191) // 8192)) * args.steps,
        "roofline": roofline("tensor", dom, achieved, peak_sust, src + " (sustained)",
                             recorded_traffic("c5", dom), dom_flop),
    }
    out["dense_vs_fused"] = dvf
    clocks = clk.summary()
    if clocks:
        out["clocks"] = clocks
    return out, None


def dense_vs_fused(H, W, y, g, steps: int = 3) -> dict:
    """The comparison of Ineshin's section 3 on the same inputs: time and peak
    device memory of one forward + backward step, (a) fused (Z = H W^T never
    stored; this library) and (b) materialised: Z computed by a library GEMM
    (torch.matmul, cuBLAS) and stored in bf16, the row kernels of this library
    on it (the gradient written over Z), and library GEMMs for dH = G W and
    dW = G^T H. Arm (b) is a comparison arm only. Peak memory is what the step
    allocates on top of H, W, the targets and g: outputs, workspaces, Z."""
    import torch
    import softmax_cross_entropy_lse_b200 as ce
    stream = torch.cuda.current_stream()

    def fused():
        loss, lse = ce.linear_ce_forward(H, W, y)
        ev[1].record(stream)
        dH, dW = ce.linear_ce_backward(g, H, W, y, lse)
        return loss, dH, dW

    def dense():
        Z = torch.matmul(H, W.t())
        r = ce.ce_forward(Z, y)
        ev[1].record(stream)
        ce.ce_backward(g, Z, y, r.lse, r.lse_lo, dlogits=Z)
        dH = torch.matmul(Z, W)
        dW = torch.matmul(Z.t(), H)
        return r.loss, dH, dW

    res = {}
    for name, fn in (("fused", fused), ("materialised", dense)):
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        release_device_memory()
        fn()  # warm-up (library handles, kernel attributes)
        release_device_memory()
        base = torch.cuda.memory_allocated()
        torch.cuda.reset_peak_memory_stats()
        fwd, bwd = [], []
        for _ in range(steps):
            ev[0].record(stream)
            outs = fn()
            ev[2].record(stream)
            torch.cuda.synchronize()
            fwd.append(ev[0].elapsed_time(ev[1]))
            bwd.append(ev[1].elapsed_time(ev[2]))
            del outs
        peak = torch.cuda.max_memory_allocated() - base
        res[name] = {"fwd_ms": round(float(np.median(fwd)), 3),
                     "bwd_ms": round(float(np.median(bwd)), 3),
                     "step_ms": round(float(np.median(np.add(fwd, bwd))), 3),
                     "peak_step_bytes": int(peak)}
    res["fused_speedup"] = round(res["materialised"]["step_ms"] / res["fused"]["step_ms"], 3)
    res["memory_ratio"] = round(res["materialised"]["peak_step_bytes"] /
                                max(res["fused"]["peak_step_bytes"], 1), 3)
    res["note"] = ("materialised arm: Z = H W^T by torch.matmul (cuBLAS) stored in bf16, this "
                   "library's row forward and VJP on it, dH and dW by torch.matmul; "
                   "dH and dW in bf16 in both arms")
    return res


# -- CPU oracle ---------------------------------------------------------------------------------
class OracleRows:
    """The float64 oracle (forward + backward) over whole rows of a row workload."""

    def __init__(self, workload, host=None):
        import oracle
        self.orc = oracle.get()
        spec = ROW_WORKLOADS[workload]
        self.eps = spec["eps"]
        self.esz = 4 if spec["dt"] == "f32" else 2
        if host is None:
            _, z32, y, kind = make_rows(workload, 0)
        else:
            z32, y, kind = host[0], host[1], host[3]
        if kind == "view":
            V = z32.shape[-1]
            z32 = z32[:, :-1].reshape(-1, V)
            y = y[:, 1:].reshape(-1)
        self.z32, self.y = z32, y
        self.N, self.V = z32.shape
        self.bytes_per_row = 3 * self.V * self.esz + 24
        self.cursor = 0

    def run(self, rows: int) -> None:
        done = 0
        chunk = max(1, int(5e7 // self.V))
        while done < rows:
            lo = self.cursor % self.N
            n = min(chunk, rows - done, self.N - lo)
            zc = self.z32[lo:lo + n].astype(np.float64)
            self.orc.ce_forward(zc, self.y[lo:lo + n], self.eps)
            self.orc.ce_backward(zc, self.y[lo:lo + n], 1.0, self.eps)
            self.cursor += n
            done += n

    def rows_for(self, seconds: float) -> int:
        probe = min(self.N, max(1, int(2e6 // self.V)))
        t = time.perf_counter()
        self.run(probe)
        per_row = max((time.perf_counter() - t) / probe, 1e-9)
        self.cursor = 0
        return int(max(1, seconds / per_row))


class OracleLinear:
    """The float64 oracle on whole rows of the fused-linear workload (loss,
    lse and the dH row of each sampled row)."""

    def __init__(self):
        import oracle
        self.orc = oracle.get()
        self.N, self.V, self.D = 8192, 151936, 4096
        _, self.hf, _, self.wf, self.y = wl.c5(seed=0)
        self.cursor = 0
        self.flop_per_row = 4.0 * self.V * self.D

    def run(self, rows: int) -> None:
        r = (self.cursor + np.arange(rows)) % self.N
        self.orc.linear_ce_forward_rows(self.hf, self.wf, self.y, rows=r)
        self.orc.linear_ce_dh_rows(self.hf, self.wf, self.y, 1.0 / self.N, rows=r)
        self.cursor += rows

    def rows_for(self, seconds: float) -> int:
        n = max(1, self.orc.num_threads())
        t = time.perf_counter()
        self.run(n)
        per_row = (time.perf_counter() - t) / n
        self.cursor = 0
        return int(max(n, (seconds / per_row) // n * n))


class OracleSoft(OracleRows):
    """The float64 oracle for probability targets (forward + backward)."""

    def __init__(self):
        import oracle
        self.orc = oracle.get()
        z, t = soft_inputs(0)
        self.z32 = wl.f32_from_bf16_bits(z)
        self.t32 = wl.f32_from_bf16_bits(t)
        self.N, self.V = self.z32.shape
        self.bytes_per_row = 5 * self.V * 2 + 32
        self.cursor = 0

    def run(self, rows: int) -> None:
        done = 0
        chunk = max(1, int(5e7 // self.V))
        while done < rows:
            lo = self.cursor % self.N
            n = min(chunk, rows - done, self.N - lo)
            zc = self.z32[lo:lo + n].astype(np.float64)
            tc = self.t32[lo:lo + n].astype(np.float64)
            self.orc.ce_soft_forward(zc, tc)
            self.orc.ce_soft_backward(zc, tc, 1.0)
            self.cursor += n
            done += n


class OracleKl(OracleRows):
    """The float64 oracle for the KL divergence (forward + backward)."""

    def __init__(self):
        import oracle
        self.orc = oracle.get()
        self.q32, self.p32 = kl_inputs(0)
        self.N, self.V = self.q32.shape
        self.bytes_per_row = 5 * self.V * 4 + 40
        self.cursor = 0

    def run(self, rows: int) -> None:
        done = 0
        chunk = max(1, int(5e7 // self.V))
        while done < rows:
            lo = self.cursor % self.N
            n = min(chunk, rows - done, self.N - lo)
            q = self.q32[lo:lo + n].astype(np.float64)
            p = self.p32[lo:lo + n].astype(np.float64)
            self.orc.kl_forward(q, p)
            self.orc.kl_backward(q, p, 1.0)
            self.cursor += n
            done += n


def _oracle_for(workload, host=None):
    if workload == "soft":
        return OracleSoft()
    if workload == "kl":
        return OracleKl()
    return OracleRows(workload, host)


def oracle_baseline(workload, seconds: float, host=None):
    """(value, unit, cores, sample) of the oracle timed for about `seconds`."""
    if workload == "c5":
        o = OracleLinear()
        rows = o.rows_for(seconds)
        t = time.perf_counter()
        o.run(rows)
        dt = time.perf_counter() - t
        return (rows * o.flop_per_row / dt / 1e12, "TFLOP/s", o.orc.num_threads(),
                f"{rows} of 8192 rows of c5 (loss, lse and dH rows), {dt:.1f} s")
    o = _oracle_for(workload, host)
    rows = min(o.rows_for(seconds), 50 * o.N)
    t = time.perf_counter()
    o.run(rows)
    dt = time.perf_counter() - t
    return (rows * o.bytes_per_row / dt / 1e9, "GB/s", o.orc.num_threads(),
            f"{rows} rows of {workload} ({rows / o.N:.3g} batches), forward + backward, {dt:.1f} s")


def run_reference(args):
    """The reference arm: the float64 oracle, as it stands, on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    if args.workload == "c5":
        o = OracleLinear()
        unit, per_row = "TFLOP/s", o.flop_per_row / 1e12
    else:
        o = _oracle_for(args.workload)
        unit, per_row = "GB/s", o.bytes_per_row / 1e9
    # each step a bounded sample, so the whole run stays within about two minutes
    step_s = min(2.0, 120.0 / (args.steps + args.warmup))
    rows = o.rows_for(step_s)
    for _ in range(args.warmup):
        o.run(rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        o.run(rows)
    wall = time.perf_counter() - t0
    value = rows * args.steps * per_row / wall
    cores = o.orc.num_threads()
    sample = f"{rows} rows of {args.workload} per step, forward + backward in float64"
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": unit,
            "n_gpus": int(os.environ.get("WORLD_SIZE", args.gpus)), "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(wall * 1e3 / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "sample_rows_per_step": rows},
            "gpu_launches": 0,
            "cpu_baseline": {"value": round(value, 4), "unit": unit, "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


EXTRA_WORKLOADS = ["c1", "c3a", "c3b", "c4a", "c4b", "c5", "soft", "kl"]
SUMMARY_KEYS = ("value", "unit", "ms_per_step", "steps", "dtype", "rows_per_s", "fwd_GBs",
                "fwd_rows_per_s", "fwd_alone_GBs", "bwd_GBs", "fwd_tflops", "fwd_ms", "bwd_ms", "workspace_bytes",
                "vs_baseline", "vs_baseline_basis", "gpu_launches", "roofline", "fused", "clocks",
                "e2e", "config", "dense_vs_fused")


def run_workload(args, rk, name):
    if name == "c5":
        return bench_linear(args, rk)
    if name == "soft":
        return bench_soft(args, rk)
    if name == "kl":
        return bench_kl(args, rk)
    args.workload = name
    return bench_rows(args, rk)


def workload_summary(out: dict) -> dict:
    """The parts of a workload's JSON line kept under the headline's 'workloads'."""
    return {k: out[k] for k in SUMMARY_KEYS if k in out}


def release_device_memory() -> None:
    import gc
    import torch
    gc.collect()
    torch.cuda.synchronize()
    torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="c2", choices=sorted(ROW_WORKLOADS) + ["c5", "soft", "kl"])
    ap.add_argument("--also", default=None,
                    help="comma-separated workloads measured after the headline one and reported "
                         "under 'workloads' (default: every other workload when the headline is "
                         "c2, none otherwise; 'none' for none)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--rows", type=int, default=0,
                    help="use only the first ROWS rows of a row workload (profiling small cases)")
    ap.add_argument("--linear-shape", default="8192,151936,4096",
                    help="N,V,D of the fused-linear workload (c5 is 8192,151936,4096)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    args.linear_shape = tuple(int(x) for x in args.linear_shape.split(","))
    if args.impl == "reference":
        return run_reference(args)

    import torch
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    rk = dist_setup(args.gpus)
    out, host = run_workload(args, rk, args.workload)
    if rk.rank == 0 and rk.world == 1 and not args.no_cpu_baseline:
        v, unit, cores, sample = oracle_baseline(args.workload, 12.0, host)
        out["cpu_baseline"] = {"value": round(v, 4), "unit": unit, "cores": cores,
                               "kind": "oracle", "sample": sample}
    host = None
    also = args.also
    if also is None:
        also = ",".join(EXTRA_WORKLOADS) if args.workload == "c2" and not args.rows else "none"
    extra = [w for w in also.split(",") if w and w != "none" and w != args.workload]
    if extra:
        out["workloads"] = {}
        sub = argparse.Namespace(**vars(args))
        sub.rows = 0
        sub.steps = min(args.steps, 20)
        sub.warmup = max(3, min(args.warmup, 5))
        for w in extra:
            sub.workload = w
            o, _ = run_workload(sub, rk, w)
            out["workloads"][w] = workload_summary(o)
            release_device_memory()
    if rk.group is not None:
        rk.group.barrier()
        rk.group.destroy_process_group()
    if rk.rank == 0:
        print(json.dumps(out), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
