#!/usr/bin/env python
"""Benchmark of the timestep-adaptive masked INT8 linear on B200.

A step is one denoising step of a whole workload: for every block and every linear of the
block, tasq_linear_forward(x, layer, step) = block-Hadamard INT8 prologue + masked INT8 GEMM,
with the step's per-layer bit widths read from the device schedule table. Every (block,
layer) has its own weights and its own activation buffer, so each step streams its whole
input set from HBM (larger than L2).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload cogvideox] [--impl tasq|reference]

The default workload is the largest one that fits a GPU, the CogVideoX-5B-shaped video DiT
(17776 tokens, 42 blocks of {qkv 3072->9216, proj 3072->3072, fc1 3072->12288, fc2 12288->3072}).

N > 1 runs under torchrun, one process per GPU, each an independent replica of the whole
workload (the path shards along tokens with no exchange); the time is the max over ranks.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import csv
import datetime
import io
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "masked-INT8 linear TOPS & tokens/s per denoise step; % of B200 INT8 tensor peak"
# INT8 dense tensor peak = measured BF16 cuBLAS peak x (4.5 POPS INT8 / 2.25 PFLOPS BF16 nominal)
INT8_OVER_BF16 = 2.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--workload", default="cogvideox", choices=list(workloads.WORKLOADS))
    p.add_argument("--no-int8-peak", action="store_true",
                   help="skip the library INT8 GEMM peak measured beside the workload")
    p.add_argument("--impl", default="tasq", choices=["tasq", "reference"])
    p.add_argument("--out-dtype", default="f16", choices=["f16", "bf16"])
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--profile-case", default=None,
                   help="workload:layer, run a few forwards of one layer (for ncu captures) and exit")
    p.add_argument("--launches", type=int, default=3)
    p.add_argument("--bits", type=int, default=None,
                   help="profile case: bit width 1..8, or 0 for the NVFP4 step (default: 5)")
    p.add_argument("--sweep-bits", default=None,
                   help="workload:layer, time one layer's prologue and GEMM at every bit width and exit")
    p.add_argument("--reps", type=int, default=20)
    p.add_argument("--gemm-mode", type=int, default=0, choices=[0, 1, 2],
                   help="GEMM kernel: 0 automatic, 1 one CTA per tile, 2 CTA pairs")
    p.add_argument("--mask-mode", type=int, default=0, choices=[0, 1, 2],
                   help="LSB mask: 0 in flight in the GEMM's weight feed (TMA at 8 bits), 1 in flight at every "
                        "width, 2 once ahead in the prologue launch into a masked copy")
    p.add_argument("--bitplanes", default=None,
                   help="workload:layer -- time the bit-plane formulation against the masked dense GEMM")
    p.add_argument("--nvfp4", action="store_true",
                   help="with --gemm-shape: time the block-scaled NVFP4 GEMM instead of the INT8 one; "
                        "with --sweep-bits: add an NVFP4 step (reported as width 0)")
    p.add_argument("--dmpq-shape", default=None,
                   help="M,D: time the on-device DMPQ predictor alone on one block input and output [M, D]")
    p.add_argument("--gemm-shape", default=None,
                   help="M,N,K: time the GEMM alone on given codes (one JSON line) and exit")
    p.add_argument("--graph", action="store_true",
                   help="capture each schedule step's launches in a CUDA graph and time graph replays")
    p.add_argument("--prologue-mode", type=int, default=0, choices=[0, 1, 2, 3],
                   help="prologue kernel: 0 automatic, 1 direct loads (32 channels a thread), 2 bulk-fed ring "
                        "where it fits, 3 direct loads with 64 channels a thread")
    return p.parse_args(argv)


def build_library():
    """Compile libtasq.so if stale and return the imported package. The build script is loaded
    by its path: importing the package first would load the library it is about to build."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_tasq_build", os.path.join(ROOT, "timestep_adaptive_bit_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import timestep_adaptive_bit_b200
    return timestep_adaptive_bit_b200


# ------------------------------------------------------------------------------ peaks, clocks
GEMM_SOURCES = ("masked_gemm.cu", "masked_gemm_pair.cu", "gemm_common.cuh", "ptx.cuh")


def profiled_traffic(workload: str):
    """DRAM bytes per GEMM launch from the committed ncu summary of this workload's step, if the
    GEMM kernel sources are still the ones the counters were taken on (else None)."""
    import hashlib
    import re
    path = os.path.join(ROOT, "profiles", f"launches_{workload}_step.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_t = re.search(r"traffic_bytes_per_launch:\s*(\d+)", text)
    m_h = re.search(r"kernel_sources_sha256:\s*([0-9a-f]{64})", text)
    if not (m_t and m_h):
        return None
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        with open(os.path.join(ROOT, "timestep_adaptive_bit_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return int(m_t.group(1)) if h.hexdigest() == m_h.group(1) else None


def max_over_ranks(value: float, dist, device) -> float:
    """Largest `value` over the ranks of the process group (the value itself without one)."""
    if dist is None:
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def int8_library_peak(torch, device, sustain_s: float = 4.0, n: int = 8192):
    """The tensor pipe's INT8 rate as a library reaches it on this GPU: torch._int_mm (cuBLASLt,
    INT8 x INT8 -> INT32) at n^3, the best of 10 launches (burst) and the mean over about
    sustain_s seconds of back-to-back launches (sustained, clocks sampled), the way the driver
    measured its BF16 figures. 2 n^3 ops per launch."""
    try:
        g = torch.Generator(device=device)
        g.manual_seed(0)
        a = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=device, generator=g)
        b = torch.randint(-127, 128, (n, n), dtype=torch.int8, device=device, generator=g).t()
        for _ in range(3):
            torch._int_mm(a, b)
        torch.cuda.synchronize()
        best = None
        for _ in range(10):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._int_mm(a, b)
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            best = ms if best is None else min(best, ms)
        sampler = ClockSampler(device.index or 0)
        sampler.start()
        reps = max(1, int(sustain_s / (best / 1e3)))
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            torch._int_mm(a, b)
        e1.record()
        torch.cuda.synchronize()
        clocks = sampler.stop()
        sust_ms = e0.elapsed_time(e1) / reps
        ops = 2.0 * n ** 3
        return {"burst_tops": ops / (best / 1e3) / 1e12, "sustained_tops": ops / (sust_ms / 1e3) / 1e12,
                "shape": [n, n, n], "library": "torch._int_mm (cuBLASLt INT8 -> INT32)",
                "sustained_launches": reps, "sustained_clocks": clocks,
                "datasheet_dense_tops": 4500.0}
    except Exception as e:   # a library without an INT8 path here: report why, keep the bench line
        return {"error": f"{type(e).__name__}: {str(e)[:200]}"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.tmp = None

    def start(self):
        try:
            self.tmp = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.tmp.flush()
        self.tmp.seek(0)
        rows = [r for r in csv.reader(io.StringIO(self.tmp.read())) if len(r) >= 9]
        self.tmp.close()
        os.unlink(self.tmp.name)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
            except ValueError:
                continue
            for name, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------------ CPU oracle leg
def oracle_sample(wl, rows: int, seed: int = 0):
    """Inputs of one block's linears for `rows` token rows, with each layer's bits at step 0."""
    data = []
    sched = workloads.schedule(wl)
    for j, (_, K, N) in enumerate(wl.block_layers):
        x = workloads.activations(wl, j, M=rows, seed=seed)
        w, s_w = workloads.weights(wl, j)
        data.append((x, w, s_w, int(sched[j, 0]), K, N))
    return data


def run_oracle_sample(wl, data):
    import oracle
    ops = 0.0
    for x, w, s_w, bits, K, N in data:
        if bits == 0:
            oracle.nvfp4_linear(x, w, s_w, wl.hadamard_n)
        else:
            oracle.masked_linear(x, w, s_w, bits, wl.hadamard_n)
        ops += 2.0 * x.shape[0] * N * K
    return ops


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        n = [i.get("num_threads", 1) for i in info if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def cpu_baseline(wl, budget_s: float = 12.0, rows: int = 256):
    data = oracle_sample(wl, rows)
    t0 = time.perf_counter()
    ops, reps = 0.0, 0
    while True:
        ops += run_oracle_sample(wl, data)
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": ops / dt / 1e12, "unit": "TOPS", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{reps} x one block ({len(wl.block_layers)} linears) of '{wl.name}' on {rows} token rows, "
                      f"step-0 bits; {dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    wl = workloads.WORKLOADS[args.workload]
    rows = 64
    data = oracle_sample(wl, rows)
    for _ in range(args.warmup):
        run_oracle_sample(wl, data)
    t0 = time.perf_counter()
    ops = 0.0
    for _ in range(args.steps):
        ops += run_oracle_sample(wl, data)
    dt = time.perf_counter() - t0
    value = ops / dt / 1e12
    sample = (f"each step: one block ({len(wl.block_layers)} linears) of '{wl.name}' on {rows} of its "
              f"{wl.tokens} token rows, step-0 bits")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / max(args.steps, 1) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "tokens": wl.tokens, "blocks": wl.blocks, "hadamard_n": wl.hadamard_n,
                   "sample_rows": rows},
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": blas_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------ GPU leg
def setup_workload(T, torch, wl, device, out_dtype, gemm_mode=0, mask_mode=0, prologue_mode=0):
    """Context with every layer of the workload, one activation buffer per (block, layer),
    one output buffer per distinct N. Weights and activations drawn on the device."""
    L = wl.num_layers
    layers, keep = [], []
    for l in range(L):
        _, K, N = wl.layer_shape(l)
        w, s_w = workloads.weights_torch(wl, l, device)
        keep.append((w, s_w))
        layers.append((N, K, w, s_w))
    stream = torch.cuda.current_stream()
    ctx = T.tasq_linear_create(layers, wl.steps, wl.hadamard_n, wl.tokens,
                               T.TASQ_OUT_F16 if out_dtype == "f16" else T.TASQ_OUT_BF16, stream)
    torch.cuda.synchronize()
    del keep, layers
    T.tasq_debug_set_gemm_mode(ctx, gemm_mode)
    T.tasq_debug_set_mask_mode(ctx, mask_mode)
    T.tasq_debug_set_prologue_mode(ctx, prologue_mode)
    T.tasq_set_schedule(ctx, workloads.schedule(wl), stream)
    xs = [workloads.activations_torch(wl, l, device) for l in range(L)]
    tdt = torch.float16 if out_dtype == "f16" else torch.bfloat16
    ys = {}
    for _, _, N in wl.block_layers:
        if N not in ys:
            ys[N] = torch.empty((wl.tokens, N), dtype=tdt, device=device)
    torch.cuda.synchronize()
    return ctx, xs, ys


def time_dmpq(T, torch, ctx, wl, xs, ys, stream, reps: int = 100):
    """CUDA-event time of tasq_dmpq_update on the block's first input and last output (same
    width). It reads both tensors once: algorithmic bytes 2 * M * D * 2."""
    D_in = wl.block_layers[0][1]
    D_out = wl.block_layers[-1][2]
    if D_in != D_out or D_in % 8 != 0:
        return None
    M = wl.tokens
    x_in, x_out = xs[0], ys[D_out]
    g = torch.zeros((1,), dtype=torch.float64, device=x_in.device)
    layers = list(range(len(wl.block_layers)))
    for _ in range(3):
        T.tasq_dmpq_update(ctx, x_in, D_in, x_out, D_out, M, D_in, layers, 0, 0.05, 8, 4, g, stream)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(reps):
        T.tasq_dmpq_update(ctx, x_in, D_in, x_out, D_out, M, D_in, layers, 0, 0.05, 8, 4, g, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    us = 1e3 * e0.elapsed_time(e1) / reps
    return {"us": us, "gbs": 4.0 * M * D_in / (us * 1e-6) / 1e9, "shape": [M, D_in], "calls": reps,
            "gamma": float(g.item())}


# threshold of the on-device predictor of dmpq_online workloads, set once per run
DMPQ_TAU = {}


def dmpq_block(T, ctx, wl, xs, b, step, stream, gamma_out=None):
    """The predictor for block b at `step`: its relative L1 change between its input and the next
    block's input (the last block: its own input against the first block's) picks INT8 (8 bits)
    or NVFP4 for all its linears, on the device."""
    per = len(wl.block_layers)
    K = wl.block_layers[0][1]
    x_in = xs[b * per]
    x_out = xs[((b + 1) % wl.blocks) * per]
    T.tasq_dmpq_update(ctx, x_in, K, x_out, K, wl.tokens, K, [b * per + j for j in range(per)], step,
                       DMPQ_TAU.get(wl.name, 0.0), 8, T.TASQ_NVFP4, gamma_out, stream)


def run_step(T, ctx, wl, xs, ys, step, stream):
    """Every linear of every block once. Linears that read the same input (q, k, v of SDXL) run
    as one group: one prologue, one GEMM each. dmpq_online workloads run the predictor before
    each block."""
    M = wl.tokens
    per = len(wl.block_layers)
    plan = wl.forward_plan()
    for b in range(wl.blocks):
        if wl.dmpq_online:
            dmpq_block(T, ctx, wl, xs, b, step, stream)
        for group in plan:
            l0 = b * per + group[0]
            _, K, N = wl.block_layers[group[0]]
            if len(group) == 1:
                T.tasq_linear_forward(ctx, xs[l0], M, K, l0, step, ys[N], N, stream)
            else:
                Ns = [wl.block_layers[j][2] for j in group]
                T.tasq_linear_forward_group(ctx, xs[l0], M, K, [b * per + j for j in group], step,
                                            [ys[n] for n in Ns], Ns, stream)


def time_same_traffic_copies(torch, wl, xs, stream, steps: int = 5):
    """The prologue's yardstick at its own sizes: for every prologue launch of a step, one
    device-to-device copy that moves the same DRAM traffic (half read from that launch's input
    tensor, half written), each bracketed by CUDA events the way the per-kernel trace brackets a
    prologue. Returns the copies' GB/s: summed traffic over summed event time."""
    M = wl.tokens
    per = len(wl.block_layers)
    plan = wl.forward_plan()
    sizes = {}
    for group in plan:
        K = wl.block_layers[group[0]][1]
        traffic = 2 * M * K + M * wl.kp(K) + 4 * M
        sizes[group[0]] = (traffic, (traffic // 2) // 16 * 16)
    dst = torch.empty((max(nb for _, nb in sizes.values()),), dtype=torch.uint8, device=xs[0].device)
    pairs = []
    with torch.cuda.stream(stream):
        for rep in range(steps + 1):
            for b in range(wl.blocks):
                for group in plan:
                    traffic, nb = sizes[group[0]]
                    src = xs[b * per + group[0]].view(torch.uint8).reshape(-1)[:nb]
                    if rep == 0:   # warm-up pass
                        dst[:nb].copy_(src, non_blocking=True)
                        continue
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    dst[:nb].copy_(src, non_blocking=True)
                    e1.record(stream)
                    pairs.append((traffic, e0, e1))
    torch.cuda.synchronize()
    total_bytes = sum(t for t, _, _ in pairs)
    total_ms = sum(e0.elapsed_time(e1) for _, e0, e1 in pairs)
    return total_bytes / (total_ms / 1e3) / 1e9 if total_ms > 0 else None


def run_step_io(T, ctx, wl, xs, ys, step, stream, x_first, y_last):
    """run_step with the step's first input read from x_first and its final output (the last
    linear of the last block) written to y_last: the buffers the end-to-end loop copies."""
    M = wl.tokens
    per = len(wl.block_layers)
    plan = wl.forward_plan()
    for b in range(wl.blocks):
        if wl.dmpq_online:
            dmpq_block(T, ctx, wl, xs, b, step, stream)
        for group in plan:
            l0 = b * per + group[0]
            _, K, N = wl.block_layers[group[0]]
            x = x_first if l0 == 0 else xs[l0]
            if len(group) == 1:
                last = b == wl.blocks - 1 and group[0] == per - 1
                T.tasq_linear_forward(ctx, x, M, K, l0, step, y_last if last else ys[N], N, stream)
            else:
                Ns = [wl.block_layers[j][2] for j in group]
                T.tasq_linear_forward_group(ctx, x, M, K, [b * per + j for j in group], step,
                                            [ys[n] for n in Ns], Ns, stream)


def launches_per_step(wl) -> int:
    """Kernels one step launches: a prologue per input, a GEMM per linear; with the on-device
    predictor, one predictor launch per block and both formats' prologue and GEMM per linear
    (the two of the format not chosen return at once)."""
    if wl.dmpq_online:
        return wl.blocks * (1 + 4 * len(wl.block_layers))
    return wl.blocks * (len(wl.forward_plan()) + len(wl.block_layers))


def profile_case(args):
    import torch
    import timestep_adaptive_bit_b200 as T
    name, _, lname = args.profile_case.partition(":")
    wl = workloads.WORKLOADS[name]
    j = [n for n, _, _ in wl.block_layers].index(lname or wl.block_layers[0][0])
    _, K, N = wl.layer_shape(j)
    dev = torch.device("cuda:0")
    w, s_w = workloads.weights_torch(wl, j, dev)
    s = torch.cuda.current_stream()
    ctx = T.tasq_linear_create([(N, K, w, s_w)], 1, wl.hadamard_n, wl.tokens, T.TASQ_OUT_F16, s)
    T.tasq_debug_set_gemm_mode(ctx, args.gemm_mode)
    T.tasq_debug_set_mask_mode(ctx, args.mask_mode)
    T.tasq_debug_set_prologue_mode(ctx, args.prologue_mode)
    bits = 5 if args.bits is None else args.bits
    T.tasq_set_schedule(ctx, np.array([[bits]], np.uint8), s)
    x = workloads.activations_torch(wl, j, dev)
    y = torch.empty((wl.tokens, N), dtype=torch.float16, device=dev)
    for _ in range(args.launches):
        T.tasq_linear_forward(ctx, x, wl.tokens, K, 0, 0, y, N, s)
    torch.cuda.synchronize()
    st = T.tasq_get_device_status(ctx)
    print(json.dumps({"profile_case": args.profile_case, "M": wl.tokens, "K": K, "N": N, "bits": bits,
                      "launches": args.launches, "device_status": st}))
    return 0 if st == 0 else 1


def gemm_shape(args):
    """CUDA-event time of the masked GEMM alone (tasq_debug_gemm on given codes) at one shape,
    back to back, for kernel-tuning experiments."""
    import torch
    import timestep_adaptive_bit_b200 as T
    M, N, K = (int(v) for v in args.gemm_shape.split(","))
    dev = torch.device("cuda:0")
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    w = torch.randint(-127, 128, (N, K), dtype=torch.int8, device=dev, generator=g)
    s_w = torch.rand((N,), device=dev, generator=g) * 0.01 + 0.001
    q = torch.randint(-127, 128, (M, K), dtype=torch.int8, device=dev, generator=g)
    s_x = torch.rand((M,), device=dev, generator=g) + 0.5
    y = torch.empty((M, N), dtype=torch.float16, device=dev)
    s = torch.cuda.current_stream()
    ctx = T.tasq_linear_create([(N, K, w, s_w)], 1, 64, M, T.TASQ_OUT_F16, s)
    T.tasq_debug_set_gemm_mode(ctx, args.gemm_mode)
    if args.nvfp4:
        # random E2M1 code bytes and finite UE4M3 block scales (0x30..0x3F: 0.5 .. 1.875)
        codes = torch.randint(0, 256, (M, K // 2), dtype=torch.uint8, device=dev, generator=g)
        sf = torch.randint(0x30, 0x40, (T.tasq_nvfp4_scale_bytes(M, K),), dtype=torch.uint8, device=dev,
                           generator=g)

        def call():
            T.tasq_debug_gemm_nvfp4(ctx, codes, sf, s_x, M, 0, y, N, T.TASQ_OUT_F16, s)
    else:
        def call():
            T.tasq_debug_gemm(ctx, q, s_x, M, 0, 0, y, N, T.TASQ_OUT_F16, s)
    for _ in range(3):
        call()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(args.reps):
        call()
    e1.record(s)
    torch.cuda.synchronize()
    us = 1e3 * e0.elapsed_time(e1) / args.reps
    peaks, _ = load_peaks()
    tops = 2.0 * M * N * K / (us * 1e-6) / 1e12
    # the NVFP4 hook converts the layer's weights (one prologue launch) before each GEMM
    print(json.dumps({"gemm_shape": [M, N, K], "nvfp4": bool(args.nvfp4), "gemm_mode": args.gemm_mode, "us": us,
                      "includes_weight_conversion": bool(args.nvfp4), "tops": tops,
                      "frac_int8_burst": tops / (peaks["bf16_tflops"] * INT8_OVER_BF16),
                      "device_status": T.tasq_get_device_status(ctx)}), flush=True)
    return 0


def dmpq_shape(args):
    """CUDA-event time of tasq_dmpq_update alone on a synthetic block input and output [M, D]
    (FP16, the output a small perturbation of the input), back to back."""
    import torch
    import timestep_adaptive_bit_b200 as T
    M, D = (int(v) for v in args.dmpq_shape.split(","))
    dev = torch.device("cuda:0")
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    x_in = torch.randn((M, D), device=dev, generator=g).to(torch.float16)
    x_out = (x_in.float() + 0.05 * torch.randn((M, D), device=dev, generator=g)).to(torch.float16)
    s = torch.cuda.current_stream()
    w = torch.zeros((64, D), dtype=torch.int8, device=dev)
    ctx = T.tasq_linear_create([(64, D, w, torch.ones(64, device=dev))], 1, 64, 16, T.TASQ_OUT_F16, s)
    gamma = torch.zeros((1,), dtype=torch.float64, device=dev)
    for _ in range(3):
        T.tasq_dmpq_update(ctx, x_in, D, x_out, D, M, D, [0], 0, 0.05, 8, 4, gamma, s)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(args.reps):
        T.tasq_dmpq_update(ctx, x_in, D, x_out, D, M, D, [0], 0, 0.05, 8, 4, gamma, s)
    e1.record(s)
    torch.cuda.synchronize()
    us = 1e3 * e0.elapsed_time(e1) / args.reps
    peaks, _ = load_peaks()
    gbs = 4.0 * M * D / (us * 1e-6) / 1e9
    print(json.dumps({"dmpq_shape": [M, D], "us": us, "gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
                      "gamma": float(gamma.item()), "device_status": T.tasq_get_device_status(ctx)}), flush=True)
    return 0


def bitplanes(args):
    """The bit-plane formulation measured (TASQ's Temporal-Precision Engine streams only the kept
    weight bit planes, TASQ technical summary section 2). On B200 the only integer tensor-core
    MMA is kind::i8, so a plane P_i of the weights (entries 0 or 1, the sign plane 0 or -1) costs
    one INT8 GEMM, and b kept planes cost b of them (plus the sum of the partial products). This
    times, at one layer's full shape, the masked dense GEMM at several widths and the same GEMM on
    a single bit plane, all on identical activation codes."""
    import torch
    import timestep_adaptive_bit_b200 as T
    name, _, lname = args.bitplanes.partition(":")
    wl = workloads.WORKLOADS[name]
    j = [n for n, _, _ in wl.block_layers].index(lname or wl.block_layers[0][0])
    _, K, N = wl.layer_shape(j)
    M = wl.tokens
    dev = torch.device("cuda:0")
    s = torch.cuda.current_stream()
    w, s_w = workloads.weights_torch(wl, j, dev)
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    Kp = w.shape[1]
    q = torch.randint(-127, 128, (M, Kp), dtype=torch.int8, device=dev, generator=g)
    s_x = torch.rand((M,), device=dev, generator=g) + 0.5
    y = torch.empty((M, N), dtype=torch.float16, device=dev)

    def timed(ctx, step):
        for _ in range(3):
            T.tasq_debug_gemm(ctx, q, s_x, M, 0, step, y, N, T.TASQ_OUT_F16, s)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(args.reps):
            T.tasq_debug_gemm(ctx, q, s_x, M, 0, step, y, N, T.TASQ_OUT_F16, s)
        e1.record(s)
        torch.cuda.synchronize()
        assert T.tasq_get_device_status(ctx) == 0
        return 1e3 * e0.elapsed_time(e1) / args.reps

    widths = (8, 6, 4, 2, 1)
    ctx = T.tasq_linear_create([(N, K, w, s_w)], len(widths), wl.hadamard_n, M, T.TASQ_OUT_F16, s)
    T.tasq_set_schedule(ctx, np.array([widths], np.uint8), s)
    T.tasq_debug_set_mask_mode(ctx, 2)        # the weights masked once ahead, as in a forward
    dense = {b: timed(ctx, i) for i, b in enumerate(widths)}
    T.tasq_linear_destroy(ctx)
    planes = {}
    for name_p, plane in (("plane_3", ((w.to(torch.int16) >> 3) & 1).to(torch.int8)),
                          ("sign_plane", -((w.to(torch.int16) >> 7) & 1).to(torch.int8))):
        ctx = T.tasq_linear_create([(N, K, plane.contiguous(), s_w)], 1, wl.hadamard_n, M, T.TASQ_OUT_F16, s)
        planes[name_p] = timed(ctx, 0)
        T.tasq_linear_destroy(ctx)
    t_plane = max(planes.values())
    out = {"bitplanes": args.bitplanes, "M": M, "N": N, "K": K,
           "dense_masked_us": {str(b): round(t, 2) for b, t in dense.items()},
           "one_plane_us": {k: round(v, 2) for k, v in planes.items()},
           "bit_plane_gemm_us_lower_bound": {str(b): round(b * t_plane, 2) for b in widths},
           "note": "b kept planes = b INT8 GEMMs on 0/1 planes; the lower bound leaves out summing them"}
    print(json.dumps(out), flush=True)
    return 0


def sweep_bits(args):
    """Per-bit-width timing of one layer at full size (CUDA-event trace of each kernel)."""
    import torch
    import timestep_adaptive_bit_b200 as T
    name, _, lname = args.sweep_bits.partition(":")
    wl = workloads.WORKLOADS[name]
    j = [n for n, _, _ in wl.block_layers].index(lname or wl.block_layers[0][0])
    _, K, N = wl.layer_shape(j)
    M = wl.tokens
    dev = torch.device("cuda:0")
    w, s_w = workloads.weights_torch(wl, j, dev)
    s = torch.cuda.current_stream()
    # bit widths 8 .. 1, then (with --nvfp4) one NVFP4 step, reported under "0"
    widths = [8, 7, 6, 5, 4, 3, 2, 1] + ([0] if args.nvfp4 else [])
    ctx = T.tasq_linear_create([(N, K, w, s_w)], len(widths), wl.hadamard_n, M, T.TASQ_OUT_F16, s)
    T.tasq_debug_set_gemm_mode(ctx, args.gemm_mode)
    T.tasq_debug_set_mask_mode(ctx, args.mask_mode)
    T.tasq_debug_set_prologue_mode(ctx, args.prologue_mode)
    T.tasq_set_schedule(ctx, np.array([widths], np.uint8), s)
    # several input buffers so consecutive launches do not find their activations in L2
    nbuf = max(2, int(math.ceil(3 * 126e6 / (M * K * 2))))
    xs = [workloads.activations_torch(wl, j, dev, seed=b) for b in range(nbuf)]
    y = torch.empty((M, N), dtype=torch.float16, device=dev)
    peaks, peak_kind = load_peaks()
    out = {"sweep": f"{name}:{wl.block_layers[j][0]}", "M": M, "K": K, "N": N, "reps": args.reps,
           "gemm_mode": args.gemm_mode, "mask_mode": args.mask_mode, "prologue_mode": args.prologue_mode,
           "bits": {}}
    for step, width in enumerate(widths):
        for r in range(3):
            T.tasq_linear_forward(ctx, xs[r % nbuf], M, K, 0, step, y, N, s)
        torch.cuda.synchronize()
        T.tasq_trace_enable(ctx, args.reps)
        for r in range(args.reps):
            T.tasq_linear_forward(ctx, xs[r % nbuf], M, K, 0, step, y, N, s)
        tr = T.tasq_trace_read(ctx)
        g_tops = tr["gemm_ops"] / (tr["gemm_ms"] / 1e3) / 1e12
        p_gbs = tr["prologue_bytes"] / (tr["prologue_ms"] / 1e3) / 1e9
        out["bits"][width] = {"gemm_us": 1e3 * tr["gemm_ms"] / args.reps, "gemm_tops": g_tops,
                                 "gemm_frac_int8_burst": g_tops / (peaks["bf16_tflops"] * INT8_OVER_BF16),
                                 "prologue_us": 1e3 * tr["prologue_ms"] / args.reps, "prologue_gbs": p_gbs,
                                 "prologue_frac_hbm": p_gbs / peaks["hbm_gbs"],
                                 "forward_us": 1e3 * (tr["prologue_ms"] + tr["gemm_ms"]) / args.reps}
    out["device_status"] = T.tasq_get_device_status(ctx)
    print(json.dumps(out), flush=True)
    return 0 if out["device_status"] == 0 else 1


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)

    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    T = build_library()

    if args.profile_case:
        return profile_case(args)
    if args.sweep_bits:
        return sweep_bits(args)
    if args.gemm_shape:
        return gemm_shape(args)
    if args.dmpq_shape:
        return dmpq_shape(args)
    if args.bitplanes:
        return bitplanes(args)

    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)

    wl = workloads.WORKLOADS[args.workload]
    ctx, xs, ys = setup_workload(T, torch, wl, device, args.out_dtype, args.gemm_mode, args.mask_mode,
                                 args.prologue_mode)
    stream = torch.cuda.current_stream()
    L = wl.num_layers
    if wl.dmpq_online:
        # the predictor's threshold: the median of the blocks' relative L1 change, measured once
        gam = torch.zeros((wl.blocks,), dtype=torch.float64, device=device)
        for b in range(wl.blocks):
            dmpq_block(T, ctx, wl, xs, b, 0, stream, gam[b:b + 1])
        torch.cuda.synchronize()
        DMPQ_TAU[wl.name] = float(gam.median().item())

    for i in range(args.warmup):
        run_step(T, ctx, wl, xs, ys, i % wl.steps, stream)
    torch.cuda.synchronize()
    graphs = {}
    if args.graph:
        # one graph per schedule step: the (layer, step) table indices are kernel arguments
        for t in sorted({i % wl.steps for i in range(args.steps)}):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                run_step(T, ctx, wl, xs, ys, t, torch.cuda.current_stream())
            graphs[t] = g
        for i in range(args.warmup):
            graphs[i % wl.steps].replay() if (i % wl.steps) in graphs else None
        torch.cuda.synchronize()

    def timed_step(i):
        if graphs:
            graphs[i % wl.steps].replay()
        else:
            run_step(T, ctx, wl, xs, ys, i % wl.steps, stream)

    sampler = ClockSampler(local_rank)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.2)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        timed_step(i)
    t1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    if dist is not None:
        dist.barrier()
    ms_max = max_over_ranks(t0.elapsed_time(t1), dist, device)

    # ---- per-kernel durations: a separate pass of the same steps with CUDA events around every
    # kernel. Events between the kernels break their programmatic-launch overlap (about 18 % on
    # the PixArt-Sigma step), so the headline above is timed without them.
    # whole cycles of the schedule where the timed steps cover one, so that every step's widths
    # weigh as much as in the timed steps
    trace_steps = max(1, min(args.steps, 40))
    if args.steps >= wl.steps:
        trace_steps = max(wl.steps, (trace_steps // wl.steps) * wl.steps)
    T.tasq_trace_enable(ctx, trace_steps * L)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    q0 = torch.cuda.Event(enable_timing=True)
    q1 = torch.cuda.Event(enable_timing=True)
    q0.record(stream)
    for i in range(trace_steps):
        run_step(T, ctx, wl, xs, ys, i % wl.steps, stream)
    q1.record(stream)
    torch.cuda.synchronize()
    traced_ms = q0.elapsed_time(q1)
    trace = T.tasq_trace_read(ctx)
    T.tasq_trace_enable(ctx, 0)
    status = T.tasq_get_device_status(ctx)
    # the widths the on-device predictor chose (the last visit of every step)
    device_table = T.tasq_get_schedule(ctx) if wl.dmpq_online else None

    # ---- end to end through the public API: pinned host input in, host result out, per step
    e2e = None
    if not args.no_e2e:
        first_K = wl.block_layers[0][1]
        last_N = wl.block_layers[-1][2]
        x_host = torch.empty((wl.tokens, first_K), dtype=torch.float16, pin_memory=True)
        x_host.copy_(xs[0].cpu())
        y_host = torch.empty((wl.tokens, last_N), dtype=ys[last_N].dtype, pin_memory=True)
        # the same steps, in the same order, as the timed loop (the schedule's widths vary by step)
        e_steps = max(1, args.steps)
        # every step copies its input in from pinned host memory and its result out; the copies run
        # on their own stream into double buffers, so step i's result leaves and step i + 1's input
        # arrives while the GPU computes
        x_dev = [torch.empty_like(xs[0]), torch.empty_like(xs[0])]
        y_dev = [torch.empty_like(ys[last_N]), torch.empty_like(ys[last_N])]
        copy_stream = torch.cuda.Stream(device=device)
        ev_in = [torch.cuda.Event(), torch.cuda.Event()]
        ev_done = [torch.cuda.Event(), torch.cuda.Event()]
        ev_out = torch.cuda.Event()
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        copy_stream.wait_event(e0)
        for i in range(min(2, e_steps)):
            with torch.cuda.stream(copy_stream):
                x_dev[i].copy_(x_host, non_blocking=True)
            ev_in[i].record(copy_stream)
        for i in range(e_steps):
            b = i % 2
            stream.wait_event(ev_in[b])
            run_step_io(T, ctx, wl, xs, ys, i % wl.steps, stream, x_dev[b], y_dev[b])
            ev_done[b].record(stream)
            copy_stream.wait_event(ev_done[b])
            with torch.cuda.stream(copy_stream):
                y_host.copy_(y_dev[b], non_blocking=True)
                if i + 2 < e_steps:
                    x_dev[b].copy_(x_host, non_blocking=True)
            if i + 2 < e_steps:
                ev_in[b].record(copy_stream)
        ev_out.record(copy_stream)
        stream.wait_event(ev_out)
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), dist, device)
        e2e = {"value": world * e_steps * wl.gemm_ops_per_step() / (e_ms / 1e3) / 1e12, "unit": "TOPS",
               "h2d_bytes_per_step": int(x_host.numel() * x_host.element_size()),
               "d2h_bytes_per_step": int(y_host.numel() * y_host.element_size()),
               "steps": e_steps, "ms_per_step": e_ms / e_steps,
               "copies": "pinned host->device input and device->host result of every step, on a second stream "
                         "into double buffers, overlapping the neighbouring steps' compute"}

    # ---- next row: the on-device DMPQ predictor on the block's first input and last output
    dmpq = time_dmpq(T, torch, ctx, wl, xs, ys, stream)
    copy_gbs = time_same_traffic_copies(torch, wl, xs, stream)

    peaks, peak_kind = load_peaks()
    int8_burst = peaks["bf16_tflops"] * INT8_OVER_BF16
    int8_sust = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * INT8_OVER_BF16
    total_ops = world * args.steps * wl.gemm_ops_per_step()
    value = total_ops / (ms_max / 1e3) / 1e12
    ms_per_step = ms_max / args.steps
    gemm_tops = trace["gemm_ops"] / (trace["gemm_ms"] / 1e3) / 1e12 if trace["gemm_ms"] > 0 else None
    # the prologue's algorithmic bytes: activations only, M (2 K + Kp + 4) per launch; a weight pass
    # (mask mode 2, or the NVFP4 steps' weight conversion) is reported apart
    pro_gbs = trace["prologue_bytes"] / (trace["prologue_ms"] / 1e3) / 1e9 if trace["prologue_ms"] > 0 else None
    int8_lib = None
    if not args.no_int8_peak:
        int8_lib = int8_library_peak(torch, device)
    # the kernel that runs most of the step's GEMM work with the automatic choice
    big = max(wl.block_layers, key=lambda l: l[1] * l[2])
    dominant = ("masked_gemm_pair_kernel" if T.tasq_gemm_choice(wl.tokens, big[2], torch.cuda.get_device_properties(
        device).multi_processor_count) else "masked_gemm_kernel")

    if dist is not None:
        T.tasq_linear_destroy(ctx)
        dist.destroy_process_group()
    if rank != 0:
        return 0 if status == 0 else 1

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl)

    sched = device_table if device_table is not None else workloads.schedule(wl)
    used = sched[:, [i % wl.steps for i in range(args.steps)]].astype(np.float64)
    nvfp4 = used == 0
    # weight bits, an NVFP4 step counted as 4; BitOPs model: weight bits x activation bits against
    # 8 x 8, the NVFP4 step being W4A4
    mean_bits = float(np.mean(np.where(nvfp4, 4.0, used)))
    bitops_ratio = float(np.mean(np.where(nvfp4, 16.0, 8.0 * used) / 64.0))
    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8+nvfp4" if np.any(nvfp4) else "int8", "data": "synthetic",
        "config": {"workload": wl.name, "tokens": wl.tokens, "blocks": wl.blocks, "schedule_steps": wl.steps,
                   "hadamard_n": wl.hadamard_n,
                   "linears": [f"{n}:{K}->{N}" for n, K, N in wl.block_layers],
                   "out_dtype": args.out_dtype, "parallelism": f"replicas{world}",
                   "launch": "cuda_graph_per_step" if args.graph else "stream",
                   "l2": "inputs larger than L2: each step reads its own activations for every (block, linear) "
                         f"({sum(x.numel() * 2 for x in xs) / 1e9:.2f} GB) and every layer's weights once"},
        "tokens_per_s_per_step": wl.tokens / (ms_per_step / 1e3) * world,
        "pct_int8_peak": 100.0 * value / (int8_burst * world),
        "mean_bits": mean_bits,
        "nvfp4_fraction": float(np.mean(nvfp4)),
        "bitops_saved_modelled": 1.0 - bitops_ratio,
        "roofline": {"bound": "tensor", "achieved": gemm_tops, "peak": int8_burst, "unit": "TFLOP/s",
                     "frac": (gemm_tops / int8_burst) if gemm_tops else None,
                     "traffic": profiled_traffic(wl.name),
                     "traffic_source": f"profiles/launches_{wl.name}_step.md (null once the GEMM sources change)",
                     "kernel": dominant, "peak_kind": f"INT8 = 2 x {peak_kind} BF16 burst",
                     "frac_of_sustained": (gemm_tops / int8_sust) if gemm_tops else None,
                     "int8_library": int8_lib,
                     "frac_of_int8_library_burst": (gemm_tops / int8_lib["burst_tops"])
                     if (gemm_tops and int8_lib and "burst_tops" in int8_lib) else None,
                     "frac_of_int8_library_sustained": (gemm_tops / int8_lib["sustained_tops"])
                     if (gemm_tops and int8_lib and "sustained_tops" in int8_lib) else None,
                     "frac_of_datasheet_dense_int8": (gemm_tops / 4500.0) if gemm_tops else None},
        "prologue_roofline": {"bound": "hbm", "achieved": pro_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                              "frac": (pro_gbs / peaks["hbm_gbs"]) if pro_gbs else None,
                              "frac_of_8000": (pro_gbs / 8000.0) if pro_gbs else None,
                              "bytes_per_step": trace["prologue_bytes"] / trace_steps,
                              "bytes": "activations only: M (2 K + Kp + 4) per prologue launch",
                              "weight_pass_bytes_per_step": trace["weight_pass_bytes"] / trace_steps,
                              "same_traffic_copy_gbs": copy_gbs,
                              "frac_of_same_traffic_copy": (pro_gbs / copy_gbs) if (pro_gbs and copy_gbs) else None},
        "gemm_share_of_step": trace["gemm_ms"] / max(traced_ms, 1e-9) if trace["gemm_ms"] else None,
        "kernel_timing": f"per-kernel CUDA events in a separate pass of {trace_steps} steps "
                         f"({traced_ms / trace_steps:.3f} ms per step with the events); the timed steps run "
                         "without them",
        "clocks": clocks,
        "gpu_launches": args.steps * launches_per_step(wl),
        "device_status": status,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "dmpq_predictor": None if dmpq is None else {
            "bound": "hbm", "achieved": dmpq["gbs"], "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": dmpq["gbs"] / peaks["hbm_gbs"], "us_per_call": dmpq["us"], "shape": dmpq["shape"],
            "calls": dmpq["calls"], "gamma": dmpq["gamma"]},
    }
    print(json.dumps(line), flush=True)
    return 0 if status == 0 else 1


if __name__ == "__main__":
    sys.exit(main())
