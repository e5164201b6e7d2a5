#!/usr/bin/env python3
"""Throughput of the W4A16 group-128 linear layer on B200.

Default workload (one "step"): the decode matvec over the seven Qwen3-4B
projections (q 2560->4096, k/v 2560->1024, o 4096->2560, gate/up 2560->9728,
down 9728->2560) for each batch size M in {1, 2, 4, 8}: 28 calls of
w4a16_matmul on synthetic seeded inputs (x ~ N(0,1) BF16, W ~ N(0,0.02)
quantised to 4 bits per 128-group).

Metric: algorithmic bytes per second (GB/s) and FLOP/s, against the HBM
roofline.  Algorithmic bytes per call = N*K/2 (codes) + 4*N*K/128 (BF16 scale
and bias) + 2*M*K (x) + 2*M*N (y); FLOPs = 2*M*N*K.

Timing: the 28 calls of a step are captured once in a CUDA graph per weight
set; two weight sets of 215 MB each (every (M, projection) pair has its own
copy) alternate between steps, so the working set between two uses of the
same bytes is 430 MB, far above the 126 MB L2.  W >= 3 warm-up steps, then K
timed steps between CUDA events on the launching stream, with a barrier and a
device synchronise on both sides; the step time is the max over ranks.

Also reported: the oracle timed on the host cores (cpu_baseline), an
end-to-end figure through the Python/C ABI with host buffers (H2D of the
step's activations, 28 calls, D2H of the outputs), SM clocks sampled during
the timed region, and the roofline of the matvec kernel.

`--impl reference` times the CPU oracle on the same workload (a bounded
sample of each step's output columns) and prints the same line with
"impl": "reference".
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import w4a16_synth as synth  # noqa: E402

METRIC = "W4A16 matmul TFLOP/s & GB/s on 1 B200 vs roofline fraction (M=1..2048)"
DECODE_M = (1, 2, 4, 8)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# the nominal roofline the targets are stated against: 8 TB/s of HBM, 2.25 PFLOP/s dense BF16
NOMINAL_PEAKS = {"hbm_gbs": 8000.0, "bf16_tflops": 2250.0}
# the decode step's kernel (the row-block matvec serves all seven projections) and the
# committed ncu record of its DRAM traffic, valid while these sources are unchanged
DECODE_KERNEL = "w4a16::mvr::rows_kernel"
KERNEL_SOURCES = ("decode_w4a16_g128_b200/csrc/rows.cuh", "decode_w4a16_g128_b200/csrc/ptx.cuh",
                  "decode_w4a16_g128_b200/csrc/plain.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "rows_decode_traffic.txt")
GEMM_SOURCES = ("decode_w4a16_g128_b200/csrc/gemm.cuh", "decode_w4a16_g128_b200/csrc/ptx.cuh",
                "decode_w4a16_g128_b200/csrc/plain.cuh")
GEMM_TRAFFIC_FILE = os.path.join(ROOT, "profiles", "gemm_m2048_gate_traffic.txt")


def algo_bytes(M, N, K):
    return N * K // 2 + 4 * N * K // 128 + 2 * M * K + 2 * M * N


def decode_calls():
    return [(M, name, K, N) for M in DECODE_M for (name, K, N) in synth.QWEN3_4B_PROJECTIONS]


PREFILL_SETS = (
    ("prefill_m128", "M=128 over the seven Qwen3-4B projections (aligned tiles)",
     [(128, name, K, N, 0) for (name, K, N) in synth.QWEN3_4B_PROJECTIONS]),
    ("partial_long_k", "M in {129,509} x N in {1000,4096} x K in {2560,9728}, x with 1% outliers x20",
     [(M, f"M{M}_N{N}_K{K}", K, N, 0) for M in (129, 509) for N in (1000, 4096) for K in (2560, 9728)]),
    ("prefill_m2048", "M=2048 over the seven Qwen3-4B projections",
     [(2048, name, K, N, 0) for (name, K, N) in synth.QWEN3_4B_PROJECTIONS]),
    ("lm_head_last_row", "lm_head 2560->151936 on the last of 2048 rows (logits_to_keep=1)",
     [(2048, "lm_head", 2560, 151936, 1)]),
    ("lm_head_all_rows", "lm_head 2560->151936 on all 2048 rows",
     [(2048, "lm_head", 2560, 151936, 0)]),
)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS, source="fallback")


def kernel_hash(sources=KERNEL_SOURCES):
    h = hashlib.sha256()
    for rel in sources:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(path=TRAFFIC_FILE, sources=KERNEL_SOURCES):
    """Per-launch DRAM bytes from the committed ncu capture, if it matches this kernel."""
    try:
        with open(path) as f:
            d = dict(line.split(":", 1) for line in f if ":" in line and not line.startswith("#"))
        d = {k.strip(): v.strip() for k, v in d.items()}
        if d.get("kernel_sha") != kernel_hash(sources):
            return None
        return int(d["dram_bytes_per_launch"])
    except (OSError, ValueError, KeyError):
        return None


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples every 200 ms while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=5)
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in self.lines:
            f = [t.strip() for t in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- distributed

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_group(world, backend):
    import torch.distributed as dist
    from datetime import timedelta
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=timedelta(seconds=300))
    return dist


def max_over_ranks(value, world, device):
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---------------------------------------------------------------- workload

def make_host_inputs():
    """Seeded inputs of the decode step: one weight set per projection, one x per (M, projection)."""
    weights = {}
    for (name, K, N) in synth.QWEN3_4B_PROJECTIONS:
        rng = synth.shape_rng(0, N, K, seed=0)
        weights[name] = synth.make_weights(rng, N, K)
    xs = {}
    for (M, name, K, N) in decode_calls():
        xs[(M, name)] = synth.make_x(synth.shape_rng(M, N, K, seed=1), M, K)
    return weights, xs


def cpu_sample(weights, xs, frac):
    """The oracle over the first ceil(frac*N) output columns of every call of a step."""
    import oracle
    nbytes = 0
    t0 = time.perf_counter()
    for (M, name, K, N) in decode_calls():
        wq, s, b = weights[name]
        n = max(1, int(math.ceil(N * frac)))
        oracle.matmul(xs[(M, name)], wq[:n], s[:n], b[:n])
        nbytes += algo_bytes(M, n, K)
    return nbytes, time.perf_counter() - t0


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    import oracle
    weights, xs = make_host_inputs()
    frac = args.ref_fraction
    for _ in range(args.warmup):
        cpu_sample(weights, xs, frac)
    total_b, total_t = 0, 0.0
    for _ in range(args.steps):
        b, t = cpu_sample(weights, xs, frac)
        total_b += b
        total_t += t
    gbs = total_b / total_t / 1e9
    ms = total_t / args.steps * 1e3
    sample = (f"oracle on the first {frac:g} of the output columns of each of the 28 calls "
              f"(M in {{1,2,4,8}} x 7 projections) per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": workload_config(),
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": oracle.threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config():
    return {
        "workload": "decode matvec: M in {1,2,4,8} x Qwen3-4B projections q 2560->4096, k/v 2560->1024, "
                    "o 4096->2560, gate/up 2560->9728, down 9728->2560 (28 calls per step)",
        "group_size": 128, "bits": 4,
        "l2": "inputs larger than L2: two rotating weight sets of 215 MB (430 MB between reuses)",
        "timing": "CUDA graph of the 28 calls per step, CUDA events on the launching stream",
        "flags": "W4A16_FLAG_STATIC_WEIGHTS (weights streamed while the previous call finishes)",
    }


def run_ours(args, world, rank, local):
    import torch
    import decode_w4a16_g128_b200 as w4

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if args.mode == "profile" and args.case:
        return profile_case(args, device, torch.cuda.Stream(device))
    if world > 1:
        init_group(world, "nccl")
    pk = peaks()

    weights, xs = make_host_inputs()
    weights_cache = {(name, K, N): weights[name] for (name, K, N) in synth.QWEN3_4B_PROJECTIONS}
    calls = decode_calls()
    nsets = 2

    def dev_bf16(a):
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)

    base_w = {name: (torch.from_numpy(wq.view(np.int32)).to(device), dev_bf16(s), dev_bf16(b))
              for name, (wq, s, b) in weights.items()}
    sets = []
    for _ in range(nsets):
        entries = []
        for (M, name, K, N) in calls:
            wq, s, b = base_w[name]
            x = dev_bf16(xs[(M, name)])
            y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
            entries.append((x, wq.clone(), s.clone(), b.clone(), y))
        sets.append(entries)
    del base_w
    step_bytes = sum(algo_bytes(M, N, K) for (M, _, K, N) in calls)
    step_flops = sum(2 * M * N * K for (M, _, K, N) in calls)

    stream = torch.cuda.Stream(device)

    # weights are static across the step: let each call start streaming them while the
    # previous call finishes (programmatic dependent launch); x is read after it completes
    flags = w4.FLAG_STATIC_WEIGHTS

    def launch_set(entries):
        for (x, wq, s, b, y) in entries:
            w4.w4a16_matmul_ex(x, wq, s, b, y=y, flags=flags)

    # warm the workspace of the capture stream, then capture one graph per set
    with torch.cuda.stream(stream):
        for entries in sets:
            launch_set(entries)
    stream.synchronize()
    graphs = []
    for entries in sets:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            launch_set(entries)
        graphs.append(g)
    torch.cuda.synchronize()
    if w4.w4a16_device_status(stream) != w4.OK:
        raise RuntimeError("device status not ok after capture")

    if args.mode == "profile":
        # exactly two eager steps (56 launches) for ncu: skip 28, capture the next 28
        with torch.cuda.stream(stream):
            launch_set(sets[0])
            launch_set(sets[0])
        torch.cuda.synchronize()
        return 0

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            graphs[i % nsets].replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for i in range(args.steps):
            graphs[i % nsets].replay()
        end.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop()
    ms_total = start.elapsed_time(end)
    ms_total = max_over_ranks(ms_total, world, device)
    ms_step = ms_total / args.steps
    status = w4.w4a16_device_status(stream)
    if status != w4.OK:
        raise RuntimeError(f"device status {status} after the timed region")

    gbs = step_bytes * world / (ms_step * 1e-3) / 1e9
    tflops = step_flops * world / (ms_step * 1e-3) / 1e12
    launches = len(calls)
    achieved = step_bytes / (ms_step * 1e-3) / 1e9      # per GPU: bytes per launch / mean launch time
    traffic = recorded_traffic()

    # End to end through the C ABI with host buffers: one H2D copy of the step's activations
    # (all 28 x, packed in one pinned buffer), the 28 calls, one D2H copy of the 28 outputs.
    import ctypes
    x_off, y_off, xo, yo = [], [], 0, 0
    for (M, name, K, N) in calls:
        x_off.append(xo)
        y_off.append(yo)
        xo += M * K
        yo += M * N
    host_x = torch.empty(xo, dtype=torch.int16).pin_memory()
    for (M, name, K, N), off in zip(calls, x_off):
        host_x[off:off + M * K] = torch.from_numpy(xs[(M, name)].view(np.int16).reshape(-1))
    host_y = torch.empty(yo, dtype=torch.int16).pin_memory()
    dev_x = torch.empty(xo, dtype=torch.int16, device=device)
    dev_y = torch.empty(yo, dtype=torch.int16, device=device)
    h2d, d2h = host_x.numel() * 2, host_y.numel() * 2
    opt = w4.make_options(flags=flags)
    P = ctypes.c_void_p

    def c_args(entries):
        out = []
        for (M, name, K, N), (x, wq, s_, b_, y), xo_, yo_ in zip(calls, entries, x_off, y_off):
            out.append((P(dev_x.data_ptr() + 2 * xo_), P(wq.data_ptr()), P(s_.data_ptr()), P(b_.data_ptr()),
                        P(dev_y.data_ptr() + 2 * yo_), M, N, K))
        return out

    set_args = [c_args(entries) for entries in sets]
    fn = w4.lib.w4a16_matmul_ex
    sp = P(stream.cuda_stream)
    optp = ctypes.byref(opt)

    def e2e_step(args):
        dev_x.copy_(host_x, non_blocking=True)
        for a in args:
            rc = fn(*a, sp, optp)
            if rc:
                raise RuntimeError(f"w4a16_matmul_ex: {w4.status_string(rc)}")
        host_y.copy_(dev_y, non_blocking=True)

    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            e2e_step(set_args[i % nsets])
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(args.steps):
            e2e_step(set_args[i % nsets])
        e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device) / args.steps
    e2e_gbs = step_bytes * world / (e2e_ms * 1e-3) / 1e9
    del dev_x, dev_y

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        nb, t, reps = 0, 0.0, 0
        while t < args.cpu_seconds or reps == 0:   # whole decode steps until the time bound is reached
            b_, t_ = cpu_sample(weights, xs, 1.0)
            nb, t, reps = nb + b_, t + t_, reps + 1
        cores = oracle.threads()
        cpu = {"value": round(nb / t / 1e9, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": f"{reps} full decode steps (all 28 calls each, {t:.1f} s) through the C oracle, "
                         "OpenMP over outputs"}
        # the same oracle on one thread: an eighth of every call's output columns per step
        oracle.set_threads(1)
        try:
            nb1, t1, reps1 = 0, 0.0, 0
            while t1 < args.cpu_seconds or reps1 == 0:
                b_, t_ = cpu_sample(weights, xs, 0.125)
                nb1, t1, reps1 = nb1 + b_, t1 + t_, reps1 + 1
        finally:
            oracle.set_threads(cores)
        cpu["single_thread"] = {"value": round(nb1 / t1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                                "sample": f"{reps1} decode steps over the first eighth of every call's "
                                          f"output columns ({t1:.1f} s), one thread"}

    if args.detail and rank == 0:
        detail(args, sets[0], calls, stream, pk)

    prefill = None
    if not args.no_prefill:
        del sets, graphs
        torch.cuda.empty_cache()
        prefill = prefill_section(device, stream, pk, weights_cache)
    quant = None
    gate_up = None
    skinny = None
    if not args.no_quantize and rank == 0:
        torch.cuda.empty_cache()
        quant = quantize_section(device, stream, pk)
        gate_up = gate_up_section(device, stream, pk)
    if not args.no_prefill and rank == 0:
        skinny = skinny_section(device, stream, pk, weights_cache)
    nbits = None
    if not args.no_quantize and rank == 0:
        nbits = bits_section(device, stream, pk)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(gbs, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": workload_config(),
            "tflops": round(tflops, 3),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": pk["hbm_gbs"],
                         "unit": "GB/s", "frac": round(achieved / pk["hbm_gbs"], 4),
                         "frac_nominal": round(achieved / NOMINAL_PEAKS["hbm_gbs"], 4), "traffic": traffic,
                         "peak_source": pk["source"], "kernel": DECODE_KERNEL,
                         "algorithmic_bytes_per_launch": round(step_bytes / launches)},
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_gbs, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h},
            "gpu_launches": launches * args.steps,
            "clocks": clocks,
        }
        if prefill is not None:
            m2048 = prefill["prefill_m2048"]
            line["roofline_gemm"] = {
                "bound": "tensor", "achieved": m2048["tflops"], "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": m2048["frac"], "frac_nominal": m2048["frac_nominal"],
                "traffic": recorded_traffic(GEMM_TRAFFIC_FILE, GEMM_SOURCES),
                "traffic_launch": "gate, M=2048 (DRAM bytes of one launch; most of y is still in L2 when it ends)",
                "peak_source": pk["source"] + " (burst)",
                "kernel": "w4a16::gm::gemm_kernel", "workload": "M=2048, seven Qwen3-4B projections"}
            line["prefill"] = prefill
            line["prefill_calls_fields"] = ["M", "projection", "N", "K", "us", "fraction of the bound's measured peak"]
        if quant is not None:
            line["quantize"] = quant
        if gate_up is not None:
            line["gate_up"] = gate_up
        if skinny is not None:
            line["skinny"] = skinny
        if nbits is not None:
            line["bits"] = nbits
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def time_calls(make_copy, launch, n_copies, reps, stream):
    """Mean device time (us) of one call: a CUDA graph of `reps` back-to-back calls
    rotating over `n_copies` distinct input sets, replayed 3 times after a warm-up."""
    import torch
    copies = [make_copy(i) for i in range(n_copies)]
    with torch.cuda.stream(stream):
        for c in copies:
            launch(c)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(reps):
            launch(copies[i % n_copies])
    with torch.cuda.stream(stream):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(3):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (3 * reps)
    del g, copies
    return us


def prefill_section(device, stream, pk, weights_cache):
    """Time every M > 8 configuration (and the last-row vocabulary projection)."""
    import torch
    import decode_w4a16_g128_b200 as w4
    out = {}
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flop_peak = pk["bf16_tflops"]
    for key, desc, calls in PREFILL_SETS:
        rows, tot_flops, tot_us, tot_bytes = [], 0, 0.0, 0
        for (M, name, K, N, keep) in calls:
            if (name, K, N) not in weights_cache:
                weights_cache[(name, K, N)] = synth.make_weights(synth.shape_rng(0, N, K, seed=0), N, K)
            wq, sc, bi = weights_cache[(name, K, N)]
            outliers = key == "partial_long_k"
            x_host = synth.make_x(synth.shape_rng(M, N, K, seed=1), M, K, outliers=outliers)
            Mo = M if keep == 0 else keep
            wbytes = algo_bytes(M, N, K)
            n_copies = int(max(2, min(16, math.ceil(2.2 * l2 / wbytes))))
            base = (torch.from_numpy(x_host.view(np.int16)).to(device).view(torch.bfloat16),
                    torch.from_numpy(wq.view(np.int32)).to(device),
                    torch.from_numpy(sc.view(np.int16)).to(device).view(torch.bfloat16),
                    torch.from_numpy(bi.view(np.int16)).to(device).view(torch.bfloat16))

            def make_copy(i, base=base, Mo=Mo, N=N):
                t = base if i == 0 else tuple(a.clone() for a in base)
                return t + (torch.empty((Mo, N), dtype=torch.bfloat16, device=device),)

            def launch(c, keep=keep):
                x, q, s_, b_, y = c
                if keep:
                    w4.w4a16_matmul_last_rows(x, q, s_, b_, keep, y=y)
                else:
                    w4.w4a16_matmul(x, q, s_, b_, y=y)

            flops = 2 * Mo * N * K
            reps = int(max(4, min(64, 2e9 / max(flops, 1))))
            us = time_calls(make_copy, launch, n_copies, reps, stream)
            del base
            b = algo_bytes(Mo, N, K)
            # compact per-call rows: [M, projection, N, K, us, fraction of the bound's peak]
            frac = b / us / 1e3 / pk["hbm_gbs"] if key == "lm_head_last_row" else flops / us / 1e6 / flop_peak
            rows.append([Mo, name, N, K, round(us, 3), round(frac, 4)])
            tot_flops += flops
            tot_us += us
            tot_bytes += b
        agg_tf = tot_flops / tot_us / 1e6
        agg_gb = tot_bytes / tot_us / 1e3
        bound = "hbm" if key == "lm_head_last_row" else "tensor"
        out[key] = {"workload": desc, "us": round(tot_us, 3), "tflops": round(agg_tf, 2),
                    "gbs": round(agg_gb, 1), "bound": bound,
                    "frac": round(agg_gb / pk["hbm_gbs"] if bound == "hbm" else agg_tf / flop_peak, 4),
                    "frac_nominal": round(agg_gb / NOMINAL_PEAKS["hbm_gbs"] if bound == "hbm"
                                          else agg_tf / NOMINAL_PEAKS["bf16_tflops"], 4),
                    "calls": rows}
        torch.cuda.empty_cache()
    return out


QUANT_CASES = (("gate 9728 x 2560, FP32", 9728, 2560, "f32"),
               ("gate 9728 x 2560, BF16", 9728, 2560, "bf16"),
               ("lm_head 151936 x 2560, BF16", 151936, 2560, "bf16"))


def quantize_section(device, stream, pk):
    """Time the on-GPU quantiser (weights -> packed codes, scales, biases): HBM-bound, its
    algorithmic bytes are the weights read once and the packed format written once."""
    import torch
    import decode_w4a16_g128_b200 as w4
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    rows, tot_b, tot_us = [], 0, 0.0
    for desc, N, K, dt in QUANT_CASES:
        esz = 4 if dt == "f32" else 2
        b = N * K * esz + N * K // 2 + 4 * N * K // 128
        g = torch.Generator(device=device).manual_seed(N)
        base = torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * 0.02
        if dt == "bf16":
            base = base.to(torch.bfloat16)
        n_copies = int(max(2, min(8, math.ceil(2.2 * l2 / b))))

        def make_copy(i, base=base, N=N, K=K):
            w = base if i == 0 else base.clone()
            return (w, torch.empty((N, K // 8), dtype=torch.int32, device=device),
                    torch.empty((N, K // 128), dtype=torch.bfloat16, device=device),
                    torch.empty((N, K // 128), dtype=torch.bfloat16, device=device))

        def launch(c):
            w4.w4a16_quantize(c[0], wq=c[1], scales=c[2], biases=c[3])

        us = time_calls(make_copy, launch, n_copies, 16, stream)
        del base
        torch.cuda.empty_cache()
        rows.append([desc, round(us, 3), round(b / us / 1e3, 1), round(b / us / 1e3 / pk["hbm_gbs"], 4)])
        tot_b += b
        tot_us += us
    gbs = tot_b / tot_us / 1e3
    return {"workload": "W4 g128 min/max quantiser, FP32 or BF16 weights to packed codes, scales and biases",
            "kernel": "w4a16::qz::quantize_kernel", "bound": "hbm", "us": round(tot_us, 3), "gbs": round(gbs, 1),
            "frac": round(gbs / pk["hbm_gbs"], 4), "peak": pk["hbm_gbs"], "calls": rows,
            "calls_fields": ["workload", "us", "GB/s", "fraction of measured HBM"]}


def gate_up_section(device, stream, pk):
    """The fused gate/up projection with SwiGLU (one row-block matvec over interleaved rows)
    against the same work as two layer calls, Qwen3-4B gate/up 2560 -> 9728, M in {1, 8}."""
    import torch
    import decode_w4a16_g128_b200 as w4
    N2, K = 9728, 2560
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    gq, gs, gb = synth.make_weights(synth.shape_rng(0, N2, K, seed=11), N2, K)
    uq, us, ub = synth.make_weights(synth.shape_rng(0, N2, K, seed=12), N2, K)

    def dev(a, bf16):
        t = torch.from_numpy(a.view(np.int16 if bf16 else np.int32)).to(device)
        return t.view(torch.bfloat16) if bf16 else t

    fused_w = (dev(synth.interleave_gate_up(gq, uq), False), dev(synth.interleave_gate_up(gs, us), True),
               dev(synth.interleave_gate_up(gb, ub), True))
    sep_w = (dev(gq, False), dev(gs, True), dev(gb, True), dev(uq, False), dev(us, True), dev(ub, True))
    b_w = 2 * algo_bytes(0, N2, K)
    n_copies = int(max(2, min(8, math.ceil(2.2 * l2 / b_w))))
    rows = []
    for M in (1, 8):
        x = dev(synth.make_x(synth.shape_rng(M, N2, K, seed=13), M, K), True)

        def copy_fused(i, M=M, x=x):
            w = fused_w if i == 0 else tuple(a.clone() for a in fused_w)
            return (x,) + w + (torch.empty((M, N2), dtype=torch.bfloat16, device=device),)

        def copy_sep(i, M=M, x=x):
            w = sep_w if i == 0 else tuple(a.clone() for a in sep_w)
            return (x,) + w + (torch.empty((M, N2), dtype=torch.bfloat16, device=device),
                               torch.empty((M, N2), dtype=torch.bfloat16, device=device))

        def fused(c):
            w4.w4a16_gate_up(c[0], c[1], c[2], c[3], h=c[4])

        def separate(c):
            w4.w4a16_matmul(c[0], c[1], c[2], c[3], y=c[7])
            w4.w4a16_matmul(c[0], c[4], c[5], c[6], y=c[8])

        us_f = time_calls(copy_fused, fused, n_copies, 16, stream)
        us_s = time_calls(copy_sep, separate, n_copies, 16, stream)
        byts = b_w + 2 * M * K + 2 * M * N2
        rows.append([M, round(us_f, 3), round(us_s, 3), round(byts / us_f / 1e3, 1),
                     round(byts / us_f / 1e3 / pk["hbm_gbs"], 4)])
    torch.cuda.empty_cache()
    return {"workload": "gate and up 2560 -> 9728 with silu(gate) * up, Qwen3-4B MLP",
            "kernel": "w4a16::mvr::rows_kernel (gated)", "bound": "hbm", "calls": rows,
            "calls_fields": ["M", "fused us", "two layer calls us (no SwiGLU)", "fused GB/s",
                             "fused fraction of measured HBM"]}


def bits_algo_bytes(M, N, K, bits):
    """Bytes a b-bit layer call must move at least: codes, scales and biases once, x and y once."""
    return N * K * bits // 8 + 4 * N * (K // 128) + 2 * M * K + 2 * M * N


def bits_section(device, stream, pk):
    """Decode (M in {1, 8}) over the seven Qwen3-4B projections with 2-, 4- and 8-bit codes
    through w4a16_matmul_bits (4 bits: the 4-bit layer's own path).  Codes are random words and
    scales / biases small random BF16 values generated on the device: the timing depends on
    the bytes, not on the values."""
    import torch
    import decode_w4a16_g128_b200 as w4
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    g = torch.Generator(device=device).manual_seed(2024)
    rows, summary = [], {}
    for bits in (2, 4, 8):
        for M in (1, 8):
            tot_us, tot_b = 0.0, 0
            for (name, K, N) in synth.QWEN3_4B_PROJECTIONS:
                G = K // 128
                base = (torch.randn((M, K), generator=g, device=device).to(torch.bfloat16),
                        torch.randint(-2 ** 31, 2 ** 31 - 1, (N, K * bits // 32), generator=g, device=device,
                                      dtype=torch.int32),
                        (0.002 + 0.001 * torch.rand((N, G), generator=g, device=device)).to(torch.bfloat16),
                        (-0.03 - 0.01 * torch.rand((N, G), generator=g, device=device)).to(torch.bfloat16))
                b = bits_algo_bytes(M, N, K, bits)
                n_copies = int(max(2, min(16, math.ceil(2.2 * l2 / b))))

                def make_copy(i, base=base, M=M, N=N):
                    t = base if i == 0 else tuple(a.clone() for a in base)
                    return t + (torch.empty((M, N), dtype=torch.bfloat16, device=device),)

                def launch(c, bits=bits):
                    w4.w4a16_matmul_bits(c[0], c[1], c[2], c[3], bits, y=c[4])

                us = time_calls(make_copy, launch, n_copies, 16, stream)
                del base
                rows.append([bits, M, name, N, K, round(us, 3), round(b / us / 1e3, 1)])
                tot_us += us
                tot_b += b
            summary[f"{bits}bit_m{M}"] = {"us": round(tot_us, 3), "gbs": round(tot_b / tot_us / 1e3, 1),
                                          "frac": round(tot_b / tot_us / 1e3 / pk["hbm_gbs"], 4)}
    torch.cuda.empty_cache()
    return {"workload": "decode M in {1, 8}, seven Qwen3-4B projections, 2-, 4- and 8-bit affine codes, g128",
            "kernel": "w4a16::nb::nbit_kernel<2|8> (4 bits: the 4-bit layer's decode path)", "bound": "hbm",
            "peak": pk["hbm_gbs"], "summary": summary, "calls": rows,
            "calls_fields": ["bits", "M", "projection", "N", "K", "us", "GB/s"]}


def skinny_section(device, stream, pk, weights_cache):
    """8 < M <= 32: slices of the row-block matvec against the GEMM, per Qwen3-4B projection
    (the measured crossover behind the automatic choice)."""
    import torch
    import decode_w4a16_g128_b200 as w4
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    rows = []
    for M in (12, 16, 24, 32):
        for (name, K, N) in synth.QWEN3_4B_PROJECTIONS:
            if (name, K, N) not in weights_cache:
                weights_cache[(name, K, N)] = synth.make_weights(synth.shape_rng(0, N, K, seed=0), N, K)
            wq, sc, bi = weights_cache[(name, K, N)]
            x = synth.make_x(synth.shape_rng(M, N, K, seed=1), M, K)
            base = (torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16),
                    torch.from_numpy(wq.view(np.int32)).to(device),
                    torch.from_numpy(sc.view(np.int16)).to(device).view(torch.bfloat16),
                    torch.from_numpy(bi.view(np.int16)).to(device).view(torch.bfloat16))
            n_copies = int(max(2, min(16, math.ceil(2.2 * l2 / algo_bytes(M, N, K)))))

            def make_copy(i, base=base, M=M, N=N):
                t = base if i == 0 else tuple(a.clone() for a in base)
                return t + (torch.empty((M, N), dtype=torch.bfloat16, device=device),)

            res = []
            for path in (w4.PATH_MATVEC_ROWS, w4.PATH_GEMM):
                def launch(c, path=path):
                    w4.w4a16_matmul_ex(c[0], c[1], c[2], c[3], y=c[4], path=path)
                res.append(time_calls(make_copy, launch, n_copies, 16, stream))
            del base
            rows.append([M, name, N, K, round(res[0], 3), round(res[1], 3)])
    torch.cuda.empty_cache()
    return {"workload": "M in {12, 16, 24, 32} x the seven Qwen3-4B projections",
            "calls": rows, "calls_fields": ["M", "projection", "N", "K", "row-block slices us", "GEMM us"]}


def profile_case(args, device, stream):
    """Three eager calls of one problem (for an ncu capture of one kernel): 'M,N,K' (the layer),
    'quant:N,K,f32|bf16' (the quantiser), 'gateup:M,N2,K' (the fused gate/up projection) or
    'bits:b,M,N,K' (the layer with b-bit codes)."""
    import torch
    import decode_w4a16_g128_b200 as w4
    if args.case.startswith("quant:"):
        n_, k_, dt = args.case[len("quant:"):].split(",")
        N, K = int(n_), int(k_)
        g = torch.Generator(device=device).manual_seed(N)
        W = torch.randn((N, K), generator=g, device=device, dtype=torch.float32) * 0.02
        if dt == "bf16":
            W = W.to(torch.bfloat16)
        with torch.cuda.stream(stream):
            for _ in range(3):
                w4.w4a16_quantize(W)
        torch.cuda.synchronize()
        return 0
    if args.case.startswith("bits:"):
        bits, M, N, K = (int(v) for v in args.case[len("bits:"):].split(","))
        prob = synth.make_problem_bits(M, N, K, bits)
        d = [torch.from_numpy(prob[k].view(np.int16 if prob[k].dtype == np.uint16 else np.int32)).to(device)
             for k in ("x", "wq", "scales", "biases")]
        with torch.cuda.stream(stream):
            for _ in range(3):
                w4.w4a16_matmul_bits(d[0].view(torch.bfloat16), d[1], d[2].view(torch.bfloat16),
                                     d[3].view(torch.bfloat16), bits)
        torch.cuda.synchronize()
        if w4.w4a16_device_status(stream) != w4.OK:
            raise RuntimeError("device status not ok")
        return 0
    if args.case.startswith("gateup:"):
        M, N2, K = (int(v) for v in args.case[len("gateup:"):].split(","))
        rng = synth.shape_rng(M, N2, K, seed=3)
        x = synth.make_x(rng, M, K)
        gw = [synth.make_weights(rng, N2, K) for _ in range(2)]
        gu = [synth.interleave_gate_up(gw[0][i], gw[1][i]) for i in range(3)]
        xd = torch.from_numpy(x.view(np.int16)).to(device).view(torch.bfloat16)
        wd = torch.from_numpy(gu[0].view(np.int32)).to(device)
        sd = torch.from_numpy(gu[1].view(np.int16)).to(device).view(torch.bfloat16)
        bd = torch.from_numpy(gu[2].view(np.int16)).to(device).view(torch.bfloat16)
        with torch.cuda.stream(stream):
            for _ in range(3):
                w4.w4a16_gate_up(xd, wd, sd, bd)
        torch.cuda.synchronize()
        if w4.w4a16_device_status(stream) != w4.OK:
            raise RuntimeError("device status not ok")
        return 0
    M, N, K = (int(v) for v in args.case.split(","))
    prob = synth.make_problem(M, N, K)
    d = [torch.from_numpy(prob[k].view(np.int16 if prob[k].dtype == np.uint16 else np.int32)).to(device)
         for k in ("x", "wq", "scales", "biases")]
    x, wq, sc, bi = d[0].view(torch.bfloat16), d[1], d[2].view(torch.bfloat16), d[3].view(torch.bfloat16)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    with torch.cuda.stream(stream):
        for _ in range(3):
            w4.w4a16_matmul(x, wq, sc, bi, y=y)
    torch.cuda.synchronize()
    if w4.w4a16_device_status(stream) != w4.OK:
        raise RuntimeError("device status not ok")
    return 0


def detail(args, entries, calls, stream, pk):
    """Per-call times (graph of 20 back-to-back repeats of one call over 8 weight copies)."""
    import torch
    import decode_w4a16_g128_b200 as w4
    rows = []
    for (x, wq, s, b, y), (M, name, K, N) in zip(entries, calls):
        copies = [(wq.clone(), s.clone(), b.clone()) for _ in range(max(2, int(400e6 // (N * K // 2)) + 1))]
        copies = copies[:32]
        reps = 64
        with torch.cuda.stream(stream):
            for (cw, cs, cb) in copies:
                w4.w4a16_matmul_ex(x, cw, cs, cb, y=y, flags=w4.FLAG_STATIC_WEIGHTS)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(reps):
                cw, cs, cb = copies[i % len(copies)]
                w4.w4a16_matmul_ex(x, cw, cs, cb, y=y, flags=w4.FLAG_STATIC_WEIGHTS)
        with torch.cuda.stream(stream):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(5):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / (5 * reps)
        gb = algo_bytes(M, N, K) / (us * 1e-6) / 1e9
        rows.append({"M": M, "proj": name, "N": N, "K": K, "us": round(us, 3), "GB/s": round(gb, 1),
                     "frac_hbm": round(gb / pk["hbm_gbs"], 3)})
        del g, copies
    if args.detail:
        with open(args.detail, "w") as f:
            json.dump(rows, f, indent=1)
    for r in rows:
        print(json.dumps(r), file=sys.stderr)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--mode", choices=("bench", "profile"), default="bench")
    ap.add_argument("--detail", default="", metavar="PATH",
                    help="also time every decode call on its own and write the table to PATH (JSON)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the M > 8 measurements")
    ap.add_argument("--no-quantize", action="store_true",
                    help="skip the quantiser, fused gate/up and 2- / 8-bit measurements")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="time bound of the CPU baseline sample")
    ap.add_argument("--case", default="", help="profile mode: one problem 'M,N,K' (three eager calls)")
    ap.add_argument("--ref-fraction", type=float, default=0.125,
                    help="reference arm: fraction of each call's output columns per step")
    args = ap.parse_args()
    if args.warmup < 3 and args.mode == "bench":
        ap.error("--warmup must be at least 3")
    world, rank, local = dist_setup(args)
    if args.impl == "reference":
        return run_reference(args, world, rank)
    return run_ours(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
