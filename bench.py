#!/usr/bin/env python3
"""Benchmark of the fused Dense-and-Sparse LUT GEMV, y = (Q + S) x.

One step = one batch-1 token through a stack of R distinct layers of the
workload's shape: R fused-kernel calls, each on its own layer instance with
its own activations.  R is at least 32 (LLaMA-7B's decoder depth) and large
enough that the stack is at least 4x the L2 cache, so every call streams its
layer from HBM.  The K timed steps are CUDA-graph replays (several steps per
graph, one kernel node per call), bracketed by a barrier and a device
synchronise, timed with CUDA events on the launching stream; the reported
time is the maximum over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Prints one JSON line on rank 0.  ``--gpus N`` without a torchrun
environment starts N ranks itself (one GPU each, independent replicas).
``--impl reference`` times the CPU oracle (plain fp64 C) on a bounded
sample of the same workload.  ``--sweep`` prints one line per workload
shape instead (for the notes).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from lut_dequant_gemv_b200 import accounting as acc  # noqa: E402

DEFAULT_WORKLOAD = "llama7b-up-3bit"
METRIC = "3-bit dense+sparse GEMV achieved HBM GB/s (LLaMA-7B up_proj 11008x4096, batch 1)"
FALLBACK_HBM_GBS = 6650.0

WORKLOAD_DESC = {
    "llama7b-q-4bit": "LLaMA-7B q_proj 4096x4096, 4-bit, 0.45% CSR outliers, batch 1",
    "llama7b-up-3bit": "LLaMA-7B MLP up_proj 11008x4096, 3-bit, 0.45% CSR outliers, batch 1",
}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=200)
    p.add_argument("--workload", default=DEFAULT_WORKLOAD)
    p.add_argument("--shape-index", type=int, default=0)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--sweep", action="store_true", help="one JSON line per workload shape")
    p.add_argument("--stack", type=int, default=0,
                   help="layers per step (default: at least 32 and at least 4x L2; never below 4x L2)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--predecode", type=int, choices=(0, 1, 8, 16), default=0,
                   help="batches of 1..8: the kernel that decodes ahead of x into tensor memory (1; 8 or 16 dense "
                        "warps per CTA) instead of the default 12-warp kernel (0)")
    p.add_argument("--mac", choices=("tensor", "cuda", "mixed"), default="tensor",
                   help="batch-1 multiply-accumulate unit of the 12-warp kernel (sqz_layer_set_mac)")
    p.add_argument("--csr", choices=("balanced", "rowwise"), default="balanced",
                   help="sparse scheme of the fused kernel (rowwise: the plain CSR comparison)")
    p.add_argument("--encode", action="store_true",
                   help="time the encoder (sqz_encode) on synthetic weights of the workload's shape instead")
    p.add_argument("--encode-iters", type=int, default=30, help="k-means iterations of --encode")
    p.add_argument("--selftest-ranks", action="store_true",
                   help="(tests) the rank plumbing alone on CPU: gloo ranks report fixed times, no GPU work")
    p.add_argument("--profile-launches", type=int, default=0,
                   help="for profiler captures: one layer instance of the shape, this many plain launches, "
                        "no timing and no JSON line")
    return p.parse_args()


# ----------------------------------------------------------------- helpers

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def instance_id(rank: int, i: int) -> int:
    """Layer instance i of a rank: every rank owns its own layers (replicas
    of the workload, no shared data and no data-path collective)."""
    return rank * 1000 + i


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The slowest rank's time: an all-reduce MAX of one float (NCCL on the
    GPU run, gloo on CPU); the value itself when there is one rank."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, bytes_per_step: int, steps: int, ms: float) -> float:
    """Whole-job throughput: every rank processes bytes_per_step per step,
    and the job takes the slowest rank's ms."""
    return world * bytes_per_step * steps / (ms / 1e3) / 1e9


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


KERNEL_SOURCES = ("common.cuh", "kernels_tc.cuh")  # the fused kernel's device code


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "lut_dequant_gemv_b200", "csrc")
    for name in KERNEL_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + b"\0" + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str, shape_key: str, batch: int = 1):
    """DRAM bytes per launch from the committed ncu summary, valid only while
    the kernel sources are unchanged since the capture."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    want = kernel_source_hash()
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            kv = dict(tok.split("=", 1) for tok in line.split())
            if (kv.get("shape") == shape_key and kv.get("batch", "1") == str(batch)
                    and kv.get("source_hash") == want and "bytes_per_launch" in kv):
                return int(kv["bytes_per_launch"])
    return None


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.0):
        self.ok = False
        self.samples, self.reasons = [], 0
        self.period = period_s
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(self._physical_index(device_index))
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML missing: report that instead of clocks
            self.err = str(e)
        self._stop = threading.Event()

    @staticmethod
    def _physical_index(i):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            try:
                return int(vis.split(",")[i])
            except Exception:
                return i
        return i

    def _run(self):
        # back to back (sleep(0) only yields to the launching thread): the
        # NVML queries themselves set the pace, a fraction of a millisecond
        # per sample, so even a timed region of a few ms gets ten or more
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
            t0 = time.perf_counter()
            while not self.samples and time.perf_counter() - t0 < 1.0:  # sampling before the region starts
                time.sleep(0.0001)
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": f"NVML unavailable: {self.err}"}
        names = [n for b, n in self.REASONS.items() if self.reasons & b]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


def shape_for(args) -> synth.Shape:
    shapes = synth.workloads()[args.workload]
    return shapes[args.shape_index]


def config_for(args, shape, instances, inst_bytes):
    return {
        "workload": f"{args.workload}: " + WORKLOAD_DESC.get(
            args.workload, f"{shape.n_out}x{shape.k_in}, {shape.bits}-bit, {shape.density:.2%} CSR, batch {shape.batch}"),
        "n_out": shape.n_out, "k_in": shape.k_in, "bits": shape.bits, "density": shape.density,
        "batch": shape.batch, "outliers": shape.dist, "csr_scheme": args.csr, "mac": getattr(args, "mac", "tensor"),
        "kernel": "decode-ahead (TMEM)" if getattr(args, "predecode", 0) and shape.batch <= 8 else "12-warp fused",
        "step": f"one token through a stack of {instances} distinct layers of this shape ({instances} calls)",
        "l2": f"inputs larger than L2: the stack holds {instances * inst_bytes / 1e6:.0f} MB",
        "parallelism": "replicas (independent layers per GPU)",
    }


# ------------------------------------------------------------- CPU oracle

def _oracle_rows_rate(orc, L, x, rows_per_call, seconds, start_row, per_row_bytes):
    """One thread: oracle calls over consecutive row blocks for `seconds`;
    returns (rows, elapsed s)."""
    done, t0, start = 0, time.perf_counter(), start_row
    while True:
        rows = (np.arange(start, start + rows_per_call) % L.n_out).astype(np.int32)
        orc.gemv_layer(L, x, rows=rows)
        done += rows_per_call
        start += rows_per_call
        el = time.perf_counter() - t0
        if el >= seconds:
            return done, el


def cpu_oracle_rate(shape, seconds: float, rows_per_call: int, threads: int = 1, instance: int = 0):
    """The oracle as it stands on `threads` host threads (ctypes releases the
    GIL, so the C oracle runs in parallel on disjoint row blocks), for about
    `seconds`; returns (GB/s, rows done, elapsed s)."""
    import oracle

    orc = oracle.default()
    L = synth.layer_for(shape, instance=instance)
    x = synth.x_for(shape, instance=instance)
    per_row_bytes = acc.gemv_bytes(shape.n_out, shape.k_in, shape.bits, L.nnz, shape.batch) / shape.n_out
    out = [None] * threads

    def work(t):
        out[t] = _oracle_rows_rate(orc, L, x, rows_per_call, seconds, t * (shape.n_out // threads), per_row_bytes)

    t0 = time.perf_counter()
    ts = [threading.Thread(target=work, args=(t,)) for t in range(threads)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    el = time.perf_counter() - t0
    rows = sum(r for r, _ in out)
    return rows * per_row_bytes / el / 1e9, rows, el


def cpu_baseline(shape, seconds_per_rep: float = 2.5, reps: int = 3):
    """Median of `reps` timings at one thread and at every host core."""
    cores = os.cpu_count() or 1
    res = {}
    for threads in sorted({1, cores}):
        runs = [cpu_oracle_rate(shape, seconds_per_rep, 64, threads) for _ in range(reps)]
        gbs = statistics.median(r[0] for r in runs)
        res[threads] = (gbs, sum(r[1] for r in runs), sum(r[2] for r in runs))
    gbs, rows, secs = res[cores]
    line = {"value": gbs, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{rows} rows of one {shape.n_out}x{shape.k_in} layer in {secs:.1f} s on {cores} host threads "
                      f"(fp64 C oracle, disjoint row blocks per thread), median of {reps}"}
    g1, r1, s1 = res[1]
    line["one_thread"] = {"value": g1, "unit": "GB/s", "cores": 1,
                          "sample": f"{r1} rows in {s1:.1f} s on one thread, median of {reps}"}
    return line


def run_reference(args):
    world, rank, local = dist_env()
    if rank != 0:
        return 0
    import oracle

    shape = shape_for(args)
    orc = oracle.default()
    L = synth.layer_for(shape)
    x = synth.x_for(shape)
    # size each step so that W + K steps take about 90 s of CPU time
    t0 = time.perf_counter()
    orc.gemv_layer(L, x, rows=np.arange(64, dtype=np.int32))
    per_row = (time.perf_counter() - t0) / 64
    rows_per_step = max(1, min(shape.n_out, int(90.0 / max(1, args.steps + args.warmup) / per_row)))
    per_row_bytes = acc.gemv_bytes(shape.n_out, shape.k_in, shape.bits, L.nnz, shape.batch) / shape.n_out

    def step(i):
        rows = ((np.arange(rows_per_step) + i * rows_per_step) % shape.n_out).astype(np.int32)
        orc.gemv_layer(L, x, rows=rows)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    el = time.perf_counter() - t0
    gbs = args.steps * rows_per_step * per_row_bytes / el / 1e9
    sample = f"{rows_per_step} of {shape.n_out} rows per step (fp64 C oracle, one thread)"
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_for(args, shape, 1, L.nbytes()),
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------ GPU arm

MIN_STACK = 32          # layers per step: at least LLaMA-7B's decoder depth
CALLS_PER_GRAPH = 512   # about this many kernel nodes per captured graph


def stack_depth(l2_bytes: int, layer_bytes: int, requested: int = 0) -> int:
    """Layers per step: at least 4x L2 in total, and MIN_STACK unless another
    depth is requested."""
    return max(requested if requested > 0 else MIN_STACK, math.ceil(4 * l2_bytes / layer_bytes))


def graph_plan(steps: int, per_graph: int):
    """Replays of the full graph and the step count of the tail graph."""
    return divmod(steps, per_graph)


def run_ours(args):
    import torch
    import torch.distributed as dist

    from lut_dequant_gemv_b200 import binding as B

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    B.lib()

    shape = shape_for(args)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    L0 = synth.layer_for(shape, seed=args.seed, instance=instance_id(rank, 0))
    inst_bytes = L0.nbytes()
    R = stack_depth(l2, inst_bytes, args.stack)
    layers, xs, ys = [], [], []
    for i in range(R):
        L = L0 if i == 0 else synth.layer_for(shape, seed=args.seed, instance=instance_id(rank, i))
        layers.append(B.create_layer_from_numpy(L.n_out, L.k_in, L.bits, L.codes, L.lut, L.rowptr, L.col, L.val,
                                                device=dev))
        if args.csr == "rowwise":
            B.sqz_layer_set_csr_mode(layers[-1], B.SQZ_CSR_ROWWISE)
        if args.predecode:
            B.sqz_layer_set_predecode(layers[-1], args.predecode)
        if args.mac != "tensor":
            B.sqz_layer_set_mac(layers[-1], {"cuda": B.SQZ_MAC_CUDA_CORES, "mixed": B.SQZ_MAC_MIXED}[args.mac])
        xs.append(torch.from_numpy(synth.x_for(shape, seed=args.seed, instance=instance_id(rank, i)).view(np.int16))
                  .to(dev))
        ys.append(torch.empty((shape.batch, shape.n_out), dtype=torch.int16, device=dev))
    nnz = L0.nnz
    bytes_per_call = acc.gemv_bytes(shape.n_out, shape.k_in, shape.bits, nnz, shape.batch)
    bytes_per_step = R * bytes_per_call

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        for i in range(R):
            B.sqz_gemv(layers[i], xs[i], ys[i], stream=stream)
    stream.synchronize()

    def capture(nsteps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for _ in range(nsteps):
                for i in range(R):
                    B.sqz_gemv(layers[i], xs[i], ys[i], stream=stream)
        return g

    per_graph = max(1, CALLS_PER_GRAPH // R)  # steps per full graph
    graphs = {per_graph: capture(per_graph)}
    for k in (args.warmup % per_graph, args.steps % per_graph):
        if k and k not in graphs:
            graphs[k] = capture(k)

    def run_steps(k):
        full, tail = graph_plan(k, per_graph)
        for _ in range(full):
            graphs[per_graph].replay()
        if tail:
            graphs[tail].replay()

    with torch.cuda.stream(stream):
        for g in graphs.values():  # first replays upload the graphs
            g.replay()
        run_steps(args.warmup)
    stream.synchronize()

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        with torch.cuda.stream(stream):
            ev0.record(stream)
            run_steps(args.steps)
            ev1.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    ms_per_step = ms / args.steps
    us_per_call = ms_per_step * 1e3 / R
    value = whole_job_gbs(world, bytes_per_step, args.steps, ms)
    per_launch_gbs = bytes_per_call / (us_per_call * 1e-6) / 1e9

    e2e = e2e_measure(B, torch, dist, shape, layers, xs, R, args, world, rank, dev, stream, bytes_per_step,
                      us_per_call)

    # ---- fp16 dense yardstick (same shape, uncompressed weights)
    yard = None
    try:
        yard = fp16_yardstick(B, torch, shape, dev, stream, l2)
    except Exception as e:  # reported, never fatal for the headline
        yard = {"error": str(e)}

    peak, peak_kind = measured_peaks()
    traffic = recorded_traffic(args.workload, shape.key, shape.batch)
    line = {
        "metric": METRIC if args.workload == DEFAULT_WORKLOAD else f"dense+sparse GEMV achieved HBM GB/s ({args.workload})",
        "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms_per_step, "us_per_call": us_per_call, "calls_per_step": R,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16 storage, f32 accumulate", "data": "synthetic",
        "config": config_for(args, shape, R, inst_bytes),
        "roofline": {"bound": "hbm", "achieved": per_launch_gbs, "peak": peak, "unit": "GB/s",
                     "frac": per_launch_gbs / peak, "traffic": traffic,
                     "peak_kind": f"{peak_kind} copy bandwidth", "algorithmic_bytes_per_launch": bytes_per_call,
                     "frac_of_nominal_8000": per_launch_gbs / 8000.0},
        "e2e": e2e,
        "gpu_launches": args.steps * R,
        "clocks": clk.summary(),
        "yardstick_fp16_dense": yard,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(shape)
    if rank == 0:
        print(json.dumps(line), flush=True)
    for lay in layers:
        lay.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def e2e_measure(B, torch, dist, shape, layers, xs_dev, R, args, world, rank, dev, stream, bytes_per_step, us_kernel):
    """End to end through the host entry point: every call copies its
    layer's x in from pinned host memory, runs the product, copies y back
    and synchronises.  One step = R calls (the same stack as the device
    measurement).  Every (layer, host buffers) pair is warmed first, so the
    timed calls replay captured graphs rather than capture them."""
    xh = [torch.from_numpy(synth.x_for(shape, seed=args.seed, instance=instance_id(rank, i)).view(np.int16).copy())
          .pin_memory() for i in range(R)]
    yh = torch.empty((shape.batch, shape.n_out), dtype=torch.int16).pin_memory()
    steps = max(1, min(args.steps, 200))
    with torch.cuda.stream(stream):
        for _ in range(max(2, min(args.warmup, 20))):
            for i in range(R):
                B.sqz_gemv_host(layers[i], xh[i], yh, stream=stream)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        t0 = time.perf_counter()
        for _ in range(steps):
            for i in range(R):
                B.sqz_gemv_host(layers[i], xh[i], yh, stream=stream)
        wall = time.perf_counter() - t0
        e1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    calls = steps * R
    us_call = ms * 1e3 / calls

    # ---- where a call's time goes: the same call without moving x and y
    # (sqz_gemv on device buffers, then a stream synchronise; wall clock, the
    # same layer rotation) is the cost of a lone synchronous product; the
    # rest of the e2e call is bringing x in and taking y out.  The kernel in a
    # chain of calls and the parts alone on an idle stream (CUDA events; they
    # carry the start-from-idle cost) are listed for reference.
    yd = torch.empty((shape.batch, shape.n_out), dtype=torch.int16, device=dev)
    xd0 = torch.empty((shape.batch, shape.k_in), dtype=torch.int16, device=dev)
    with torch.cuda.stream(stream):
        for i in range(R):
            B.sqz_gemv(layers[i], xs_dev[i], yd, stream=stream)
            stream.synchronize()
        n_sync = max(R, min(calls, 2000))
        t0 = time.perf_counter()
        for j in range(n_sync):
            B.sqz_gemv(layers[j % R], xs_dev[j % R], yd, stream=stream)
            stream.synchronize()
        sync_us = (time.perf_counter() - t0) / n_sync * 1e6

    def timed(fn, n=50):
        out = []
        with torch.cuda.stream(stream):
            for i in range(n):
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn(i)
                b.record(stream)
                b.synchronize()
                out.append(a.elapsed_time(b) * 1e3)
        return statistics.median(out)

    kern_us = timed(lambda i: B.sqz_gemv(layers[i % R], xs_dev[i % R], yd, stream=stream))
    h2d_us = timed(lambda i: xd0.copy_(xh[i % R], non_blocking=True))
    d2h_us = timed(lambda i: yh.copy_(yd, non_blocking=True))
    lib = B.lib()
    n = 20000
    t0 = time.perf_counter()
    for _ in range(n):
        lib.sqz_version()
    ctypes_us = (time.perf_counter() - t0) / n * 1e6
    return {"value": whole_job_gbs(world, bytes_per_step, steps, ms), "unit": "GB/s",
            "h2d_bytes_per_step": R * 2 * shape.batch * shape.k_in,
            "d2h_bytes_per_step": R * 2 * shape.batch * shape.n_out,
            "us_per_call": us_call, "wall_us_per_call": wall * 1e6 / calls, "steps": steps, "calls_per_step": R,
            "api": "sqz_gemv_host (pinned host x/y)",
            "breakdown_us": {"synchronous_product_without_io": sync_us,
                             "moving_x_in_and_y_out": us_call - sync_us,
                             "ctypes_round_trip": ctypes_us,
                             "kernel_in_a_chain_of_calls": us_kernel,
                             "alone_from_idle_events": {"kernel": kern_us, "h2d_copy_engine": h2d_us,
                                                        "d2h_copy_engine": d2h_us}}}


def fp16_yardstick(B, torch, shape, dev, stream, l2):
    """fp16 dense GEMV over the same shape (2*N*K weight bytes), same protocol."""
    wbytes = 2 * shape.n_out * shape.k_in
    n = max(2, math.ceil(4 * l2 / wbytes))
    g = torch.Generator(device=dev).manual_seed(1)
    ws = [(torch.randn(shape.n_out, shape.k_in, device=dev, generator=g) * 0.02).half() for _ in range(n)]
    x = torch.randn(shape.batch, shape.k_in, device=dev, generator=g).half()
    y = torch.empty(shape.batch, shape.n_out, device=dev, dtype=torch.half)
    torch.cuda.synchronize(dev)
    reps = n * max(1, 256 // n)
    with torch.cuda.stream(stream):
        for i in range(n):
            B.sqz_fp16_gemv(ws[i], x, y, stream=stream)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=stream):
            for j in range(reps):
                B.sqz_fp16_gemv(ws[j % n], x, y, stream=stream)
        gr.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(5):
            gr.replay()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    us = e0.elapsed_time(e1) * 1e3 / (5 * reps)
    nbytes = acc.fp16_dense_bytes(shape.n_out, shape.k_in, shape.batch)
    del ws
    return {"us_per_call": us, "GB/s": nbytes / (us * 1e-6) / 1e9, "bytes": nbytes}


def run_sweep(args):
    """One JSON line per workload shape (single GPU, short)."""
    import subprocess

    for name, shapes in synth.workloads().items():
        for i in range(len(shapes)):
            cmd = [sys.executable, __file__, "--workload", name, "--shape-index", str(i), "--steps",
                   str(args.steps), "--warmup", str(args.warmup), "--no-cpu-baseline", "--stack", str(args.stack or 1)]
            subprocess.run(cmd, check=True)
    return 0


def run_profile_launches(args):
    """One layer instance, N back-to-back launches on the default stream (a
    short, bounded program for an ncu capture of one launch per shape).
    ``--workload all``: every shape of every workload in turn, N launches
    each, one layer alive at a time (launch N*s + j of the fused kernel is
    launch j of shape s, in the order printed)."""
    import torch

    from lut_dequant_gemv_b200 import binding as B

    B.lib()
    if args.workload == "all":
        shapes = [(name, i) for name, ss in synth.workloads().items() for i in range(len(ss))]
    else:
        shapes = [(args.workload, args.shape_index)]
    for name, i in shapes:
        shape = synth.workloads()[name][i]
        L = synth.layer_for(shape, seed=args.seed)
        layer = B.create_layer_from_numpy(L.n_out, L.k_in, L.bits, L.codes, L.lut, L.rowptr, L.col, L.val)
        x = torch.from_numpy(synth.x_for(shape, seed=args.seed).view(np.int16)).cuda()
        y = torch.empty((shape.batch, shape.n_out), dtype=torch.int16, device="cuda")
        for _ in range(args.profile_launches):
            B.sqz_gemv(layer, x, y)
        torch.cuda.synchronize()
        print(f"{name} {i} {shape.key} B{shape.batch}: {args.profile_launches} launches", flush=True)
        layer.close()
    return 0


def run_encode(args):
    """The encoder on one layer of the workload's shape: synthetic Student-t
    fp16 weights, the shape's bits and outlier fraction; ms per layer on the
    device (CUDA events, K timed calls after W warm-up calls) and the fp64
    oracle on a bounded sample (the whole outlier split plus the k-means of
    a few rows, scaled to the layer)."""
    import torch

    from lut_dequant_gemv_b200 import binding as B

    B.lib()
    shape = shape_for(args)
    w_np = synth.make_weights(shape.n_out, shape.k_in, seed=args.seed, key=shape.key)
    w = torch.from_numpy(w_np.view(np.int16).copy()).cuda()
    frac = shape.density if shape.density > 0 else 0.0045
    steps, warmup = max(1, min(args.steps, 20)), max(3, min(args.warmup, 5))
    for _ in range(warmup):
        out = B.sqz_encode(w, shape.bits, frac, args.encode_iters, want_iters=True)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        out = B.sqz_encode(w, shape.bits, frac, args.encode_iters, want_iters=True)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    iters = out[5].cpu().numpy()
    n_w = shape.n_out * shape.k_in
    line = {"metric": "encoder weights per second (Dense-and-Sparse split + per-row k-means)",
            "value": n_w / (ms * 1e-3), "unit": "weights/s", "n_gpus": 1, "steps": steps, "warmup": warmup,
            "ms_per_layer": ms, "higher_is_better": True, "dtype": "fp16 in, fp64 k-means, exact integer sums",
            "data": "synthetic (0.02 x Student-t(4) weights)",
            "config": {"workload": f"{shape.n_out}x{shape.k_in}, {shape.bits}-bit, outlier fraction {frac}",
                       "kmeans_iters": args.encode_iters, "iters_mean": float(iters.mean()),
                       "rows_at_iteration_limit": float((iters == args.encode_iters).mean())}}
    if not args.no_cpu_baseline:
        import oracle

        orc = oracle.default()
        w2 = w_np.reshape(shape.n_out, shape.k_in)
        m = orc.outliers_per_tail(w2.size, frac)
        t0 = time.perf_counter()
        marks = orc.select_outliers(w2, m)
        t_split = time.perf_counter() - t0
        n_rows = 8
        dense = np.where(marks[:n_rows] != 0, 0.0, w2[:n_rows].view(np.float16).astype(np.float64))
        t0 = time.perf_counter()
        for r in range(n_rows):
            orc.kmeans_row(dense[r], 1 << shape.bits, args.encode_iters)
        t_rows = (time.perf_counter() - t0) / n_rows
        t_layer = t_split + t_rows * shape.n_out
        line["cpu_baseline"] = {"value": n_w / t_layer, "unit": "weights/s", "cores": 1, "kind": "oracle",
                                "sample": f"outlier split of the whole layer ({t_split:.1f} s) plus the k-means "
                                          f"of 8 rows, scaled to {shape.n_out} rows ({t_layer:.0f} s per layer)"}
    print(json.dumps(line), flush=True)
    return 0


def free_port() -> int:
    import socket

    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def spawn_ranks(args) -> int:
    """`--gpus N` outside torchrun: start N ranks of this script (one GPU
    each; independent replicas) through torch.distributed.run on this node
    and return its exit status.  Refuses when fewer than N GPUs are visible."""
    import subprocess

    if not args.selftest_ranks:
        import torch

        have = torch.cuda.device_count()
        if have < args.gpus:
            print(f"bench.py: --gpus {args.gpus} but only {have} CUDA device(s) are visible", file=sys.stderr)
            return 2
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", f"--master-port={free_port()}", os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def run_selftest(args):
    """Rank plumbing without a GPU: gloo ranks, rank r reports 10*(r+1) ms;
    rank 0 prints the slowest rank's time, the world size and the whole-job
    value exactly as the GPU arm computes them."""
    import datetime

    import torch.distributed as dist

    world, rank, _ = dist_env()
    if world > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    ms = max_over_ranks(10.0 * (rank + 1), world)
    if rank == 0:
        print(json.dumps({"n_gpus": world, "ms": ms, "value": whole_job_gbs(world, 1_000_000, args.steps, ms),
                          "steps": args.steps}), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return spawn_ranks(args)
    if args.selftest_ranks:
        return run_selftest(args)
    if args.encode:
        return run_encode(args)
    if args.profile_launches:
        return run_profile_launches(args)
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
