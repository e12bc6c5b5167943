#!/usr/bin/env python
"""Throughput of the LLM.int8() forward linear layer on B200.

One step = one full forward (outlier columns, row quantisation + gathers, the
int8 tensor-core product with the fused fp16 outlier product and epilogue) over
one batch of seeded synthetic input already resident in HBM.  The default
workload is BLOOM-176B's FFN-up projection at prefill: X fp16 [8192, 14336]
with 8 outlier feature dimensions, W [57344, 14336] quantised to int8 CB/SCB.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                        [--impl ours|reference]
Under torchrun (N > 1) every rank runs an independent problem of the same
shape (weak scaling; no data-path collective); the reported time is the max
over ranks and the value is the work of all ranks divided by it.
``--impl reference`` times the CPU oracle (the plain C++ restatement of the
method, one thread per core) on a bounded sample of the same workload.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from int8_mixed_precision_column_b200 import workloads  # noqa: E402

METRIC = "int8-decomposed linear TOPS & tokens/s at BLOOM shapes; % of int8 TC peak / HBM"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
INT8_PER_BF16 = 2.0  # nominal dense int8 : bf16 tensor throughput on B200 (4.5 : 2.25 POPS)

WORKLOADS = {
    "toy": lambda dev, seed: workloads.toy(seed=seed, device=dev),
    "bloom176b_ffn_up_prefill": lambda dev, seed: workloads.bloom_ffn_up_prefill(8192, seed=seed, device=dev),
    "bloom176b_ffn_up_prefill_T1024": lambda dev, seed: workloads.bloom_ffn_up_prefill(1024, seed=seed, device=dev),
    "llama7b_prefill": lambda dev, seed: workloads.llama7b_prefill(seed=seed, device=dev),
    "bloom176b_ffn_up_decode_T1": lambda dev, seed: workloads.bloom_ffn_up_decode(1, seed=seed, device=dev),
    "bloom176b_ffn_up_decode_T4": lambda dev, seed: workloads.bloom_ffn_up_decode(4, seed=seed, device=dev),
    "bloom176b_ffn_up_decode_T16": lambda dev, seed: workloads.bloom_ffn_up_decode(16, seed=seed, device=dev),
    "density_sweep_nout0": lambda dev, seed: workloads.density_sweep(0, seed=seed, device=dev),
    "density_sweep_nout8": lambda dev, seed: workloads.density_sweep(8, seed=seed, device=dev),
    "density_sweep_nout64": lambda dev, seed: workloads.density_sweep(64, seed=seed, device=dev),
    "density_sweep_nout512": lambda dev, seed: workloads.density_sweep(512, seed=seed, device=dev),
    "density_sweep_nout8_thr0": lambda dev, seed: workloads.density_sweep(8, threshold=0.0, seed=seed, device=dev),
    "density_sweep_nout8_thr0.1": lambda dev, seed: workloads.density_sweep(8, threshold=0.1, seed=seed,
                                                                            device=dev),
}
DEFAULT_WORKLOAD = "bloom176b_ffn_up_prefill"


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def load_peaks() -> tuple[dict, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# Kernel source files each measured kernel is built from: a DRAM-traffic figure
# recorded in profiles/traffic.json is reported only while these are unchanged.
KERNEL_SOURCES = {
    "gemm_i8_tc2_kernel": ["gemm_tc2.cu", "common.cuh", "kernels.h"],
    "gemm_i8_tc_kernel": ["gemm_tc.cu", "common.cuh", "kernels.h"],
    "gemv_i8_decode_kernel": ["gemv_decode.cu", "common.cuh", "kernels.h"],
}


def kernel_source_hash(kernel: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "int8_mixed_precision_column_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic(kernel: str, workload: str) -> tuple[float | None, str]:
    """DRAM bytes per launch from an ncu capture committed under profiles/, or None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None, "no capture recorded"
    with open(path) as f:
        rec = json.load(f).get(kernel, {}).get(workload)
    if rec is None:
        return None, "no capture for this kernel and workload"
    if rec.get("source_sha256") != kernel_source_hash(kernel):
        return None, "kernel changed since the capture"
    return float(rec["dram_bytes_per_launch"]), rec.get("command", "")


def dist_env() -> tuple[int, int, int]:
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def reduce_max(v: float, world: int, device) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def ensure_library(world: int, local_rank: int) -> None:
    """Build the library if it is stale, on local rank 0 only; the other ranks
    wait at a barrier and then load the finished file."""
    from int8_mixed_precision_column_b200 import build, native

    if world == 1 or local_rank == 0:
        build.build()
    barrier(world)
    native.lib()


def rank_seed(rank: int) -> int:
    """Each rank draws its own independent problem (weak scaling)."""
    return 1000 * rank


def whole_job(ops_per_rank: float, tokens_per_rank: int, world: int, ms_per_step_max: float) -> tuple[float, float]:
    """(TOPS, tokens/s) of all ranks together, timed by the slowest rank."""
    sec = ms_per_step_max * 1e-3
    return ops_per_rank * world / sec / 1e12, tokens_per_rank * world / sec


def algorithmic_work(T: int, K: int, N: int, n_out: int) -> dict:
    """Ops and bytes one forward must do, independent of the implementation."""
    return {
        "int8_ops": 2.0 * T * N * K,
        "fp16_flops": 2.0 * T * N * n_out,
        # HBM bytes of the product kernel: CB once, X codes once, Y once, scales, bias
        "product_bytes": float(N * K + T * K + 2 * T * N + 4 * N + 2 * N + 4 * T + 2 * T * n_out
                               + 2 * N * n_out),
    }


def pci_bus_id(dev) -> str | None:
    """nvidia-smi style bus id ("00000000:1B:00.0") of a torch device, if torch exposes it."""
    pr = torch.cuda.get_device_properties(dev)
    try:
        return f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
    except AttributeError:
        return None


class ClockSampler:
    """nvidia-smi clocks/throttle sampling during the timed region (rank 0's GPU)."""

    FIELDS = ("timestamp,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = (bus_id or "").lower()
        self.proc = None
        self.path = None
        self.t0 = self.t1 = 0.0

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def mark_begin(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                rows.append(parts)
        os.unlink(self.path)
        mine = [r for r in rows if self.bus_id and r[1].lower()[-12:] == self.bus_id[-12:]] or rows

        def ts(r):
            try:
                return time.mktime(time.strptime(r[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
            except ValueError:
                return None

        window = [r for r in mine if ts(r) is not None and self.t0 - 1.0 <= ts(r) <= self.t1 + 1.0] or mine
        sm = [float(r[2]) for r in window if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in window if r[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in window for n, v in zip(names, r[6:10]) if v.lower() == "active"})
        pw = [float(r[4]) for r in window if r[4].replace(".", "").isdigit()]
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(window), "power_w_max": max(pw) if pw else None}


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------

def run_sharded(args, rank, world, local_rank) -> dict | None:
    """One layer split along N over the ranks (strong scaling: the total work
    is the one layer), Y assembled on every rank by the product kernels'
    stores into every rank's symmetric output buffer."""
    from int8_mixed_precision_column_b200 import native, sharded

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    ensure_library(world, local_rank)
    p = WORKLOADS[args.workload]("cuda", rank_seed(0))  # the same layer and batch on every rank
    if args.threshold is not None:
        p.threshold = args.threshold
    T, K, N = p.T, p.K, p.N
    CB, SCB = native.int8_quantize_weight(p.W)
    del p.W
    layer = sharded.NShardedLinear(CB, SCB, p.bias, T_max=T, mode="peer")
    del CB, SCB
    torch.cuda.empty_cache()
    X = p.X
    for _ in range(args.warmup):
        layer.forward(X, p.threshold)
    torch.cuda.synchronize()
    st, where = layer.check_status()
    if st != 0:
        raise RuntimeError(f"device status {native.int8_status_string(st)} at {where:#x}")
    sampler = ClockSampler(pci_bus_id(dev))
    if rank == 0:
        sampler.start()
        time.sleep(1.0)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    sampler.mark_begin()
    e0.record()
    for _ in range(args.steps):
        layer.forward(X, p.threshold)
    e1.record()
    torch.cuda.synchronize()
    sampler.mark_end()
    barrier(world)
    clocks = sampler.stop() if rank == 0 else None
    st, where = layer.check_status()
    if st != 0:
        raise RuntimeError(f"device status {native.int8_status_string(st)} at {where:#x}")
    ms = reduce_max(e0.elapsed_time(e1) / args.steps, world, dev)
    n_outliers = int(layer.n_out.item())
    if rank != 0:
        return None
    ops = 2.0 * T * N * K
    peaks, peak_src = load_peaks()
    per_rank_ops = ops / world
    achieved = per_rank_ops / (ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"] * INT8_PER_BF16
    return {
        "metric": METRIC, "value": ops / (ms * 1e-3) / 1e12, "unit": "TOPS", "tokens_per_s": T / (ms * 1e-3),
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": "int8 x int8 -> int32 (+ fp16 outlier product, fp32 accumulate), fp16 in/out",
        "data": "synthetic (seeded; X ~ N(0,1) with planted outlier columns, W ~ N(0, 0.02^2))",
        "config": {"workload": args.workload, "T": T, "K": K, "N": N, "threshold": p.threshold,
                   "n_out": n_outliers, "parallelism": f"N-sharded x{world}, Y gathered by peer stores",
                   "l2": "inputs larger than L2 (no flush)" if T * K * 3 + N * K // world > 2 * L2_BYTES
                   else "L2 not flushed (working set below 2 x L2)"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TOPS", "frac": achieved / peak,
                     "traffic": None, "traffic_source": "whole sharded forward per rank (3 kernels + 2 barriers)",
                     "kernel": "whole forward", "peak_source": f"{peak_src} bf16_tflops (burst) x {INT8_PER_BF16}"},
        "gpu_launches": (2 if T <= 16 else (3 if p.threshold > 0 else 2)) * args.steps,
        "clocks": clocks, "e2e": None, "device": torch.cuda.get_device_name(dev),
    }


def run_e2e(args, X, CB, SCB, bias, threshold, T, K, N, world, dev) -> dict:
    """The metric end to end through the library's host-buffer calls.

    Every step copies its X from pinned host memory, runs the forward and
    copies Y, idx and n_out back.  Two forms: the blocking call
    (int8_linear_forward_host, one step at a time) and the non-blocking one
    (int8_linear_forward_host_async) alternating between two streams and two
    workspaces, so one step's Y download overlaps the next step's X upload
    and kernels.  The pipelined form is the reported value.
    """
    from int8_mixed_precision_column_b200 import native

    Xh = X.cpu().pin_memory()
    nbytes = native.int8_linear_forward_host_workspace_bytes(T, K, N)
    slots = []
    for _ in range(2):
        slots.append({"stream": torch.cuda.Stream(dev),
                      "ws": torch.empty(nbytes, dtype=torch.uint8, device=dev),
                      "Y": torch.empty((T, N), dtype=X.dtype).pin_memory(),
                      "idx": torch.empty((K,), dtype=torch.int32).pin_memory(),
                      "n": torch.empty((1,), dtype=torch.int32).pin_memory()})
    ne = max(3, min(args.steps, 20))
    s0 = slots[0]

    def blocking():
        native.int8_linear_forward_host(Xh, CB, SCB, bias, threshold, s0["Y"], s0["ws"], s0["idx"], s0["n"])

    for _ in range(min(args.warmup, 3)):
        blocking()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(ne):
        blocking()
    e1.record()
    torch.cuda.synchronize()
    barrier(world)
    blocking_ms = reduce_max(e0.elapsed_time(e1) / ne, world, dev)

    main = torch.cuda.current_stream(dev)

    def pipelined(n):
        start, ends = torch.cuda.Event(enable_timing=True), []
        start.record(main)
        for sl in slots:
            sl["stream"].wait_event(start)
        for i in range(n):
            sl = slots[i % 2]
            native.int8_linear_forward_host_async(Xh, CB, SCB, bias, threshold, sl["Y"], sl["ws"], sl["idx"],
                                                  sl["n"], stream=sl["stream"])
        for sl in slots:
            ev = torch.cuda.Event()
            ev.record(sl["stream"])
            main.wait_event(ev)
        end = torch.cuda.Event(enable_timing=True)
        end.record(main)
        return start, end

    pipelined(min(args.warmup, 3) + 1)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    start, end = pipelined(ne)
    torch.cuda.synchronize()
    barrier(world)
    for sl in slots:
        st, where = native.int8_check_status(sl["ws"])
        if st != 0:
            raise RuntimeError(f"device status {native.int8_status_string(st)} at {where:#x}")
    e2e_ms = reduce_max(start.elapsed_time(end) / ne, world, dev)
    return {"value": whole_job(2.0 * T * N * K, T, world, e2e_ms)[0], "unit": "TOPS",
            "ms_per_step": e2e_ms, "steps": ne,
            "h2d_bytes_per_step": T * K * 2,
            "d2h_bytes_per_step": T * N * 2 + K * 4 + 4,
            "api": "int8_linear_forward_host_async on 2 streams (pinned host X/Y, resident CB/SCB)",
            "blocking": {"value": whole_job(2.0 * T * N * K, T, world, blocking_ms)[0], "ms_per_step": blocking_ms,
                         "api": "int8_linear_forward_host (one step at a time)"}}


DECODE_TOKENS = (1, 4, 16)


def run_decode_lines(args, rank, world, dev) -> dict:
    """The HBM-bound half of the metric: BLOOM-176B FFN-up decode forwards
    (X [T, 14336] with 8 outlier dims, W [57344, 14336] as int8 CB/SCB) for
    T in 1, 4, 16, each timed like the headline workload: CB (822 MB) is
    larger than L2, so steps run back to back without a flush (a flush by
    writing a scratch buffer would leave L2 full of dirty lines that the next
    step has to write back), timed by CUDA events around all steps, max over
    ranks."""
    from int8_mixed_precision_column_b200 import native

    peaks, peak_src = load_peaks()
    lines = {}
    sampler = ClockSampler(pci_bus_id(dev))
    if rank == 0:
        sampler.start()
        time.sleep(0.5)
    sampler.mark_begin()
    for T in DECODE_TOKENS:
        p = workloads.bloom_ffn_up_decode(T, seed=rank_seed(rank), device="cuda")
        K, N = p.K, p.N
        CB, SCB = native.int8_quantize_weight(p.W)
        del p.W
        X, bias = p.X, p.bias
        Y = torch.empty((T, N), dtype=torch.float16, device=dev)
        idx = torch.empty((K,), dtype=torch.int32, device=dev)
        n_out = torch.empty((1,), dtype=torch.int32, device=dev)
        ws = native.new_workspace(T, K, N, dev)
        for _ in range(args.warmup):
            native.int8_linear_forward(X, CB, SCB, bias, p.threshold, Y=Y, idx=idx, n_out=n_out, workspace=ws)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        torch.cuda.synchronize()
        e0.record()
        for i in range(args.steps):
            native.int8_linear_forward(X, CB, SCB, bias, p.threshold, Y=Y, idx=idx, n_out=n_out, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        barrier(world)
        st, where = native.int8_check_status(ws)
        if st != 0:
            raise RuntimeError(f"device status {native.int8_status_string(st)} at {where:#x}")
        ms = reduce_max(e0.elapsed_time(e1) / args.steps, world, dev)
        nstage = max(3, min(args.steps, 20))
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(nstage)]
        for row in ev:
            for e in row:
                e.record()
        for i in range(nstage):
            native.int8_linear_forward_timed(X, CB, SCB, bias, p.threshold, Y, idx, n_out, ws, ev[i])
        torch.cuda.synchronize()
        prep_ms = reduce_max(statistics.mean(e[0].elapsed_time(e[2]) for e in ev), world, dev)
        prod_ms = reduce_max(statistics.mean(e[2].elapsed_time(e[3]) for e in ev), world, dev)
        n_o = int(n_out.item())
        work = algorithmic_work(T, K, N, n_o)
        step_gbs = work["product_bytes"] / (ms * 1e-3) / 1e9
        prod_gbs = work["product_bytes"] / (prod_ms * 1e-3) / 1e9
        lines[f"T{T}"] = {
            "workload": f"bloom176b_ffn_up_decode_T{T}", "T": T, "K": K, "N": N, "n_out": n_o,
            "ms_per_step": ms, "tokens_per_s": T * world / (ms * 1e-3),
            "TOPS": work["int8_ops"] * world / (ms * 1e-3) / 1e12,
            "algorithmic_bytes_per_step": work["product_bytes"],
            "GBps": step_gbs, "frac_of_hbm": step_gbs / peaks["hbm_gbs"],
            "stage_ms": {"prep": prep_ms, "product": prod_ms},
            "product_kernel": {"kernel": "gemv_i8_decode_kernel", "GBps": prod_gbs,
                               "frac_of_hbm": prod_gbs / peaks["hbm_gbs"]},
        }
        del CB, SCB, X, Y, ws, p
        torch.cuda.empty_cache()
    sampler.mark_end()
    clocks = sampler.stop() if rank == 0 else None
    return {"note": "BLOOM-176B FFN-up decode, whole forward (one-kernel prep + weight-streaming GEMV) per step; "
                    "bytes = CB + SCB + bias + X codes + Y (the algorithmic HBM traffic); inputs larger than L2 "
                    "(no flush); stage_ms from a separate pass with events between the kernels",
            "peak": peaks["hbm_gbs"], "peak_source": f"{peak_src} hbm_gbs (copy)", "lines": lines,
            "clocks": clocks}


def run_ours(args, rank, world, local_rank) -> dict | None:
    from int8_mixed_precision_column_b200 import native

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    ensure_library(world, local_rank)
    p = WORKLOADS[args.workload]("cuda", rank_seed(rank))
    if args.threshold is not None:
        p.threshold = args.threshold
    T, K, N = p.T, p.K, p.N
    cpu_sample = sample_problem(p, 256, 4096) if (world == 1 and not args.no_cpu_baseline) else None
    elem = torch.bfloat16 if args.dtype == "bf16" else torch.float16
    if elem != torch.float16:
        # the same seeded problem, rounded to bf16 (X, W, bias)
        p.X, p.W = p.X.to(elem), p.W.to(elem)
        p.bias = None if p.bias is None else p.bias.to(elem)
        cpu_sample = None
    bias = p.bias
    CB, SCB = native.int8_quantize_weight(p.W)
    del p.W
    torch.cuda.empty_cache()
    X = p.X
    Y = torch.empty((T, N), dtype=elem, device=dev)
    idx = torch.empty((K,), dtype=torch.int32, device=dev)
    n_out = torch.empty((1,), dtype=torch.int32, device=dev)
    ws = native.new_workspace(T, K, N, dev)
    working_set = T * K * 3 + N * K + T * N * 2
    flush = working_set < 2 * L2_BYTES
    # L2 flush between steps: write a buffer twice the size of L2, then read
    # another one, so that L2 holds clean lines of neither the workload nor
    # the flush (dirty flush lines would be written back during the timed step)
    scrub = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=dev) if flush else None
    scrub_ro = torch.ones(2 * L2_BYTES // 4, dtype=torch.int32, device=dev) if flush else None

    def flush_l2():
        scrub.add_(1)
        scrub_ro.sum()

    nsteps = args.steps
    # Steps are timed as plain forwards (the kernels chain by programmatic
    # launch); the per-stage breakdown and the product kernel's duration come
    # from a separate pass of int8_linear_forward_timed, whose stage events
    # sit between the kernels.
    nstage = max(3, min(nsteps, 20))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(nstage)]
    for row in ev:
        for e in row:
            e.record()
    bounds = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(nsteps)]
    outer = [torch.cuda.Event(enable_timing=True) for _ in range(2)]

    def step():
        native.int8_linear_forward(X, CB, SCB, bias, p.threshold, Y=Y, idx=idx, n_out=n_out, workspace=ws,
                                   path=args.path)

    for i in range(args.warmup):
        if flush:
            flush_l2()
        step()
    torch.cuda.synchronize()
    st, where = native.int8_check_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {native.int8_status_string(st)} at {where:#x}")
    n_outliers = int(n_out.item())

    sampler = ClockSampler(pci_bus_id(dev))
    if rank == 0:
        sampler.start()
        time.sleep(1.0)
    barrier(world)
    torch.cuda.synchronize()
    sampler.mark_begin()
    # With a flush, each step is bracketed by its own events (the flush stays
    # outside them); without one, steps run back to back between the outer
    # events only.
    outer[0].record()
    for i in range(nsteps):
        if flush:
            flush_l2()
            bounds[i][0].record()
        step()
        if flush:
            bounds[i][1].record()
    outer[1].record()
    torch.cuda.synchronize()
    sampler.mark_end()
    barrier(world)
    clocks = sampler.stop() if rank == 0 else None
    st, where = native.int8_check_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {native.int8_status_string(st)} at {where:#x}")
    total_ms = sum(bounds[i][0].elapsed_time(bounds[i][1]) for i in range(nsteps)) if flush else \
        outer[0].elapsed_time(outer[1])
    ms_per_step = reduce_max(total_ms / nsteps, world, dev)

    for i in range(nstage):
        if flush:
            flush_l2()
        native.int8_linear_forward_timed(X, CB, SCB, bias, p.threshold, Y, idx, n_out, ws, ev[i], path=args.path)
    torch.cuda.synchronize()
    st, where = native.int8_check_status(ws)
    if st != 0:
        raise RuntimeError(f"device status {native.int8_status_string(st)} at {where:#x}")
    prod_ms = [ev[i][2].elapsed_time(ev[i][3]) for i in range(nstage)]
    outl_ms = [ev[i][0].elapsed_time(ev[i][1]) for i in range(nstage)]
    rowq_ms = [ev[i][1].elapsed_time(ev[i][2]) for i in range(nstage)]

    # end to end through the host-buffer entry points: pinned X in, Y/idx/n_out out, every step
    e2e = None
    if not args.no_e2e and elem == torch.float16:  # the blocking host entry point takes fp16
        ws = None
        torch.cuda.empty_cache()
        e2e = run_e2e(args, X, CB, SCB, bias, p.threshold, T, K, N, world, dev)

    decode_lines = None
    if args.workload == DEFAULT_WORKLOAD and not args.no_decode and elem == torch.float16:
        # the headline workload's buffers are released before the decode layers are built
        X = Y = idx = n_out = CB = SCB = scrub = scrub_ro = ws = bias = None
        p.X = p.bias = None
        torch.cuda.empty_cache()
        decode_lines = run_decode_lines(args, rank, world, dev)

    if rank != 0:
        return None
    work = algorithmic_work(T, K, N, n_outliers)
    peaks, peak_src = load_peaks()
    prod_avg = statistics.mean(prod_ms)
    product = native.int8_linear_product_kernel(T, K, N, args.path)  # the kernel the forward ran
    decode = product == native.PATH_DECODE
    traffic_key = args.workload if elem == torch.float16 else f"{args.workload}_bf16"
    if decode:
        achieved = work["product_bytes"] / (prod_avg * 1e-3) / 1e9
        traffic, traffic_src = recorded_traffic("gemv_i8_decode_kernel", traffic_key)
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "traffic_source": traffic_src,
                "kernel": "gemv_i8_decode_kernel",
                "peak_source": f"{peak_src} hbm_gbs (copy)",
                "algorithmic_bytes_per_launch": work["product_bytes"], "ms_per_launch": prod_avg}
    else:
        # combined roofline: the 16-bit outlier product runs at the bf16 peak,
        # i.e. one of its flops costs INT8_PER_BF16 int8 ops of tensor time
        peak = peaks["bf16_tflops"] * INT8_PER_BF16
        equiv_ops = work["int8_ops"] + INT8_PER_BF16 * work["fp16_flops"]
        achieved = equiv_ops / (prod_avg * 1e-3) / 1e12
        kname = "gemm_i8_tc_kernel" if product == native.PATH_TENSOR_CORE_1SM else "gemm_i8_tc2_kernel"
        traffic, traffic_src = recorded_traffic(kname, traffic_key)
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TOPS",
                "frac": achieved / peak, "traffic": traffic, "traffic_source": traffic_src,
                "algorithmic_bytes_per_launch": work["product_bytes"],
                "kernel": kname,
                "peak_source": f"{peak_src} bf16_tflops (burst) x {INT8_PER_BF16} nominal int8:bf16 ratio",
                "algorithmic_ops_per_launch": work["int8_ops"], "fp16_flops_per_launch": work["fp16_flops"],
                "achieved_counts": "int8 ops + 2 x 16-bit outlier flops (int8-equivalent tensor work)",
                "ms_per_launch": prod_avg}
    # kernels per forward: decode = the one-kernel prep + the GEMV; otherwise
    # outlier pass (only with a threshold) + row quantisation + product
    launches_per_step = 2 if decode else (3 if p.threshold > 0 else 2)
    tops, tok_s = whole_job(work["int8_ops"], T, world, ms_per_step)
    out = {
        "metric": METRIC,
        "value": tops,
        "unit": "TOPS",
        "tokens_per_s": tok_s,
        "n_gpus": world,
        "steps": nsteps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": f"int8 x int8 -> int32 (+ {args.dtype} outlier product, fp32 accumulate), {args.dtype} in/out",
        "data": "synthetic (seeded; X ~ N(0,1) with planted outlier columns, W ~ N(0, 0.02^2))",
        "config": {"workload": args.workload, "T": T, "K": K, "N": N, "threshold": p.threshold, "path": args.path,
                   "elem": args.dtype,
                   "n_out": n_outliers, "parallelism": f"independent problem per rank x{world}",
                   "l2": ("L2 flushed between steps (write 252 MB, then read 252 MB)" if flush
                          else "inputs larger than L2 (no flush)")},
        "stage_ms_note": "per-stage CUDA events from a separate pass with events between the kernels "
                         "(no programmatic overlap there); value and ms_per_step time plain forwards",
        "stage_ms": {"outliers": statistics.mean(outl_ms), "rowquant": statistics.mean(rowq_ms),
                     "product": prod_avg},
        "roofline": roof,
        "gpu_launches": launches_per_step * nsteps,
        "clocks": clocks,
        "e2e": e2e,
        "device": torch.cuda.get_device_name(dev),
    }
    if decode_lines is not None:
        out["decode"] = decode_lines
    if cpu_sample is not None:
        out["cpu_baseline"] = cpu_baseline(cpu_sample, p.threshold, seconds=args.cpu_seconds)
    return out


# ---------------------------------------------------------------------------
# CPU oracle baseline / reference arm
# ---------------------------------------------------------------------------

def sample_problem(p, rows: int, cols: int):
    """A sub-problem of the workload: `rows` token rows x `cols` output features."""
    gen = np.random.default_rng(1234)
    T, N = p.T, p.N
    r = np.sort(gen.choice(T, size=min(rows, T), replace=False))
    c = np.sort(gen.choice(N, size=min(cols, N), replace=False))
    X = p.X[torch.as_tensor(r, device=p.X.device)].cpu().numpy()
    W = p.W[torch.as_tensor(c, device=p.W.device)].cpu().numpy()
    b = None if p.bias is None else p.bias[torch.as_tensor(c, device=p.bias.device)].cpu().numpy()
    return X, W, b


def host_threads() -> int:
    """Cores this process may run on (the C++ oracle starts one thread per core)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpp_oracle():
    """The plain C++ oracle (oracle/llm_int8_ref.cpp), one thread per host core."""
    from oracle import cpp

    cpp.build()
    return cpp.Oracle(threads=host_threads())


def oracle_rate(X, W, b, thr, seconds: float) -> tuple[float, int, float]:
    """Run the C++ oracle's forward on (X, W) repeatedly for ~`seconds`; returns (TOPS, reps, s/rep)."""
    O = cpp_oracle()
    CB, SCB = O.quantize_weight(W)  # layer set-up, not part of a step
    T, K = X.shape
    N = W.shape[0]
    reps, t0 = 0, time.perf_counter()
    while True:
        O.linear_forward(X, CB, SCB, b, thr)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return 2.0 * T * N * K * reps / el / 1e12, reps, el / reps


def cpu_baseline(sample, threshold: float, seconds: float = 12.0) -> dict:
    X, W, b = sample
    v, reps, per = oracle_rate(X, W, b, threshold, seconds)
    return {"value": v, "unit": "TOPS", "cores": host_threads(), "kind": "oracle",
            "sample": f"full forward of the plain C++ oracle (every stage, plain loops, one thread per core) on "
                      f"{X.shape[0]} token rows x {W.shape[0]} output features of the workload (K={X.shape[1]}), "
                      f"repeated {reps}x ({per:.2f} s each)"}


def run_reference(args, rank, world, local_rank) -> dict | None:
    if rank != 0:
        return None
    p = WORKLOADS[args.workload]("cpu", 0)
    T, K, N = p.T, p.K, p.N
    X, W, b = sample_problem(p, rows=64, cols=2048)
    O = cpp_oracle()
    CB, SCB = O.quantize_weight(W)
    for _ in range(args.warmup):
        O.linear_forward(X, CB, SCB, b, p.threshold)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        O.linear_forward(X, CB, SCB, b, p.threshold)
    el = time.perf_counter() - t0
    ms = el / args.steps * 1e3
    ops = 2.0 * X.shape[0] * W.shape[0] * K
    v = ops / (ms * 1e-3) / 1e12
    sample = (f"plain C++ oracle forward on {X.shape[0]} token rows x {W.shape[0]} output features of the "
              f"workload (T={T}, K={K}, N={N}) per step")
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "TOPS",
            "tokens_per_s": X.shape[0] / (ms * 1e-3), "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8 codes, int64 dot products, fp64 reference arithmetic (plain C++)",
            "data": "synthetic (seeded)",
            "config": {"workload": args.workload, "T": T, "K": K, "N": N, "threshold": p.threshold},
            "cpu_baseline": {"value": v, "unit": "TOPS", "cores": host_threads(), "kind": "oracle", "sample": sample},
            "e2e": {"value": v, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------

def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=60)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--threshold", type=float, default=None,
                    help="override the workload's outlier threshold (<= 0 switches the decomposition off)")
    ap.add_argument("--path", type=int, default=0, choices=[0, 1, 2, 3],
                    help="product kernel: 0 auto, 1 tensor core (SM pairs), 2 decode GEMV, 3 tensor core (single SM)")
    ap.add_argument("--dtype", default="fp16", choices=["fp16", "bf16"],
                    help="16-bit element type of X, bias, Y and the outlier product")
    ap.add_argument("--shard-n", action="store_true",
                    help="split one layer along N over the ranks (strong scaling; Y gathered by peer stores)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the BLOOM FFN-up decode lines the default workload's line carries")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local_rank = dist_env()
    if args.impl == "reference":
        out = run_reference(args, rank, world, local_rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    pg = world > 1 or args.shard_n
    if pg:
        import datetime
        import socket
        import torch.distributed as dist
        if world == 1:
            with socket.socket() as sk:
                sk.bind(("127.0.0.1", 0))
                os.environ.setdefault("MASTER_PORT", str(sk.getsockname()[1]))
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        out = run_sharded(args, rank, world, local_rank) if args.shard_n else run_ours(args, rank, world, local_rank)
        if out is not None:
            print(json.dumps(out), flush=True)
    finally:
        if pg:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
