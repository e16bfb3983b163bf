#!/usr/bin/env python
"""Benchmark of the fused EQ-Linear forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl eqlin|reference]

One step = one eqlin_forward over the whole batch of the headline workload (p4,
Cin = Cout = 96, N = 64*56*56 tokens, bf16 I/O): weights prepared once, outside the
timed region; inputs already resident in HBM.  Prints ONE JSON line (rank 0):
tokens/s over all ranks, ms per step, the roofline of the fused kernel (algorithmic
bytes / HBM peak, Fourier FLOPs / bf16 tensor peak), clocks sampled during the timed
region, an end-to-end figure through the host-buffer API, and the CPU float64
oracle's throughput on a bounded sample.

The same line carries a ``workloads`` object with every synthetic workload
(tiny p4 fp32, p4 C96, p8 C64, p4 MLP 192->768, C16 C32), each measured in this run
the same way: us per launch over back-to-back launches, tokens/s, roofline,
dense-equivalent TFLOP/s, the backward calls, the MLP block, the pages' dense
baseline as context (one cuBLAS GEMM on the replicated group-circulant weight), and
the oracle on a bounded sample of that workload.  The headline runs first, then the
other workloads.

Multi-GPU (torchrun): every rank runs the full workload on its own GPU (tokens
are independent, no collective on the data path): weak scaling; the timed
region is bracketed by barriers and the slowest rank's time is used.

--impl reference times the float64 CPU oracle on the host cores instead (the
method's plain definition), on bounded token samples of the same workload.  That
arm never loads the CUDA library.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

# the package loads libeqlin.so lazily: importing the input generators maps no CUDA code
from cyclic_group_dft_b200 import workloads  # noqa: E402

METRIC = "EQ-Linear tokens/s and % of roofline (HBM vs bf16 TC), p4 Cin=Cout=96"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024
# the synthetic workloads of the method's configurations, measured in every run
BENCH_WORKLOADS = ("tiny_p4_fp32", "p4_c96_bf16", "p8_c64_bf16", "p4_mlp_bf16", "c16_c32_bf16")
# device code of each fused kernel: a recorded ncu traffic figure is reported only
# while these files are unchanged since the capture
KERNEL_SOURCES = {
    "eqlin_fwd_tc": ["eqlin_fwd_tc.cuh", "group_dft.cuh", "io16.cuh", "sm100_ptx.cuh", "eqlin_layout.h"],
    "eqlin_fwd_tm": ["eqlin_fwd_tm.cuh", "eqlin_fwd_tc.cuh", "group_dft.cuh", "io16.cuh", "sm100_ptx.cuh",
                     "eqlin_layout.h"],
    "eqlin_fwd_tcr": ["eqlin_fwd_tcr.cuh", "eqlin_fwd_tc.cuh", "group_dft.cuh", "io16.cuh", "sm100_ptx.cuh",
                      "eqlin_layout.h"],
}
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "eqlin_fwd_traffic.json")

# NVML clock-event reason bits
REASON_BITS = {
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
    0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
    0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


# ------------------------------------------------------------------ cost model
def algorithmic_bytes(wl: workloads.Workload, N: int) -> int:
    """Read x once, write y once, read the frequency-domain weights (G*Cin*Cout
    values in the I/O dtype) and the fp32 bias once."""
    e = wl.elem_bytes
    bias = 4 * wl.Cout if wl.bias_var is not None else 0
    return N * wl.Cin * wl.G * e + N * wl.Cout * wl.G * e + wl.G * wl.Cin * wl.Cout * e + bias


def backward_bytes(wl: workloads.Workload, N: int) -> dict:
    """Algorithmic bytes of the two backward calls.  Input gradient: read dy once,
    write dx once, read its weights once.  Weight gradient: read x and dy once,
    write dw and dbias once (fp32)."""
    e = wl.elem_bytes
    act = N * (wl.Cin + wl.Cout) * wl.G * e
    return {"dx": act + wl.G * wl.Cin * wl.Cout * e,
            "dw": act + 4 * (wl.G * wl.Cin * wl.Cout + wl.Cout)}


def fourier_flops(wl: workloads.Workload, N: int) -> int:
    """Per-frequency real products: 2 real + 4 per complex frequency = 2G-2 blocks."""
    return 2 * N * wl.Cin * wl.Cout * (2 * wl.G - 2)


def dense_equivalent_flops(wl: workloads.Workload, N: int) -> int:
    return 2 * N * (wl.Cout * wl.G) * (wl.Cin * wl.G)


def load_peaks() -> tuple[dict, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "cyclic_group_dft_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload: str) -> dict | None:
    """DRAM reads plus L2 write bytes per launch from a committed ncu capture, if the
    kernel is unchanged since.  Reads are counted at DRAM; writes are the sectors the SMs
    write into L2 (every byte the kernel stores), because part of y is still dirty in L2
    when the kernel ends and its DRAM write-back falls outside the kernel."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    entry = d.get(workload)
    if not entry or entry.get("kernel") not in KERNEL_SOURCES:
        return None
    if entry.get("source_hash") != kernel_source_hash(entry["kernel"]):
        return None
    if "dram_read_bytes_per_launch" not in entry or "l2_write_bytes_per_launch" not in entry:
        return None
    return {"bytes": entry["dram_read_bytes_per_launch"] + entry["l2_write_bytes_per_launch"],
            "dram_read": entry["dram_read_bytes_per_launch"], "l2_write": entry["l2_write_bytes_per_launch"],
            "kernel": entry["kernel"]}


def rotating_sets(wl: workloads.Workload, N: int) -> tuple[int, int]:
    """(bytes of one x/y set, number of sets): enough sets that consecutive launches
    never find their inputs in L2."""
    set_bytes = N * (wl.Cin + wl.Cout) * wl.G * wl.elem_bytes
    return set_bytes, max(2, math.ceil(2 * L2_BYTES / set_bytes))


def line_config(wl: workloads.Workload, world: int) -> dict:
    """The `config` of the JSON line: the workload and how it is run, identical in the
    GPU and the reference arm (kernel details are reported apart, under `kernel`)."""
    set_bytes, n_sets = rotating_sets(wl, wl.N)
    return {"workload": wl.name, "N": wl.N, "Cin": wl.Cin, "Cout": wl.Cout, "G": wl.G, "io": wl.io_dtype,
            "global_batch": world * wl.N, "parallelism": f"replicas{world}" if world > 1 else "single",
            "l2": f"inputs larger than L2; {n_sets} rotating x/y sets of {set_bytes / 1e6:.0f} MB"}


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML: every period_s in a thread
    while the timed region runs (the first one period after its start) and once right
    after it (stop).  An NVML query just before or while the kernels run slows them
    (B200, p4 C96, 20 back-to-back launches: 62.4 us per launch with 10 ms sampling from
    the start against 60.2 us without, 61.8 us with one query just before the start, still
    1 us slower with one query before the 5 warm-up launches), so a region shorter than
    one period is represented by the sample taken right after it.  Construct it (NVML
    initialisation) before the warm-up: a host delay between the warm-up and the timed
    region lets the GPU idle, and the region then starts slow (63.0 us after a 20 ms
    pause)."""

    def __init__(self, device_index: int, period_s: float = 0.05):
        self.samples: list[tuple[int, int]] = []
        self.max_mhz = None
        self.error = None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            try:
                idx = torch.cuda._get_nvml_device_index(device_index)
            except Exception:
                idx = device_index
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as exc:  # no NVML: report it, do not guess
            self._nvml = None
            self.error = f"nvml unavailable: {exc}"

    def _sample(self):
        p = self._nvml
        try:
            mhz = p.nvmlDeviceGetClockInfo(self._h, p.NVML_CLOCK_SM)
            try:
                reasons = p.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            except AttributeError:
                reasons = p.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
            self.samples.append((int(mhz), int(reasons)))
        except Exception as exc:
            self.error = str(exc)

    def _run(self):
        while not self._stop.wait(self.period):
            self._sample()

    def start(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
            self._sample()

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "error": self.error}
        mhz = [m for m, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = [name for bit, name in REASON_BITS.items() if bits & bit and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples),
                "sampling": f"NVML, every {self.period * 1e3:.0f} ms inside the timed region (the first one "
                            "period after its start) and right after it"}


# ------------------------------------------------------------------ CPU oracle
def oracle_rate(wl: workloads.Workload, target_s: float, seed: int = 0, cap_tokens: int | None = None,
                threads: int | None = None):
    """Time the float64 oracle on a token prefix sized for ~target_s seconds, on `threads`
    host threads (default: every core this process may run on).
    Returns (tokens/s, tokens, seconds, threads)."""
    import oracle
    if threads is None:
        threads = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    x, w, bias = workloads.make_inputs(wl, seed=seed, N=64)
    xf, wf = x.double().numpy(), w.double().numpy()
    bf = None if bias is None else bias.double().numpy()
    t0 = time.perf_counter()
    oracle.forward(xf, wf, bf, threads=threads)
    dt = max(time.perf_counter() - t0, 1e-6)
    per_token = dt / 64
    n = int(min(max(target_s / per_token, 64), cap_tokens or wl.N, wl.N))
    x, _, _ = workloads.make_inputs(wl, seed=seed, N=n)
    xf = x.double().numpy()
    t0 = time.perf_counter()
    oracle.forward(xf, wf, bf, threads=threads)
    dt = time.perf_counter() - t0
    return n / dt, n, dt, threads


def cpu_baseline(wl: workloads.Workload, seconds: float, single_core_seconds: float = 0.0) -> dict:
    rate, n_s, dt, threads = oracle_rate(wl, seconds)
    out = {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
           "sample": f"{n_s} of {wl.N} tokens of {wl.name} in {dt:.1f} s (float64 definition loops, "
                     f"OpenMP over tokens)"}
    if single_core_seconds > 0:
        rate1, n1, dt1, _ = oracle_rate(wl, single_core_seconds, threads=1)
        out["single_core"] = {"value": rate1, "unit": "tokens/s", "cores": 1,
                              "sample": f"{n1} of {wl.N} tokens in {dt1:.1f} s"}
    return out


# ------------------------------------------------------------------ helpers
def reduce_max(value: float, device) -> float:
    """Max of `value` over all ranks (identity without a process group).  Every rank
    must call it at the same point."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tokens_per_s(world: int, steps: int, tokens_per_rank: int, max_elapsed_ms: float) -> float:
    """Whole-job throughput: every rank processes `tokens_per_rank` tokens per step
    (replicas, weak scaling); the job takes as long as its slowest rank."""
    return world * steps * tokens_per_rank / (max_elapsed_ms / 1e3)


def dist_info():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def emit(d: dict) -> None:
    print(json.dumps(d), flush=True)


def roofline(wl: workloads.Workload, N: int, avg_launch_s: float, peaks: dict, peak_kind: str) -> dict:
    """Roofline of one launch: algorithmic bytes and Fourier FLOPs against the measured
    HBM copy peak and bf16 tensor peak; the bound is the slower of the two."""
    bytes_launch = algorithmic_bytes(wl, N)
    flops_launch = fourier_flops(wl, N)
    gbs = bytes_launch / avg_launch_s / 1e9
    tflops = flops_launch / avg_launch_s / 1e12
    t_hbm = bytes_launch / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops_launch / (peaks["bf16_tflops"] * 1e12)
    if t_hbm >= t_tc:
        roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"]}
    else:
        roof = {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": tflops / peaks["bf16_tflops"]}
    tr = recorded_traffic(wl.name) if N == wl.N else None
    roof["traffic"] = None if tr is None else tr["bytes"]
    if tr is not None:
        roof["traffic_detail"] = {"dram_read": tr["dram_read"], "l2_write": tr["l2_write"],
                                  "over_algorithmic": tr["bytes"] / bytes_launch, "kernel": tr["kernel"],
                                  "source": "ncu capture (profiles/eqlin_fwd_traffic.json): dram__bytes_read.sum "
                                            "+ 32 * lts__t_sectors_srcunit_tex_op_write.sum (bytes the SMs "
                                            "write into L2), scaled to a full launch by tokens"}
    roof["peak_source"] = f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured" else "fallback"
    roof["roofline_time_us"] = 1e6 * max(t_hbm, t_tc)
    roof["kernel_us"] = 1e6 * avg_launch_s
    roof["frac_of_roofline_time"] = max(t_hbm, t_tc) / avg_launch_s
    roof["bytes_per_launch"] = bytes_launch
    roof["fourier_flops_per_launch"] = flops_launch
    roof["tensor_tflops"] = tflops
    roof["tensor_frac"] = tflops / peaks["bf16_tflops"]                       # burst peak: the headline
    roof["tensor_frac_sustained"] = tflops / peaks["bf16_tflops_sustained"]   # seconds-long GEMM peak
    return roof


def run_reference(args, wl) -> None:
    world, rank, _ = dist_info()
    if rank != 0:
        return
    # size each step so that warmup + steps finish in about two minutes
    rate, _, _, threads = oracle_rate(wl, target_s=1.0)
    per_step_s = min(120.0 / max(args.steps + args.warmup, 1), 20.0)
    n = int(max(64, min(wl.N, rate * per_step_s)))
    import oracle
    x, w, bias = workloads.make_inputs(wl, N=n)
    xf, wf = x.double().numpy(), w.double().numpy()
    bf = None if bias is None else bias.double().numpy()
    for _ in range(args.warmup):
        oracle.forward(xf, wf, bf, threads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.forward(xf, wf, bf, threads=threads)
    dt = time.perf_counter() - t0
    value = args.steps * n / dt
    sample = (f"{n} of {wl.N} tokens of {wl.name} per step (tokens are independent: the whole batch takes "
              f"N / {n} times as long)")
    emit({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps * wl.N / n, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": line_config(wl, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    })


# ------------------------------------------------------------------ GPU arm
class Ctx:
    def __init__(self, eq, dev, world, stream, peaks, peak_kind, graph=False):
        self.eq, self.dev, self.world, self.stream = eq, dev, world, stream
        self.peaks, self.peak_kind = peaks, peak_kind
        self.graph = graph

    def barrier(self):
        if self.world > 1:
            torch.distributed.barrier()


def time_back_to_back(ctx: Ctx, fn, K: int, clocks: ClockSampler | None = None, graph: bool = True) -> float:
    """Elapsed ms (max over ranks) of K calls fn(i, stream) between two events on the
    launching stream, with no event between the calls.  With `graph`, the K calls are
    captured once into a CUDA graph and the timed region is one replay of it: the same K
    launches with their arguments, without the host's per-call cost (argument checks,
    tensor-map encoding, launch) on the critical path."""
    if graph:
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(ctx.dev)
        with torch.cuda.graph(g, stream=cap):
            for i in range(K):
                fn(i, cap)
        g.replay()                      # upload and one untimed run
        torch.cuda.synchronize(ctx.dev)
        run = g.replay
    else:
        def run():
            for i in range(K):
                fn(i, ctx.stream)
    ctx.barrier()
    torch.cuda.synchronize(ctx.dev)
    if clocks is not None:
        clocks.start()
    st = torch.cuda.current_stream(ctx.dev)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(st)
    run()
    t1.record(st)
    torch.cuda.synchronize(ctx.dev)
    if clocks is not None:
        clocks.stop()
    ctx.barrier()
    return reduce_max(t0.elapsed_time(t1), ctx.dev)


def host_link_rates(dev, x_pin, x_dev, y_dev, y_pin, N: int, reps: int = 3) -> dict:
    """The host link's own rates for the bytes e2e moves: one pinned host -> device copy of
    x, one device -> host copy of y, and both at once on two streams (the host-buffer path
    overlaps them), each the best of `reps`, from CUDA events.  `bound_tokens_per_s` is the
    e2e rate the concurrent copies alone allow."""
    main = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def timed(use_in: bool, use_out: bool) -> float:
        best = float("inf")
        for _ in range(reps):
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(main)
            for st, use, fn in ((s_in, use_in, lambda: x_dev.copy_(x_pin, non_blocking=True)),
                                (s_out, use_out, lambda: y_pin.copy_(y_dev, non_blocking=True))):
                if use:
                    st.wait_event(e0)
                    with torch.cuda.stream(st):
                        fn()
                    done = torch.cuda.Event()
                    done.record(st)
                    main.wait_event(done)
            e1.record(main)
            torch.cuda.synchronize(dev)
            best = min(best, e0.elapsed_time(e1) * 1e-3)
        return best

    bx, by = x_pin.numel() * x_pin.element_size(), y_pin.numel() * y_pin.element_size()
    t_in, t_out, t_both = timed(True, False), timed(False, True), timed(True, True)
    return {"h2d_gbs": bx / t_in / 1e9, "d2h_gbs": by / t_out / 1e9, "both_s": t_both,
            "both_gbs": (bx + by) / t_both / 1e9, "bound_tokens_per_s": N / t_both,
            "method": "pinned cudaMemcpyAsync of the step's x and y, best of 3, CUDA events"}


def setup_workload(ctx: Ctx, wl: workloads.Workload, args) -> dict:
    """Seeded inputs on the host, the prepared handle and the rotating x/y sets on the
    device (everything a workload's measurement needs, before any of it is timed)."""
    eq, dev = ctx.eq, ctx.dev
    x_cpu, w, bias = workloads.make_inputs(wl)
    h = eq.prepare(w.to(dev), None if bias is None else bias.to(dev), io_dtype=wl.torch_dtype,
                   backward=not args.no_backward)
    _, n_sets = rotating_sets(wl, wl.N)
    xs = [x_cpu.to(dev) for _ in range(n_sets)]
    ys = [torch.empty(wl.N, wl.Cout, wl.G, dtype=wl.torch_dtype, device=dev) for _ in range(n_sets)]
    return {"x_cpu": x_cpu, "w": w, "bias": bias, "h": h, "xs": xs, "ys": ys, "n_sets": n_sets}


def measure_workload(ctx: Ctx, wl: workloads.Workload, K: int, warmup: int, headline: bool, args,
                     setup: dict | None = None) -> dict:
    """One workload: K back-to-back forward launches (timed, first), a per-launch pass,
    (headline only) the end-to-end host-buffer figure and the clocks of the timed region,
    then the backward calls and the MLP block."""
    eq, dev, stream = ctx.eq, ctx.dev, ctx.stream
    su = setup if setup is not None else setup_workload(ctx, wl, args)
    x_cpu, h, xs, ys, n_sets = su["x_cpu"], su["h"], su["xs"], su["ys"], su["n_sets"]
    backward = not args.no_backward
    N = wl.N

    def fwd(i, st=stream):
        h.forward(xs[i % n_sets], out=ys[i % n_sets], stream=st)

    # The timed loop calls the C entry point eqlin_forward directly with precomputed
    # arguments (the binding's checks ran on the same tensors during the warm-up), so the
    # host reaches the first launch within microseconds of the start event.
    lib = eq.library()
    x_ptrs = [t.data_ptr() for t in xs]
    y_ptrs = [t.data_ptr() for t in ys]
    st_ptr = stream.cuda_stream
    rcs = []

    def fwd_c(i, st=None):
        rcs.append(lib.eqlin_forward(h.ptr, x_ptrs[i % n_sets], y_ptrs[i % n_sets], N,
                                     st.cuda_stream if st is not None else st_ptr))

    for i in range(warmup):
        fwd(i)
    torch.cuda.synchronize(dev)
    if h.device_status() != eq.EQLIN_OK:
        raise RuntimeError(f"{wl.name}: device status not OK after warm-up")

    out = {}
    # ------------------------------------------------------- timed region
    # First, on a GPU that this process has not yet loaded for seconds (a long load makes
    # the same launches a few percent slower): W warm-up launches and then K back-to-back
    # steps, one fused launch each, bracketed by two events on the
    # launching stream.  No event sits between the launches: an event there would end
    # the overlap of one launch's tail with the next one's prologue (programmatic
    # dependent launch), which is how the kernel runs in a real stream of layers.
    # The average launch duration of the kernel is therefore elapsed / K.
    clocks = ClockSampler(dev.index) if headline else None
    for i in range(warmup):
        fwd(i)
    elapsed_ms = time_back_to_back(ctx, fwd_c, K, clocks, graph=ctx.graph)
    if any(rc != eq.EQLIN_OK for rc in rcs):
        raise RuntimeError(f"{wl.name}: eqlin_forward returned {sorted(set(rcs))}")
    status = h.device_status()
    avg_launch_s = elapsed_ms / K / 1e3
    # with --graph, the same K launches issued one by one from the host, for comparison
    stream_ms = time_back_to_back(ctx, fwd_c, K, graph=False) if ctx.graph else elapsed_ms
    out.update({"N": N, "Cin": wl.Cin, "Cout": wl.Cout, "G": wl.G, "io": wl.io_dtype,
           "kernel": {"path": h.path, "stages": h.attr("stages"), "tokens_per_tile": h.attr("tokens_per_tile")},
           "steps": K, "elapsed_ms": elapsed_ms, "us_per_launch": 1e3 * elapsed_ms / K,
           "timing": "one CUDA-graph replay of the K launches" if ctx.graph else "K launches from the host",
           "us_per_launch_host_launches": 1e3 * stream_ms / K,
           "tokens_per_s": aggregate_tokens_per_s(ctx.world, K, N, elapsed_ms),
           "roofline": roofline(wl, N, avg_launch_s, ctx.peaks, ctx.peak_kind),
           "dense_equivalent_tflops": dense_equivalent_flops(wl, N) / avg_launch_s / 1e12,
           "device_status": status})
    if algorithmic_bytes(wl, N) / (ctx.peaks["hbm_gbs"] * 1e9) < 2e-6:
        out["roofline"]["note"] = ("launch-bound: the roofline time is below the ~2 us cost of one kernel "
                                   "launch, so the fraction measures launch latency, not the kernel's "
                                   "arithmetic or memory traffic")
    if clocks is not None:
        out["clocks"] = clocks.summary()

    # Launch-duration distribution, outside the timed region: an event pair around
    # each launch (which serialises the launches, so each one also pays its own
    # prologue and tail).
    KL = min(K, 100)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(KL)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(KL)]
    for i in range(KL):
        starts[i].record(stream)
        fwd(i)
        ends[i].record(stream)
    torch.cuda.synchronize(dev)
    launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    out["launch_us"] = {"mean": 1e3 * statistics.mean(launch_ms), "median": 1e3 * statistics.median(launch_ms),
                        "min": 1e3 * min(launch_ms), "max": 1e3 * max(launch_ms), "launches": len(launch_ms),
                        "note": "each launch bracketed by its own events (serialised), outside the timed region"}

    # ------------------------------------------------------- end to end (headline)
    if headline and args.e2e_steps > 0:
        E = args.e2e_steps
        x_pin = x_cpu.pin_memory()
        y_pin = torch.empty(N, wl.Cout, wl.G, dtype=wl.torch_dtype).pin_memory()
        h.forward_host(x_pin, y_pin)  # warm the path
        e2e_ms = time_back_to_back(ctx, lambda i, st: h.forward_host(x_pin, y_pin, stream=st), E, graph=False)
        out["e2e"] = {"value": aggregate_tokens_per_s(ctx.world, E, N, e2e_ms), "unit": "tokens/s", "steps": E,
                      "h2d_bytes_per_step": x_pin.numel() * x_pin.element_size(),
                      "d2h_bytes_per_step": y_pin.numel() * y_pin.element_size(),
                      "api": "eqlin_forward_host (C ABI: pinned host x and y, chunked copies in and out "
                             "overlapping the fused kernel on two streams)",
                      "link": host_link_rates(dev, x_pin, xs[0], ys[0], y_pin, N)}
        del x_pin, y_pin

    # ------------------------------------------------------- backward calls
    # Measured after the forward's timed region, on the same rotating buffer sets (the
    # forward outputs stand in for dy): us per call from CUDA events around Kb
    # back-to-back calls, against the same roofline model as the forward.
    if backward:
        Kb = max(10, min(max(K, 100), 200))
        dxs = [torch.empty(N, wl.Cin, wl.G, dtype=wl.torch_dtype, device=dev) for _ in range(n_sets)]
        dw_t = torch.empty(wl.Cout, wl.Cin, wl.G, dtype=torch.float32, device=dev)
        db_t = torch.empty(wl.Cout, dtype=torch.float32, device=dev)
        ws_t = torch.empty(max(16, eq.eqlin_backward_dw_workspace_size(h, N)), dtype=torch.uint8, device=dev)
        calls = {
            "dx": lambda i, st=stream: h.backward_dx(ys[i % n_sets], out=dxs[i % n_sets], stream=st),
            "dw": lambda i, st=stream: eq.eqlin_backward_dw(h, xs[i % n_sets], ys[i % n_sets], stream=st,
                                                            dw=dw_t, dbias=db_t, workspace=ws_t),
        }
        bwd = {}
        bb = backward_bytes(wl, N)
        t_tc = fourier_flops(wl, N) / (ctx.peaks["bf16_tflops"] * 1e12)
        for key, fn in calls.items():
            for i in range(max(3, warmup)):
                fn(i)
            ms = time_back_to_back(ctx, fn, Kb, graph=ctx.graph)
            t = ms / Kb * 1e-3
            t_h = bb[key] / (ctx.peaks["hbm_gbs"] * 1e9)
            t_roof = max(t_h, t_tc)
            bwd[key] = {"us_per_call": 1e6 * t, "calls": Kb, "bytes": bb[key], "roofline_time_us": 1e6 * t_roof,
                        "bound": "hbm" if t_h >= t_tc else "tensor", "frac_of_roofline_time": t_roof / t,
                        "tokens_per_s": N / t}
        bwd["device_status"] = h.device_status()
        bwd["kernels"] = {"dx": "fused forward kernel on the adjoint operator (1 launch)",
                          "dw": "tcgen05 contraction over tokens + deterministic reduction and inverse DFT "
                                "(2 launches)" if wl.io_dtype != "f32" else
                                "float64 CUDA-core kernel (clear + kernel + convert)"}
        out["backward"] = bwd
        del dxs, ws_t

    # ------------------------------------------------------- MLP block
    # The equivariant MLP block y = L2(GELU(L1(x))) at the workload's channels with a
    # 4x hidden layer (square 16-bit workloads): one fused launch (eqlin_mlp_forward,
    # the hidden activation stays on chip), timed like the backward calls; the
    # two-launch form (GELU in the first forward's epilogue, the hidden activation
    # through HBM) is timed beside it for comparison.
    if not args.no_mlp_block and wl.io_dtype != "f32" and wl.Cin == wl.Cout:
        out["mlp_block"] = measure_mlp_block(ctx, wl, xs, ys, n_sets, K, warmup)

    # ------------------------------------------------------- dense baseline (context)
    if not args.no_dense_context and wl.io_dtype != "f32":
        out["dense_context"] = measure_dense_context(ctx, wl, su["w"], su["bias"], h, xs, n_sets, K, warmup,
                                                     out["us_per_launch"])

    h.close()
    del xs, ys
    torch.cuda.empty_cache()
    return out


def group_circulant_matrix(w: torch.Tensor) -> torch.Tensor:
    """The replicated dense weight of the pages' baseline ("Declaracion del Problema"):
    M[(o,g),(i,h)] = w[o,i,(g-h) mod G] as a [Cout*G, Cin*G] matrix, built by indexing on
    w's device, so that y[n] = M x[n] over the flattened [Cin*G] token."""
    Cout, Cin, G = w.shape
    gi = torch.arange(G, device=w.device)
    idx = (gi.view(G, 1) - gi.view(1, G)) % G                      # [g, h] -> (g - h) mod G
    return w[:, :, idx].permute(0, 2, 1, 3).reshape(Cout * G, Cin * G).contiguous()


def measure_dense_context(ctx: Ctx, wl: workloads.Workload, w, bias, h, xs, n_sets: int, K: int, warmup: int,
                          fused_us: float) -> dict:
    """The pages' baseline, for context: the layer as one dense GEMM over the replicated
    weight ("Declaracion del Problema": the group-circulant matrix M[(o,g),(i,h)] =
    w[o,i,(g-h) mod G], built on the device by indexing, then the GEMM F.linear runs,
    y = x M^T + b, as torch.addmm (torch.mm without bias) into preallocated outputs: a
    cuBLAS bf16 GEMM with fp32 accumulation and no allocation in the timed loop), timed
    like the fused kernel: K back-to-back calls between two events on rotating x/y sets.
    Its output is compared with the fused kernel's (relative norm difference), which
    checks the matrix's convention."""
    dev, stream = ctx.dev, ctx.stream
    G, N = wl.G, wl.N
    M = group_circulant_matrix(w.to(dev))
    bd = None if bias is None else bias.to(dev).repeat_interleave(G)
    x2 = [t.view(N, wl.Cin * G) for t in xs]
    y2 = [torch.empty(N, wl.Cout * G, dtype=wl.torch_dtype, device=dev) for _ in range(n_sets)]
    Mt = M.t()

    def run(i, st=stream):
        if bd is None:
            torch.mm(x2[i % n_sets], Mt, out=y2[i % n_sets])
        else:
            torch.addmm(bd, x2[i % n_sets], Mt, out=y2[i % n_sets])

    for i in range(max(3, warmup)):
        run(i)
    ms = time_back_to_back(ctx, run, K, graph=False)
    us = 1e3 * ms / K
    y_d = y2[(K - 1) % n_sets].float()
    y_f = h.forward(xs[(K - 1) % n_sets], stream=stream).view(N, wl.Cout * G).float()
    diff = ((y_d - y_f).norm() / y_f.norm()).item()
    dense_fl = 2.0 * N * (wl.Cin * G) * (wl.Cout * G)
    return {"us_per_call": us, "calls": K, "dense_flops": dense_fl, "dense_tflops": dense_fl / (us * 1e-6) / 1e12,
            "fused_over_dense_speedup": us / fused_us, "rel_diff_vs_fused": diff,
            "what": "the GEMM of F.linear (torch.addmm / torch.mm into preallocated outputs) on the replicated "
                    "group-circulant [Cout*G, Cin*G] matrix: cuBLAS, bf16 in, fp32 accumulate; x/y sets rotate "
                    "as in the fused timing; context, not a target"}


def measure_mlp_block(ctx: Ctx, wl: workloads.Workload, xs, ys, n_sets: int, K: int, warmup: int) -> dict:
    eq, dev, stream, peaks = ctx.eq, ctx.dev, ctx.stream, ctx.peaks
    N, H, e = wl.N, 4 * wl.Cin, wl.elem_bytes
    w1, b1, w2, b2 = workloads.make_mlp_weights(wl, H)
    Kb = max(10, min(max(K, 100), 200))
    fl = 2 * N * wl.Cin * H * (2 * wl.G - 2) + 2 * N * H * wl.Cout * (2 * wl.G - 2)
    t_tc = fl / (peaks["bf16_tflops"] * 1e12)

    def timed(fn) -> float:
        for i in range(max(3, warmup)):
            fn(i)
        return 1e3 * time_back_to_back(ctx, fn, Kb, graph=ctx.graph) / Kb   # us per block

    # fused: x in, y out, both weight sets once
    m = eq.eqlin_mlp_prepare(w1.to(dev), b1.to(dev), w2.to(dev), b2.to(dev))
    us = timed(lambda i, st=stream: m.forward(xs[i % n_sets], out=ys[i % n_sets], stream=st))
    fbytes = N * (wl.Cin + wl.Cout) * wl.G * e + wl.G * (wl.Cin * H + H * wl.Cout) * e
    t_h = fbytes / (peaks["hbm_gbs"] * 1e9)
    res = {"H": H, "us_per_block": us, "calls": Kb, "launches_per_block": 1, "kernel": "eqlin_mlp_tc_kernel",
           "device_status": m.device_status(), "tokens_per_s": N / (us * 1e-6), "bytes": fbytes,
           "fourier_flops": fl, "roofline_time_us": 1e6 * max(t_h, t_tc), "bound": "hbm" if t_h >= t_tc else "tensor",
           "frac_of_roofline_time": max(t_h, t_tc) / (us * 1e-6),
           "tensor_tflops": fl / (us * 1e-6) / 1e12}
    m.close()
    # two launches, the hidden activation through HBM (for comparison)
    h1 = eq.prepare(w1.to(dev), b1.to(dev), io_dtype=wl.torch_dtype, activation="gelu")
    h2 = eq.prepare(w2.to(dev), b2.to(dev), io_dtype=wl.torch_dtype)
    hidden = torch.empty(N, H, wl.G, dtype=wl.torch_dtype, device=dev)
    us2 = timed(lambda i, st=stream: eq.mlp_block(h1, h2, xs[i % n_sets], hidden=hidden, out=ys[i % n_sets],
                                                  stream=st))
    tbytes = N * (wl.Cin + 2 * H + wl.Cout) * wl.G * e + wl.G * (wl.Cin * H + H * wl.Cout) * e
    t_h2 = tbytes / (peaks["hbm_gbs"] * 1e9)
    res["two_launches"] = {"us_per_block": us2, "bytes": tbytes, "roofline_time_us": 1e6 * max(t_h2, t_tc),
                           "frac_of_roofline_time": max(t_h2, t_tc) / (us2 * 1e-6),
                           "device_status": max(h1.device_status(), h2.device_status(), key=abs)}
    res["speedup_over_two_launches"] = us2 / us
    del hidden
    h1.close()
    h2.close()
    return res


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=workloads.HEADLINE, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="eqlin", choices=["eqlin", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="oracle sample of the headline workload, seconds on all cores")
    ap.add_argument("--cpu-seconds-other", type=float, default=3.0,
                    help="oracle sample of each other workload, seconds on all cores")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", action="store_true",
                    help="measure only --workload (no workloads object)")
    ap.add_argument("--graph", action="store_true",
                    help="time one CUDA-graph replay of the K launches instead of K launches from the host "
                         "(the graph is replayed once, untimed, to upload it)")
    ap.add_argument("--no-mlp-block", action="store_true",
                    help="skip the extra measurement of the equivariant MLP block L2(GELU(L1(x))), H = 4 C")
    ap.add_argument("--no-dense-context", action="store_true",
                    help="skip the pages' baseline, one dense cuBLAS GEMM on the replicated weight, timed "
                         "as context (dense_context in each 16-bit workload)")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the extra measurement of the backward calls (input and weight gradients)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's token count (profiling a smaller case; implies --only)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    wl = workloads.WORKLOADS[args.workload]
    if args.tokens is not None:
        wl = wl.with_n(args.tokens)
        args.only = True

    if args.impl == "reference":
        run_reference(args, wl)
        return

    import cyclic_group_dft_b200 as eq
    eq.library()   # the CUDA library; fails loudly when it is missing

    world, rank, local = dist_info()
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks, peak_kind = load_peaks()
    ctx = Ctx(eq, dev, world, torch.cuda.current_stream(dev), peaks, peak_kind, graph=args.graph)

    # every other workload first (each step count at least 100 launches: their launches
    # are short), the headline last with exactly --steps timed launches
    # the headline first, then every other workload (each step count at least 100 launches:
    # their launches are short)
    head = measure_workload(ctx, wl, args.steps, args.warmup, True, args)
    results = {}
    if not args.only:
        for name in BENCH_WORKLOADS:
            if name == wl.name:
                continue
            results[name] = measure_workload(ctx, workloads.WORKLOADS[name], max(args.steps, 100), args.warmup,
                                             False, args)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, args.cpu_seconds, min(args.cpu_seconds, 5.0))
        for name, r in results.items():
            r["cpu_baseline"] = cpu_baseline(workloads.WORKLOADS[name], args.cpu_seconds_other)
        head["cpu_baseline"] = cpu

    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    if not args.only:
        ordered = {name: head if name == wl.name else results[name] for name in BENCH_WORKLOADS}
        wl_obj = {name: {k: v for k, v in r.items() if k not in ("e2e", "clocks")}
                  for name, r in ordered.items()}
    else:
        wl_obj = None

    line = {
        "metric": METRIC,
        "value": head["tokens_per_s"],
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": head["elapsed_ms"] / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.io_dtype,
        "data": "synthetic",
        "config": line_config(wl, world),
        "timing": head["timing"],
        "us_per_launch_host_launches": head["us_per_launch_host_launches"],
        "kernel": head["kernel"],
        "roofline": head["roofline"],
        "dense_equivalent_tflops": head["dense_equivalent_tflops"],
        "launch_us": head["launch_us"],
        "clocks": head.get("clocks"),
        "e2e": head.get("e2e"),
        "gpu_launches": args.steps,
        "device_status": head["device_status"],
        "cpu_baseline": cpu,
        "backward": head.get("backward"),
        "mlp_block": head.get("mlp_block"),
        "dense_context": head.get("dense_context"),
        "workloads": wl_obj,
    }
    emit(line)


if __name__ == "__main__":
    main()
