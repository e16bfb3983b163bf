#!/usr/bin/env python
"""Benchmark of the fused EQ-Linear forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl eqlin|reference]

One step = one eqlin_forward over the whole workload batch (weights prepared
once, outside the timed region; inputs already resident in HBM).  Prints ONE
JSON line (rank 0): tokens/s over all ranks, ms per step, the roofline of the
fused kernel (algorithmic bytes / HBM peak, Fourier FLOPs / bf16 tensor peak),
clocks sampled during the timed region, an end-to-end figure through the host
buffer API, and the CPU float64 oracle's throughput on a bounded sample.

Multi-GPU (torchrun): every rank runs the full workload on its own GPU (tokens
are independent, no collective on the data path): weak scaling; the timed
region is bracketed by barriers and the slowest rank's time is used.

--impl reference times the float64 CPU oracle on the host cores instead (the
method's plain definition), on bounded token samples of the same workload.
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

from cyclic_group_dft_b200 import workloads  # noqa: E402

METRIC = "EQ-Linear tokens/s and % of roofline (HBM vs bf16 TC), p4 Cin=Cout=96"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024
# device code of each fused kernel: a recorded ncu traffic figure is reported only
# while these files are unchanged since the capture
KERNEL_SOURCES = {
    "eqlin_fwd_tc": ["eqlin_fwd_tc.cuh", "group_dft.cuh", "io16.cuh", "sm100_ptx.cuh", "eqlin_layout.h"],
    "eqlin_fwd_tm": ["eqlin_fwd_tm.cuh", "group_dft.cuh", "io16.cuh", "sm100_ptx.cuh", "eqlin_layout.h"],
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


def recorded_traffic(workload: str):
    """DRAM bytes per launch from a committed ncu capture, if the kernel is unchanged since."""
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
    return entry.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML in a thread."""

    def __init__(self, device_index: int, period_s: float = 0.01):
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
        while not self._stop.is_set():
            self._sample()
            self._stop.wait(self.period)

    def start(self):
        if self._nvml is not None:
            self._sample()
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
                "samples": len(self.samples)}


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
    sample = f"{n} of {wl.N} tokens per step (tokens are independent; rate scales linearly)"
    emit({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps * wl.N / n, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "N": wl.N, "Cin": wl.Cin, "Cout": wl.Cout, "G": wl.G,
                   "io": wl.io_dtype},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    })


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default=workloads.HEADLINE, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--impl", default="eqlin", choices=["eqlin", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-mlp-block", action="store_true",
                    help="skip the extra measurement of the equivariant MLP block L2(GELU(L1(x))), H = 4 C")
    ap.add_argument("--no-backward", action="store_true",
                    help="skip the extra measurement of the backward calls (input and weight gradients)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's token count (profiling a smaller case)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    wl = workloads.WORKLOADS[args.workload]
    if args.tokens is not None:
        wl = wl.with_n(args.tokens)

    if args.impl == "reference":
        run_reference(args, wl)
        return

    import cyclic_group_dft_b200 as eq

    world, rank, local = dist_info()
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    x_cpu, w, bias = workloads.make_inputs(wl)
    h = eq.prepare(w.to(dev), None if bias is None else bias.to(dev), io_dtype=wl.torch_dtype,
                   backward=not args.no_backward)
    N = wl.N
    set_bytes = N * (wl.Cin + wl.Cout) * wl.G * wl.elem_bytes
    n_sets = max(2, math.ceil(2 * L2_BYTES / set_bytes))
    xs = [x_cpu.to(dev) for _ in range(n_sets)]
    ys = [torch.empty(N, wl.Cout, wl.G, dtype=wl.torch_dtype, device=dev) for _ in range(n_sets)]
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for i in range(args.warmup):
        h.forward(xs[i % n_sets], out=ys[i % n_sets], stream=stream)
    torch.cuda.synchronize(dev)
    if h.device_status() != eq.EQLIN_OK:
        raise RuntimeError("device status not OK after warm-up")

    # ----------------------------------------------------------- timed region
    # K back-to-back steps, one fused launch each, bracketed by two events on the
    # launching stream.  No event sits between the launches: an event there would end
    # the overlap of one launch's tail with the next one's prologue (programmatic
    # dependent launch), which is how the kernel runs in a real stream of layers.
    # The average launch duration of the kernel is therefore elapsed / K.
    K = args.steps
    clocks = ClockSampler(dev.index)
    barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_begin.record(stream)
    for i in range(K):
        h.forward(xs[i % n_sets], out=ys[i % n_sets], stream=stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    clocks.stop()
    barrier()
    elapsed_ms = t_begin.elapsed_time(t_end)
    status = h.device_status()

    elapsed_ms = reduce_max(elapsed_ms, dev)
    value = aggregate_tokens_per_s(world, K, N, elapsed_ms)
    avg_launch_s = elapsed_ms / K / 1e3

    # Launch-duration distribution, outside the timed region: an event pair around
    # each launch (which serialises the launches, so each one also pays its own
    # prologue and tail).
    KL = min(K, 100)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(KL)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(KL)]
    for i in range(KL):
        starts[i].record(stream)
        h.forward(xs[i % n_sets], out=ys[i % n_sets], stream=stream)
        ends[i].record(stream)
    torch.cuda.synchronize(dev)
    launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]

    # ----------------------------------------------------------- end to end
    E = args.e2e_steps
    e2e = None
    if E > 0:
        x_pin = x_cpu.pin_memory()
        y_pin = torch.empty(N, wl.Cout, wl.G, dtype=wl.torch_dtype).pin_memory()
        h.forward_host(x_pin, y_pin)  # warm the path
        barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(E):
            h.forward_host(x_pin, y_pin, stream=stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e2e_ms = reduce_max(e0.elapsed_time(e1), dev)
        e2e = {"value": aggregate_tokens_per_s(world, E, N, e2e_ms), "unit": "tokens/s", "steps": E,
               "h2d_bytes_per_step": x_pin.numel() * x_pin.element_size(),
               "d2h_bytes_per_step": y_pin.numel() * y_pin.element_size(),
               "api": "eqlin_forward_host (C ABI: pinned host x and y, chunked copies in and out "
                      "overlapping the fused kernel on two streams)"}

    # ----------------------------------------------------------- backward calls
    # Measured after the forward's timed region, on the same rotating buffer sets
    # (the forward outputs stand in for dy): us per call from CUDA events around
    # Kb back-to-back calls, against the same roofline model as the forward.
    bwd = None
    if not args.no_backward:
        Kb = max(10, min(K, 200))
        dxs = [torch.empty(N, wl.Cin, wl.G, dtype=wl.torch_dtype, device=dev) for _ in range(n_sets)]
        dw_t = torch.empty(wl.Cout, wl.Cin, wl.G, dtype=torch.float32, device=dev)
        db_t = torch.empty(wl.Cout, dtype=torch.float32, device=dev)
        ws_t = torch.empty(max(16, eq.eqlin_backward_dw_workspace_size(h, N)), dtype=torch.uint8, device=dev)
        calls = {
            "dx": lambda i: h.backward_dx(ys[i % n_sets], out=dxs[i % n_sets], stream=stream),
            "dw": lambda i: eq.eqlin_backward_dw(h, xs[i % n_sets], ys[i % n_sets], stream=stream,
                                                 dw=dw_t, dbias=db_t, workspace=ws_t),
        }
        bwd = {}
        for key, fn in calls.items():
            for i in range(max(3, args.warmup)):
                fn(i)
            barrier()
            torch.cuda.synchronize(dev)
            b0 = torch.cuda.Event(enable_timing=True)
            b1 = torch.cuda.Event(enable_timing=True)
            b0.record(stream)
            for i in range(Kb):
                fn(i)
            b1.record(stream)
            torch.cuda.synchronize(dev)
            barrier()
            bwd[key] = {"us_per_call": 1e3 * reduce_max(b0.elapsed_time(b1), dev) / Kb, "calls": Kb}
        bwd["device_status"] = h.device_status()
        bwd["kernels"] = {"dx": "fused forward kernel on the adjoint operator (1 launch)",
                          "dw": "tcgen05 contraction over tokens + deterministic reduction and inverse DFT "
                                "(2 launches)" if wl.io_dtype != "f32" else
                                "float64 CUDA-core kernel (clear + kernel + convert)"}
        del dxs

    # ----------------------------------------------------------- MLP block
    # The equivariant MLP block y = L2(GELU(L1(x))) at the workload's channels with a
    # 4x hidden layer (16-bit square workloads): two fused launches, GELU in the first
    # one's epilogue, the hidden activation through HBM.  Timed like the backward calls.
    mlp = None
    if not args.no_mlp_block and wl.io_dtype != "f32" and wl.Cin == wl.Cout:
        H = 4 * wl.Cin
        w1, b1, w2, b2 = workloads.make_mlp_weights(wl, H)
        h1 = eq.prepare(w1.to(dev), b1.to(dev), io_dtype=wl.torch_dtype, activation="gelu")
        h2 = eq.prepare(w2.to(dev), b2.to(dev), io_dtype=wl.torch_dtype)
        hidden = torch.empty(N, H, wl.G, dtype=wl.torch_dtype, device=dev)
        Kb = max(10, min(K, 200))
        for i in range(max(3, args.warmup)):
            eq.mlp_block(h1, h2, xs[i % n_sets], hidden=hidden, out=ys[i % n_sets], stream=stream)
        barrier()
        torch.cuda.synchronize(dev)
        m0 = torch.cuda.Event(enable_timing=True)
        m1 = torch.cuda.Event(enable_timing=True)
        m0.record(stream)
        for i in range(Kb):
            eq.mlp_block(h1, h2, xs[i % n_sets], hidden=hidden, out=ys[i % n_sets], stream=stream)
        m1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        us = 1e3 * reduce_max(m0.elapsed_time(m1), dev) / Kb
        mlp = {"H": H, "us_per_block": us, "calls": Kb, "launches_per_block": 2,
               "device_status": max(h1.device_status(), h2.device_status(), key=abs),
               "tokens_per_s": N / (us * 1e-6)}
        del hidden
        h1.close()
        h2.close()

    # ----------------------------------------------------------- CPU baseline
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, n_s, dt, threads = oracle_rate(wl, args.cpu_seconds)
        rate1, n1, dt1, _ = oracle_rate(wl, min(args.cpu_seconds, 5.0), threads=1)
        cpu = {"value": rate, "unit": "tokens/s", "cores": threads, "kind": "oracle",
               "sample": f"{n_s} of {wl.N} tokens of {wl.name} in {dt:.1f} s (float64 definition loops, OpenMP over tokens)",
               "single_core": {"value": rate1, "unit": "tokens/s", "cores": 1,
                               "sample": f"{n1} of {wl.N} tokens in {dt1:.1f} s"}}

    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_kind = load_peaks()
    bytes_launch = algorithmic_bytes(wl, N)
    flops_launch = fourier_flops(wl, N)
    gbs = bytes_launch / avg_launch_s / 1e9
    tflops = flops_launch / avg_launch_s / 1e12
    t_hbm = bytes_launch / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops_launch / (peaks["bf16_tflops"] * 1e12)
    bound = "hbm" if t_hbm >= t_tc else "tensor"
    if bound == "hbm":
        roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"]}
    else:
        roof = {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": tflops / peaks["bf16_tflops"]}
    roof["traffic"] = recorded_traffic(wl.name)
    roof["peak_source"] = f"{peak_kind} (MEASURED_PEAKS.json)" if peak_kind == "measured" else "fallback"
    roof["roofline_time_us"] = 1e6 * max(t_hbm, t_tc)
    roof["kernel_us"] = 1e6 * avg_launch_s
    roof["frac_of_roofline_time"] = max(t_hbm, t_tc) / avg_launch_s
    roof["bytes_per_launch"] = bytes_launch
    roof["tensor_tflops"] = tflops
    roof["tensor_frac"] = tflops / peaks["bf16_tflops"]                       # burst peak: the headline
    roof["tensor_frac_sustained"] = tflops / peaks["bf16_tflops_sustained"]   # seconds-long GEMM peak

    if mlp is not None:
        e, H = wl.elem_bytes, mlp["H"]
        # two launches: x in, hidden out and back in, y out, both weight sets
        mbytes = N * (wl.Cin + 2 * H + wl.Cout) * wl.G * e + 2 * wl.G * wl.Cin * H * e
        mflops = 2 * N * wl.Cin * H * (2 * wl.G - 2) + 2 * N * H * wl.Cout * (2 * wl.G - 2)
        t_mh = mbytes / (peaks["hbm_gbs"] * 1e9)
        t_mt = mflops / (peaks["bf16_tflops"] * 1e12)
        t = mlp["us_per_block"] * 1e-6
        mlp.update({"bytes": mbytes, "fourier_flops": mflops, "roofline_time_us": 1e6 * max(t_mh, t_mt),
                    "bound": "hbm" if t_mh >= t_mt else "tensor", "frac_of_roofline_time": max(t_mh, t_mt) / t,
                    "fused_block_roofline_us": 1e6 * max(N * (wl.Cin + wl.Cout) * wl.G * e / (peaks["hbm_gbs"] * 1e9),
                                                         t_mt),
                    "note": "roofline of the two-launch form (hidden activation through HBM); "
                            "fused_block_roofline_us is the bound of a single fused kernel"})
    if bwd is not None:
        bb = backward_bytes(wl, N)
        for key in ("dx", "dw"):
            t = bwd[key]["us_per_call"] * 1e-6
            t_h = bb[key] / (peaks["hbm_gbs"] * 1e9)
            t_roof = max(t_h, t_tc)
            bwd[key].update({"bytes": bb[key], "roofline_time_us": 1e6 * t_roof,
                             "bound": "hbm" if t_h >= t_tc else "tensor",
                             "frac_of_roofline_time": t_roof / t, "tokens_per_s": N / t})

    emit({
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": elapsed_ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": wl.io_dtype,
        "data": "synthetic",
        "config": {
            "workload": wl.name, "N": N, "Cin": wl.Cin, "Cout": wl.Cout, "G": wl.G, "io": wl.io_dtype,
            "global_batch": world * N, "parallelism": f"replicas{world}" if world > 1 else "single",
            "l2": f"inputs larger than L2; {n_sets} rotating x/y sets of {set_bytes / 1e6:.0f} MB",
            "kernel_path": h.path, "stages": h.attr("stages"), "tokens_per_tile": h.attr("tokens_per_tile"),
        },
        "roofline": roof,
        "dense_equivalent_tflops": dense_equivalent_flops(wl, N) / avg_launch_s / 1e12,
        "launch_us": {"mean": 1e3 * statistics.mean(launch_ms), "median": 1e3 * statistics.median(launch_ms),
                      "min": 1e3 * min(launch_ms), "max": 1e3 * max(launch_ms), "launches": len(launch_ms),
                      "note": "each launch bracketed by its own events (serialised), outside the timed region"},
        "clocks": clocks.summary(),
        "e2e": e2e,
        "gpu_launches": K,
        "device_status": status,
        "cpu_baseline": cpu,
        "backward": bwd,
        "mlp_block": mlp,
    })
    h.close()


if __name__ == "__main__":
    main()
