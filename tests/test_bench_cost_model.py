"""The roofline denominators of bench.py: algorithmic bytes and FLOPs per launch for
every workload, against the figures of the hot-path scope table (bytes moved: read x
once, write y once, read the frequency-domain weights and the bias once; Fourier FLOPs
2*N*Cin*Cout*(2G-2); dense-equivalent FLOPs 2*N*(Cin*G)*(Cout*G))."""
from __future__ import annotations

import importlib.util
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_cost", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv, sys.argv = sys.argv, ["bench.py"]
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


# (workload, MB moved, Fourier GFLOP, dense-equivalent GFLOP), rounded as tabulated
TABLE = [
    ("tiny_p4_fp32", 0.135, 0.00079, 0.00210),
    ("p4_c96_bf16", 308.36, 22.20, 59.19),
    ("p8_c64_bf16", 51.45, 2.88, 13.15),
    ("p4_mlp_bf16", 504.50, 115.96, 309.24),
    ("c16_c32_bf16", 536.90, 16.11, 137.44),
]


@pytest.mark.parametrize("name,mb,gf,dense", TABLE)
def test_cost_model_matches_the_scope_table(name, mb, gf, dense):
    b = _bench()
    from cyclic_group_dft_b200 import workloads
    wl = workloads.WORKLOADS[name]
    assert b.algorithmic_bytes(wl, wl.N) / 1e6 == pytest.approx(mb, rel=2e-3)
    assert b.fourier_flops(wl, wl.N) / 1e9 == pytest.approx(gf, rel=5e-3)
    assert b.dense_equivalent_flops(wl, wl.N) / 1e9 == pytest.approx(dense, rel=5e-3)


def test_fourier_share_of_the_dense_count():
    """(2G-2)/G^2 of the dense MACs: 6/16 at G = 4 ([FEL] p4 section), 14/64 at G = 8."""
    b = _bench()
    from cyclic_group_dft_b200 import workloads
    for name, ratio in (("p4_c96_bf16", 6 / 16), ("p8_c64_bf16", 14 / 64), ("c16_c32_bf16", 30 / 256)):
        wl = workloads.WORKLOADS[name]
        assert b.fourier_flops(wl, wl.N) / b.dense_equivalent_flops(wl, wl.N) == pytest.approx(ratio, rel=1e-12)


def test_oracle_rate_reports_its_threads():
    """The CPU baseline's timing helper: a bounded sample, on the threads asked for."""
    b = _bench()
    from cyclic_group_dft_b200 import workloads
    wl = workloads.WORKLOADS["tiny_p4_fp32"]
    rate, n, dt, threads = b.oracle_rate(wl, 0.05, threads=1)
    assert threads == 1 and 64 <= n <= wl.N and rate > 0 and dt > 0


def test_reference_arm_maps_no_cuda_library():
    """bench.py --impl reference times the float64 oracle only: importing the bench, the
    seeded input generators and the oracle maps the oracle's library, never libeqlin.so."""
    import subprocess
    code = ("import sys; sys.argv = ['bench.py']; sys.path.insert(0, %r); import bench, oracle; "
            "from cyclic_group_dft_b200 import workloads; "
            "x, w, b = workloads.make_inputs(workloads.WORKLOADS['tiny_p4_fp32'], N=8); "
            "oracle.forward(x, w, b); maps = open('/proc/self/maps').read(); "
            "print(int('libeqlin.so' in maps), int('eqlin_oracle' in maps))") % ROOT
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.split()[-2:] == ["0", "1"], out.stdout


def test_both_arms_share_the_config():
    """The GPU line and the reference line carry the same `config` (line_config)."""
    b = _bench()
    from cyclic_group_dft_b200 import workloads
    wl = workloads.WORKLOADS["p4_c96_bf16"]
    c = b.line_config(wl, 1)
    assert c == b.line_config(wl, 1)
    assert set(c) == {"workload", "N", "Cin", "Cout", "G", "io", "global_batch", "parallelism", "l2"}
    assert c["N"] == 64 * 56 * 56 and c["workload"] == "p4_c96_bf16"
    assert b.BENCH_WORKLOADS == ("tiny_p4_fp32", "p4_c96_bf16", "p8_c64_bf16", "p4_mlp_bf16", "c16_c32_bf16")


def test_clock_sampler_stays_out_of_short_timed_regions(monkeypatch):
    """The clock sampler queries NVML right after the timed region (stop); while the region
    runs its thread waits one period before its first query, so a region shorter than the
    period sees no query at all.  A fake NVML counts them."""
    import threading
    import types
    calls = []
    fake = types.SimpleNamespace(
        NVML_CLOCK_SM=0,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByIndex=lambda i: "h",
        nvmlDeviceGetMaxClockInfo=lambda h, c: 1965,
        nvmlDeviceGetClockInfo=lambda h, c: calls.append(threading.current_thread().name) or 1965,
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: 0,
    )
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    b = _bench()
    c = b.ClockSampler(0, period_s=0.5)
    assert not calls              # constructing it queries no clock
    c.start()
    c.stop()                      # a region far shorter than the period
    assert len(calls) == 1        # the sample right after the region only
    s = c.summary()
    assert s["sm_mhz"] == 1965 and s["samples"] == 1 and "right after it" in s["sampling"]
    calls.clear()
    c = b.ClockSampler(0, period_s=0.01)
    c.start()
    threading.Event().wait(0.1)   # a region of ten periods is sampled inside
    c.stop()
    assert len(calls) >= 5


@pytest.mark.parametrize("Cout,Cin,G", [(3, 5, 2), (4, 3, 4), (2, 3, 8), (3, 2, 16)])
def test_dense_baseline_matrix_is_the_oracle_one(Cout, Cin, G):
    """The dense baseline the bench times beside the fused kernel multiplies by the same
    replicated group-circulant matrix as the oracle's dense_weight, and that matrix
    reproduces the oracle's forward."""
    import numpy as np
    import torch

    import oracle
    b = _bench()
    gen = torch.Generator().manual_seed(Cout * 100 + Cin * 10 + G)
    w = torch.randn(Cout, Cin, G, generator=gen, dtype=torch.float64)
    x = torch.randn(7, Cin, G, generator=gen, dtype=torch.float64)
    M = b.group_circulant_matrix(w)
    assert np.array_equal(M.numpy(), oracle.dense_weight(w.numpy()))
    y = (x.reshape(7, Cin * G) @ M.T).reshape(7, Cout, G)
    np.testing.assert_allclose(y.numpy(), oracle.forward(x.numpy(), w.numpy()), rtol=1e-12, atol=1e-12)
