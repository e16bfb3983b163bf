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
