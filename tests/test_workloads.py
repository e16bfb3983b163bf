"""The seeded synthetic inputs (no GPU): shapes, dtypes, determinism, the variance
reading (second parameter = variance, so var(y) stays near 1), weights independent of N,
the bias-free MLP workload, and the sampled-token helper."""
from __future__ import annotations

import math

import pytest
import torch

from cyclic_group_dft_b200 import workloads


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_shapes_dtypes_and_determinism(name):
    wl = workloads.WORKLOADS[name]
    x, w, b = workloads.make_inputs(wl, N=300)
    assert x.shape == (300, wl.Cin, wl.G) and w.shape == (wl.Cout, wl.Cin, wl.G)
    assert x.dtype == wl.torch_dtype and w.dtype == wl.torch_dtype
    assert (b is None) == (wl.bias_var is None)
    x2, w2, b2 = workloads.make_inputs(wl, N=300)
    assert torch.equal(x, x2) and torch.equal(w, w2) and (b is None or torch.equal(b, b2))
    x3, _, _ = workloads.make_inputs(wl, seed=wl.seed + 1, N=300)
    assert not torch.equal(x, x3)


def test_weights_do_not_depend_on_n():
    wl = workloads.WORKLOADS["p4_c96_bf16"]
    _, w_a, b_a = workloads.make_inputs(wl, N=10)
    _, w_b, b_b = workloads.make_inputs(wl, N=5000)
    assert torch.equal(w_a, w_b) and torch.equal(b_a, b_b)


def test_variances_follow_the_reading():
    wl = workloads.WORKLOADS["p4_c96_bf16"]
    x, w, b = workloads.make_inputs(wl, N=20000)
    assert float(x.float().var()) == pytest.approx(1.0, rel=0.03)
    assert float(w.float().var()) == pytest.approx(1.0 / (wl.Cin * wl.G), rel=0.05)
    assert float(b.float().var()) == pytest.approx(0.1, rel=0.5)   # 96 draws
    assert wl.w_var == pytest.approx(1.0 / (wl.Cin * wl.G))


def test_the_mlp_workload_has_no_bias_and_the_headline_sizes():
    assert workloads.WORKLOADS["p4_mlp_bf16"].bias_var is None
    wl = workloads.WORKLOADS[workloads.HEADLINE]
    assert (wl.N, wl.Cin, wl.Cout, wl.G) == (64 * 56 * 56, 96, 96, 4)
    assert workloads.WORKLOADS["p8_c64_bf16"].N == 32 * 28 * 28


def test_sample_tokens_covers_the_ends_and_is_sorted():
    idx = workloads.sample_tokens(100000, 512, seed=3)
    assert idx[0] == 0 and idx[-1] == 99999 and bool((idx[1:] > idx[:-1]).all())
    assert len(idx) <= 512
    assert torch.equal(idx, workloads.sample_tokens(100000, 512, seed=3))
    assert torch.equal(workloads.sample_tokens(50, 512), torch.arange(50))


def test_mlp_weights_shapes_and_scales():
    wl = workloads.WORKLOADS["p4_c96_bf16"]
    w1, b1, w2, b2 = workloads.make_mlp_weights(wl, 384)
    assert w1.shape == (384, 96, 4) and w2.shape == (96, 384, 4) and b1.shape == (384,) and b2.shape == (96,)
    assert float(w1.float().var()) == pytest.approx(1.0 / (96 * 4), rel=0.05)
    assert float(w2.float().var()) == pytest.approx(1.0 / (384 * 4), rel=0.05)
    assert math.isfinite(float(b1.float().sum()))
