"""The allocation-free forward, eqlin_forward_noalloc, against the handle API.

Some callers cannot call cudaMalloc: a framework whose device memory is owned by
its own pool, or a host loop that cannot take the synchronisation and latency of
an allocation.  For them the library offers one entry point that keeps everything
beyond the caller's inputs and output in a fixed array inside the library.  These
tests call it through the C ABI twice in a row and compare each result with the
existing entry points (eqlin_prepare_weights + eqlin_forward).  Both run the same
weight transform and the same fused kernels, so the outputs must be identical bit
for bit; one case is also checked directly against the float64 oracle at the
tolerances the other tests use.  The file is named to be collected last.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

import cyclic_group_dft_b200 as eq
from cyclic_group_dft_b200 import workloads
from parity_util import check, oracle_forward

DEV = "cuda:0"
CODE = {torch.bfloat16: eq.EQLIN_BF16, torch.float16: eq.EQLIN_F16, torch.float32: eq.EQLIN_F32}


def _noalloc_raw(x, w, bias, y):
    N, Cin, G = x.shape
    Cout = w.shape[0]
    return eq.library().eqlin_forward_noalloc(
        x.data_ptr(), w.data_ptr(), None if bias is None else bias.data_ptr(), y.data_ptr(),
        N, Cout, Cin, G, CODE[x.dtype], torch.cuda.current_stream().cuda_stream)


def _handle_api(x, w, bias):
    h = eq.prepare(w, bias, io_dtype=x.dtype)
    y = h.forward(x)
    torch.cuda.synchronize()
    h.close()
    return y


@pytest.mark.gpu
def test_noalloc_two_calls_equal_handle_api():
    # two calls in a row per case, cases of different shapes and dtypes in a row, so
    # each call overwrites the previous one's scratch
    cases = [("p4_c96_bf16", 0, 1031), ("p8_c64_bf16", 1, 777), ("tiny_p4_fp32", 2, 300),
             ("p4_c96_f16", 4, 2050), ("c16_c32_bf16", 5, 515), ("p4_c96_bf16", 3, 4099)]
    for name, seed, N in cases:
        wl = workloads.WORKLOADS[name]
        x, w, bias = workloads.make_inputs(wl, seed=seed, N=N)
        x, w = x.to(DEV), w.to(DEV)
        bias = None if bias is None else bias.to(DEV)
        ref = _handle_api(x, w, bias)
        for call in range(2):
            y = torch.full((N, wl.Cout, wl.G), float("nan"), dtype=x.dtype, device=DEV)
            assert _noalloc_raw(x, w, bias, y) == eq.EQLIN_OK, eq.eqlin_last_error()
            torch.cuda.synchronize()
            assert torch.equal(y, ref), (name, call, (y.float() - ref.float()).abs().max().item())


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["p4_c96_bf16", "tiny_p4_fp32", "p4_c96_f16"])
def test_noalloc_against_oracle(name):
    wl = workloads.WORKLOADS[name]
    N = 1031 if wl.N > 1031 else wl.N
    x, w, bias = workloads.make_inputs(wl, seed=7, N=N)
    ref = oracle_forward(x, w, bias)
    xd, wd = x.to(DEV), w.to(DEV)
    bd = None if bias is None else bias.to(DEV)
    for call in range(2):
        y = eq.eqlin_forward_noalloc(xd, wd, bd)
        torch.cuda.synchronize()
        r = check(x.dtype, y, ref)
        assert r["ok"], (name, call, r)


@pytest.mark.gpu
def test_noalloc_streamed_weights_and_no_bias():
    wl = workloads.WORKLOADS["p4_mlp_bf16"]             # Cout = 768: weights streamed, no bias
    x, w, bias = workloads.make_inputs(wl, N=513)
    x, w = x.to(DEV), w.to(DEV)
    ref = _handle_api(x, w, None)
    for _ in range(2):
        y = eq.eqlin_forward_noalloc(x, w, None)
        torch.cuda.synchronize()
        assert torch.equal(y, ref)


@pytest.mark.gpu
def test_noalloc_rejects_shapes_beyond_its_scratch():
    x = torch.zeros(8, 1024, 4, dtype=torch.bfloat16, device=DEV)
    w = torch.zeros(1024, 1024, 4, dtype=torch.bfloat16, device=DEV)
    y = torch.empty(8, 1024, 4, dtype=torch.bfloat16, device=DEV)
    assert _noalloc_raw(x, w, None, y) == eq.EQLIN_ERR_UNSUPPORTED
    assert "scratch" in eq.eqlin_last_error()


def test_noalloc_validates_on_host():
    lib = eq.library()
    null = ctypes.c_void_p(0)
    assert lib.eqlin_forward_noalloc(16, null, null, 16, 4, 8, 8, 4, eq.EQLIN_BF16, null) == eq.EQLIN_ERR_INVALID_ARG
    assert lib.eqlin_forward_noalloc(16, 16, null, 16, 4, 8, 8, 3, eq.EQLIN_BF16, null) == eq.EQLIN_ERR_UNSUPPORTED
    assert lib.eqlin_forward_noalloc(16, 16, null, 16, -1, 8, 8, 4, eq.EQLIN_BF16, null) == eq.EQLIN_ERR_INVALID_ARG
    assert lib.eqlin_forward_noalloc(null, 16, null, null, 0, 8, 8, 4, eq.EQLIN_BF16, null) == eq.EQLIN_OK


def test_noalloc_binding_rejects_a_wrong_output():
    # the binding checks y before any call: a y that is too small, of another dtype or
    # not contiguous would let the kernel write past its storage
    x = torch.zeros(4, 8, 4, dtype=torch.bfloat16)
    w = torch.zeros(8, 8, 4, dtype=torch.bfloat16)
    for y in (torch.empty(3, 8, 4, dtype=torch.bfloat16), torch.empty(4, 8, 4, dtype=torch.float16),
              torch.empty(4, 4, 8, dtype=torch.bfloat16).transpose(1, 2)):
        with pytest.raises(ValueError):
            eq.eqlin_forward_noalloc(x, w, None, y=y)
