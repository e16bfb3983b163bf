"""The allocation-free forward, eqlin_forward_noalloc, against the handle API.

Some callers cannot call cudaMalloc: a framework whose device memory is owned by
its own pool, or a host loop that cannot take the synchronisation and latency of
an allocation.  For them the library offers one entry point that keeps everything
beyond the caller's inputs and output in a fixed array inside the library.  These
tests call it through the C ABI twice in a row and compare each result with the
existing entry points (eqlin_prepare_weights + eqlin_forward) at the tolerances
the other tests use.  The file is named to be collected last.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

import cyclic_group_dft_b200 as eq
from cyclic_group_dft_b200 import workloads
from parity_util import check

DEV = "cuda:0"
CODE = {torch.bfloat16: eq.EQLIN_BF16, torch.float32: eq.EQLIN_F32}


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
def test_noalloc_two_calls_match_handle_api():
    # two calls in a row, different workloads, so the second overwrites the first's scratch
    cases = [("p4_c96_bf16", 0, 1031), ("p8_c64_bf16", 1, 777), ("tiny_p4_fp32", 2, 300),
             ("p4_c96_bf16", 3, 4099)]
    for name, seed, N in cases:
        wl = workloads.WORKLOADS[name]
        x, w, bias = workloads.make_inputs(wl, seed=seed, N=N)
        x, w = x.to(DEV), w.to(DEV)
        bias = None if bias is None else bias.to(DEV)
        ref = _handle_api(x, w, bias).float().cpu().numpy()
        for call in range(2):
            y = torch.full((N, wl.Cout, wl.G), float("nan"), dtype=x.dtype, device=DEV)
            assert _noalloc_raw(x, w, bias, y) == eq.EQLIN_OK, eq.eqlin_last_error()
            torch.cuda.synchronize()
            r = check(x.dtype, y, ref)
            assert r["ok"], (name, call, r)


@pytest.mark.gpu
def test_noalloc_streamed_weights_and_no_bias():
    wl = workloads.WORKLOADS["p4_mlp_bf16"]             # Cout = 768: weights streamed, no bias
    x, w, bias = workloads.make_inputs(wl, N=513)
    x, w = x.to(DEV), w.to(DEV)
    ref = _handle_api(x, w, None).float().cpu().numpy()
    y = eq.eqlin_forward_noalloc(x, w, None)
    torch.cuda.synchronize()
    assert check(torch.bfloat16, y, ref)["ok"]


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
