"""GPU parity of the backward pass (input, weight and bias gradients) against the
float64 oracle, through the C ABI, on identical seeded inputs.

* every workload at a small N spanning several token chunks plus a ragged tail;
* every workload at its full size: dx on sampled tokens (tokens are independent),
  dw / dbias on sampled output and input channels (dw[o,i,:] depends on dy[:,o,:]
  and x[:,i,:] only, so the oracle runs on those channel slices at full N);
* odd channel counts, several tiles of the weight gradient, every G, both bf16
  fused kernels for dx;
* properties: the adjoint identity <y(x), dy> = <x, dx(dy)>, determinism of the
  weight gradient, N = 0 and N = 1, argument errors.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import cyclic_group_dft_b200 as eq
import oracle
from cyclic_group_dft_b200 import workloads
from parity_util import check

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _make(wl, N, seed):
    """x, w, bias from the workload recipe, plus dy ~ N(0, 1) from a second generator."""
    x, w, bias = workloads.make_inputs(wl, seed=seed, N=N)
    g = torch.Generator().manual_seed(1000 + seed)
    dy = torch.randn(N, wl.Cout, wl.G, generator=g).to(wl.torch_dtype)
    return x, w, bias, dy


def _prep(w, bias, dtype):
    return eq.prepare(w.to(DEV), None if bias is None else bias.to(DEV), io_dtype=dtype, backward=True)


def _assert(dtype, got, ref, label):
    r = check(dtype, got, ref)
    assert r["ok"], f"{label}: {r}"


def _dw_dtype(io):
    # dw is fp32 output either way; its accuracy follows the arithmetic: the bf16
    # path rounds the spectra to bf16 (normwise bound), the fp32 path is float64
    return io


@pytest.mark.parametrize("seed", [0, 1])
@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_backward_small_n(name, seed):
    wl = workloads.WORKLOADS[name]
    N = 1031 if name != "tiny_p4_fp32" else wl.N + 37
    x, w, bias, dy = _make(wl, N, seed)
    h = _prep(w, bias, wl.torch_dtype)
    dx = h.backward_dx(dy.to(DEV))
    dw, db = h.backward_dw(x.to(DEV), dy.to(DEV))
    torch.cuda.synchronize()
    assert h.device_status() == eq.EQLIN_OK
    _assert(wl.torch_dtype, dx.cpu(), oracle.backward_dx(dy, w), f"{name} dx")
    dw_ref, db_ref = oracle.backward_dw(dy, x)
    _assert(_dw_dtype(wl.torch_dtype), dw.cpu(), dw_ref, f"{name} dw")
    _assert(_dw_dtype(wl.torch_dtype), db.cpu(), db_ref, f"{name} dbias")
    h.close()


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_backward_full_size_sampled(name):
    wl = workloads.WORKLOADS[name]
    x, w, bias, dy = _make(wl, wl.N, 0)
    h = _prep(w, bias, wl.torch_dtype)
    xd, dyd = x.to(DEV), dy.to(DEV)
    dx = h.backward_dx(dyd)
    dw, db = h.backward_dw(xd, dyd)
    torch.cuda.synchronize()
    assert h.device_status() == eq.EQLIN_OK
    idx = workloads.sample_tokens(wl.N, 512, seed=5)
    _assert(wl.torch_dtype, dx.cpu()[idx], oracle.backward_dx(dy[idx], w), f"{name} dx full N")
    rng = np.random.default_rng(9)
    osel = np.sort(rng.choice(wl.Cout, size=min(8, wl.Cout), replace=False))
    isel = np.sort(rng.choice(wl.Cin, size=min(8, wl.Cin), replace=False))
    dw_ref, db_ref = oracle.backward_dw(dy[:, osel, :], x[:, isel, :])
    got = dw.cpu()[osel][:, isel]
    _assert(_dw_dtype(wl.torch_dtype), got, dw_ref, f"{name} dw full N")
    _assert(_dw_dtype(wl.torch_dtype), db.cpu()[osel], db_ref, f"{name} dbias full N")
    h.close()


SHAPES = [  # (Cout, Cin, G): odd channel counts, several weight-gradient tiles, every G
    (8, 16, 2), (96, 96, 2), (50, 40, 4), (100, 64, 4), (200, 32, 4), (130, 96, 4),
    (24, 8, 8), (64, 64, 8), (136, 64, 8), (32, 32, 16), (16, 8, 16), (160, 16, 16),
    (128, 128, 4), (256, 96, 4), (192, 768, 4),
]


@pytest.mark.parametrize("io", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("Cout,Cin,G", SHAPES)
def test_backward_shapes(Cout, Cin, G, io):
    gen = torch.Generator().manual_seed(Cout * 1000 + Cin * 10 + G + 77)
    N = 419
    x = torch.randn(N, Cin, G, generator=gen).to(io)
    w = (torch.randn(Cout, Cin, G, generator=gen) / np.sqrt(Cin * G)).to(io)
    dy = torch.randn(N, Cout, G, generator=gen).to(io)
    h = _prep(w, None, io)
    dx = h.backward_dx(dy.to(DEV))
    dw, db = h.backward_dw(x.to(DEV), dy.to(DEV))
    torch.cuda.synchronize()
    assert h.device_status() == eq.EQLIN_OK
    _assert(io, dx.cpu(), oracle.backward_dx(dy, w), f"dx {Cout},{Cin},{G} {io}")
    dw_ref, db_ref = oracle.backward_dw(dy, x)
    _assert(io, dw.cpu(), dw_ref, f"dw {Cout},{Cin},{G} {io}")
    _assert(io, db.cpu(), db_ref, f"dbias {Cout},{Cin},{G} {io}")
    h.close()


@pytest.mark.parametrize("kernel", ["tn", "tm"])
@pytest.mark.parametrize("Cout,Cin,G", [(96, 96, 4), (64, 64, 8), (32, 32, 16), (768, 192, 4), (50, 40, 4)])
def test_backward_dx_both_fused_kernels(Cout, Cin, G, kernel, monkeypatch):
    monkeypatch.setenv("EQLIN_KERNEL", kernel)
    gen = torch.Generator().manual_seed(Cout + Cin + G)
    N = 777
    w = (torch.randn(Cout, Cin, G, generator=gen) / np.sqrt(Cin * G)).to(torch.bfloat16)
    dy = torch.randn(N, Cout, G, generator=gen).to(torch.bfloat16)
    h = _prep(w, None, torch.bfloat16)
    dx = h.backward_dx(dy.to(DEV))
    torch.cuda.synchronize()
    _assert(torch.bfloat16, dx.cpu(), oracle.backward_dx(dy, w), f"dx {Cout},{Cin},{G} {kernel}")
    h.close()


@pytest.mark.parametrize("name", ["p4_c96_bf16", "tiny_p4_fp32"])
def test_adjoint_identity_on_gpu(name):
    """<forward(x), dy> equals <x, backward_dx(dy)> (bias zero) up to rounding."""
    wl = workloads.WORKLOADS[name]
    x, w, _, dy = _make(wl, 2048, 3)
    h = _prep(w, None, wl.torch_dtype)
    y = h.forward(x.to(DEV)).double()
    dx = h.backward_dx(dy.to(DEV)).double()
    lhs = float((y * dy.to(DEV).double()).sum())
    rhs = float((x.to(DEV).double() * dx).sum())
    scale = float(y.abs().sum() * dy.abs().max()) + 1e-30
    tol = 1e-6 if wl.torch_dtype == torch.float32 else 1e-2
    assert abs(lhs - rhs) <= tol * scale, (lhs, rhs, scale)
    h.close()


def test_weight_gradient_is_deterministic():
    wl = workloads.WORKLOADS["p4_c96_bf16"]
    x, w, bias, dy = _make(wl, 65536 + 19, 4)
    h = _prep(w, bias, wl.torch_dtype)
    xd, dyd = x.to(DEV), dy.to(DEV)
    a = h.backward_dw(xd, dyd)
    b = h.backward_dw(xd, dyd)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    h.close()


@pytest.mark.parametrize("N", [0, 1, 31, 32, 33])
def test_backward_tiny_batches(N):
    wl = workloads.WORKLOADS["p4_c96_bf16"]
    x, w, bias, dy = _make(wl, max(N, 1), 6)
    x, dy = x[:N], dy[:N]
    h = _prep(w, bias, wl.torch_dtype)
    dx = h.backward_dx(dy.to(DEV))
    dw, db = h.backward_dw(x.to(DEV), dy.to(DEV))
    torch.cuda.synchronize()
    assert dx.shape == (N, wl.Cin, wl.G)
    if N == 0:
        assert not dw.any() and not db.any()
    else:
        _assert(torch.bfloat16, dx.cpu(), oracle.backward_dx(dy, w), f"dx N={N}")
        dw_ref, db_ref = oracle.backward_dw(dy, x)
        _assert(torch.bfloat16, dw.cpu(), dw_ref, f"dw N={N}")
        _assert(torch.bfloat16, db.cpu(), db_ref, f"dbias N={N}")
    h.close()


def test_backward_argument_errors():
    wl = workloads.WORKLOADS["p4_c96_bf16"]
    x, w, bias, dy = _make(wl, 256, 7)
    h = eq.prepare(w.to(DEV), bias.to(DEV))            # no backward flag
    with pytest.raises(eq.EqlinError) as e:
        h.backward_dx(dy.to(DEV))
    assert e.value.status == eq.EQLIN_ERR_INVALID_ARG
    need = eq.eqlin_backward_dw_workspace_size(h, 256)
    assert need > 0
    small = torch.empty(need - 16, dtype=torch.uint8, device=DEV)
    with pytest.raises(eq.EqlinError) as e:
        eq.eqlin_backward_dw(h, x.to(DEV), dy.to(DEV), workspace=small)
    assert e.value.status == eq.EQLIN_ERR_INVALID_ARG and "workspace" in str(e.value)
    # weight gradient needs no backward flag
    dw, db = h.backward_dw(x.to(DEV), dy.to(DEV))
    torch.cuda.synchronize()
    dw_ref, db_ref = oracle.backward_dw(dy, x)
    _assert(torch.bfloat16, dw.cpu(), dw_ref, "dw without the flag")
    h.close()


@pytest.mark.parametrize("Cout,Cin,G", [(1, 1, 8), (1, 1, 16), (2, 2, 4), (4, 4, 2), (3, 5, 8), (1024, 1024, 4),
                                        (64, 2048, 4)])
def test_backward_edge_channel_counts(Cout, Cin, G):
    """dx, dw and dbias at the fewest channels a 16-byte row allows and for large layers."""
    gen = torch.Generator().manual_seed(Cout * 5 + Cin + G)
    N = 333 if Cout * Cin < 2 ** 17 else 97
    x = torch.randn(N, Cin, G, generator=gen).to(torch.bfloat16)
    w = (torch.randn(Cout, Cin, G, generator=gen) / np.sqrt(Cin * G)).to(torch.bfloat16)
    dy = torch.randn(N, Cout, G, generator=gen).to(torch.bfloat16)
    h = _prep(w, None, torch.bfloat16)
    dx = h.backward_dx(dy.to(DEV))
    dw, db = h.backward_dw(x.to(DEV), dy.to(DEV))
    torch.cuda.synchronize()
    assert h.device_status() == eq.EQLIN_OK
    _assert(torch.bfloat16, dx.cpu(), oracle.backward_dx(dy, w), f"dx {Cout},{Cin},{G}")
    dw_ref, db_ref = oracle.backward_dw(dy, x)
    _assert(torch.bfloat16, dw.cpu(), dw_ref, f"dw {Cout},{Cin},{G}")
    _assert(torch.bfloat16, db.cpu(), db_ref, f"dbias {Cout},{Cin},{G}")
    h.close()


def test_forward_backward_and_mlp_block_replay_from_a_cuda_graph():
    """The calls a training or serving step makes -- the forward, dx, dw + dbias (two
    launches, the second a programmatic dependent) and the fused MLP block -- captured once
    into a CUDA graph on a side stream and replayed: every replay equals the calls made
    one by one, bit for bit."""
    wl = workloads.WORKLOADS["p4_c96_bf16"]
    N = 3 * 148 * 64 + 77
    x, w, bias = workloads.make_inputs(wl, seed=41, N=N)
    dev = torch.device(DEV)
    h = eq.prepare(w.to(dev), bias.to(dev), io_dtype=wl.torch_dtype, backward=True)
    H = 4 * wl.Cin
    w1, b1, w2, b2 = workloads.make_mlp_weights(wl, H)
    m = eq.eqlin_mlp_prepare(w1.to(dev), b1.to(dev), w2.to(dev), b2.to(dev))
    xd = x.to(dev)
    y = torch.empty(N, wl.Cout, wl.G, dtype=wl.torch_dtype, device=dev)
    dx = torch.empty(N, wl.Cin, wl.G, dtype=wl.torch_dtype, device=dev)
    dw = torch.empty(wl.Cout, wl.Cin, wl.G, dtype=torch.float32, device=dev)
    db = torch.empty(wl.Cout, dtype=torch.float32, device=dev)
    ym = torch.empty(N, wl.Cout, wl.G, dtype=wl.torch_dtype, device=dev)
    ws = torch.empty(max(16, eq.eqlin_backward_dw_workspace_size(h, N)), dtype=torch.uint8, device=dev)

    def step(st):
        h.forward(xd, out=y, stream=st)
        h.backward_dx(y, out=dx, stream=st)
        eq.eqlin_backward_dw(h, xd, y, stream=st, dw=dw, dbias=db, workspace=ws)
        m.forward(xd, out=ym, stream=st)

    side = torch.cuda.Stream(dev)
    step(side)
    side.synchronize()
    ref = [t.clone() for t in (y, dx, dw, db, ym)]
    for t in (y, dx, dw, db, ym):
        t.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        step(side)
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        for got, want in zip((y, dx, dw, db, ym), ref):
            assert torch.equal(got, want)
    assert h.device_status() == eq.EQLIN_OK and m.device_status() == eq.EQLIN_OK
    del g
    h.close()
    m.close()
