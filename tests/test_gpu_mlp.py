"""GPU parity of the GELU epilogue and of the equivariant MLP block
y = L2(GELU(L1(x))) (two forwards, the first prepared with activation="gelu")
against the float64 oracle, through the C ABI, on identical seeded inputs.

Tolerance of the block.  The two-launch block stores the hidden activation in the
I/O dtype, so for fp32 I/O the reference rounds the oracle's float64 hidden activation
to fp32 as well and the 1e-5 bound of one layer applies to the second layer's output;
against the all-float64 oracle the fp32 block is held to a normwise 1e-6 (the floored
elementwise metric turns the 2^-24 rounding of ~H*G hidden values into ~1.6e-5 at the
outputs nearest zero).  For 16-bit I/O each layer contributes its own rounding (spectra,
the stored hidden activation, the output), so the derived normwise bound of one layer
is doubled (bf16 1.2e-2, fp16 3e-3), still inside the 2e-2 specification bound.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import cyclic_group_dft_b200 as eq
import oracle
from parity_util import BF16_DERIVED, F16_DERIVED, TOL_BF16_NORMWISE, check, f32_maxrel, normwise

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _block(N, Cin, H, Cout, G, io, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(N, Cin, G, generator=g).to(io)
    w1 = (torch.randn(H, Cin, G, generator=g) / np.sqrt(Cin * G)).to(io)
    b1 = (torch.randn(H, generator=g) * 0.3).to(io)
    w2 = (torch.randn(Cout, H, G, generator=g) / np.sqrt(H * G)).to(io)
    b2 = (torch.randn(Cout, generator=g) * 0.3).to(io)
    return x, w1, b1, w2, b2


@pytest.mark.parametrize("io", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("Cout,Cin,G", [(96, 96, 4), (64, 64, 8), (32, 32, 16), (50, 40, 4), (200, 32, 4)])
def test_gelu_epilogue(Cout, Cin, G, io):
    x, w, b, _, _ = _block(517, Cin, Cout, Cout, G, io, Cout + Cin + G)
    h = eq.prepare(w.to(DEV), b.to(DEV), io_dtype=io, activation="gelu")
    assert h.attr("activation") == 1
    y = h.forward(x.to(DEV))
    torch.cuda.synchronize()
    assert h.device_status() == eq.EQLIN_OK
    ref = oracle.gelu(oracle.forward(x, w, b))
    r = check(io, y.cpu(), ref)
    assert r["ok"], r
    h.close()


@pytest.mark.parametrize("io", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("Cin,H,Cout,G", [(96, 384, 96, 4), (64, 256, 64, 8), (32, 128, 32, 16), (48, 80, 24, 2)])
def test_mlp_block(Cin, H, Cout, G, io):
    x, w1, b1, w2, b2 = _block(1031, Cin, H, Cout, G, io, Cin * 7 + H + G)
    h1 = eq.prepare(w1.to(DEV), b1.to(DEV), io_dtype=io, activation="gelu")
    h2 = eq.prepare(w2.to(DEV), b2.to(DEV), io_dtype=io)
    y = eq.mlp_block(h1, h2, x.to(DEV))
    torch.cuda.synchronize()
    assert h1.device_status() == eq.EQLIN_OK and h2.device_status() == eq.EQLIN_OK
    ref = oracle.mlp_forward(x, w1, b1, w2, b2)
    got = y.float().cpu().numpy()
    if io == torch.float32:
        hidden32 = oracle.gelu(oracle.forward(x, w1, b1)).astype(np.float32)
        assert f32_maxrel(got, oracle.forward(hidden32, w2, b2)) <= 1e-5
        assert normwise(got, ref) <= 1e-6
    else:
        bound = 2 * (F16_DERIVED if io == torch.float16 else BF16_DERIVED)
        err = normwise(got, ref)
        assert err <= min(bound, TOL_BF16_NORMWISE), err
    h1.close()
    h2.close()


def test_mlp_block_is_equivariant_on_gpu():
    x, w1, b1, w2, b2 = _block(512, 96, 384, 96, 4, torch.float32, 5)
    h1 = eq.prepare(w1.to(DEV), b1.to(DEV), activation="gelu")
    h2 = eq.prepare(w2.to(DEV), b2.to(DEV))
    y = eq.mlp_block(h1, h2, x.to(DEV)).cpu().double().numpy()
    for s in range(4):
        ys = eq.mlp_block(h1, h2, torch.roll(x, s, dims=-1).to(DEV)).cpu().double().numpy()
        assert np.abs(ys - np.roll(y, s, axis=-1)).max() <= 1e-5 * np.abs(y).max()
    h1.close()
    h2.close()


def test_mlp_block_rejects_mismatched_handles():
    x, w1, b1, w2, b2 = _block(16, 96, 384, 96, 4, torch.bfloat16, 6)
    plain = eq.prepare(w1.to(DEV), b1.to(DEV))
    h2 = eq.prepare(w2.to(DEV), b2.to(DEV))
    with pytest.raises(ValueError):
        eq.mlp_block(plain, h2, x.to(DEV))          # first layer without GELU
    h1 = eq.prepare(w1.to(DEV), b1.to(DEV), activation="gelu")
    with pytest.raises(ValueError):
        eq.mlp_block(h1, h1, x.to(DEV))             # 384 outputs into a 96-input layer
    for h in (plain, h2, h1):
        h.close()
