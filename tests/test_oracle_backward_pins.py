"""Pins for the oracle's backward pass (gradients with respect to x, w, bias).

The backward functions are checked against things other than themselves:

* torch autograd in float64 through a dense block-circulant weight built by
  index arithmetic (the chain rule done by a library);
* scipy's ``linalg.circulant``: dx is the transposed dense matrix applied to dy;
* numpy's FFT: dx is a circular correlation, dX_k = sum_o conj(W_k) dY_k, and
  dW_k = sum_n dY_k conj(X_k) (the conjugate form of the convolution theorem
  of section "Enfoque Algoritmico" on the page "Flash EQ-Linear: ...");
* central finite differences of the pinned forward oracle (the loss is linear
  in x and w, so the differences are exact up to rounding);
* hand-worked examples in tests/golden/hand_backward.txt;
* invariants: the adjoint identity <y(x), dy> = <x, dx(dy)>, cyclic-shift
  equivariance of dx, G = 1 reduces to the plain linear layer's gradients.

``test_backward_pins_reject_mutants`` plants plausible mistakes in copies of
the backward definition (on the CPU) and checks each fails at least one pin.
"""
from __future__ import annotations

import itertools
import os

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from conftest import parse_blocks

RNG = np.random.default_rng(4321)

SHAPES = [  # (N, Cin, Cout, G)
    (3, 1, 1, 1), (4, 3, 2, 1), (5, 2, 3, 2), (4, 3, 2, 3), (6, 4, 5, 4),
    (3, 2, 2, 5), (4, 3, 4, 8), (2, 5, 3, 16), (7, 8, 8, 4), (3, 6, 2, 6),
]


def _rand(N, Cin, Cout, G, rng=RNG):
    return (rng.standard_normal((N, Cin, G)), rng.standard_normal((Cout, Cin, G)),
            rng.standard_normal((N, Cout, G)))


def _rel(a, b):
    a, b = np.asarray(a), np.asarray(b)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


# A backward implementation is a pair bwd = (dx_fn(dy, w), dw_fn(dy, x)).
ORACLE_BWD = (oracle.backward_dx, oracle.backward_dw)


def pin_autograd(bwd) -> float:
    dx_fn, dw_fn = bwd
    worst = 0.0
    for N, Cin, Cout, G in SHAPES:
        x, w, dy = _rand(N, Cin, Cout, G)
        xt = torch.tensor(x, requires_grad=True)
        wt = torch.tensor(w, requires_grad=True)
        bt = torch.zeros(Cout, dtype=torch.float64, requires_grad=True)
        g = torch.arange(G)
        idx = (g[:, None] - g[None, :]) % G                      # [g, h] -> (g-h) mod G
        M = wt[:, :, idx]                                         # [Cout, Cin, G(g), G(h)]
        M = M.permute(0, 2, 1, 3).reshape(Cout * G, Cin * G)
        y = (xt.reshape(N, Cin * G) @ M.T).reshape(N, Cout, G) + bt[None, :, None]
        (y * torch.tensor(dy)).sum().backward()
        dw, db = dw_fn(dy, x)
        worst = max(worst, _rel(dx_fn(dy, w), xt.grad.numpy()), _rel(dw, wt.grad.numpy()),
                    _rel(db, bt.grad.numpy()))
    return worst


def pin_circulant(bwd) -> float:
    dx_fn, _ = bwd
    worst = 0.0
    for N, Cin, Cout, G in SHAPES:
        x, w, dy = _rand(N, Cin, Cout, G)
        # scipy.linalg.circulant(c)[g, h] = c[(g - h) mod G]
        M = np.block([[scipy.linalg.circulant(w[o, i]) for i in range(Cin)]
                      for o in range(Cout)])
        dx_ref = (dy.reshape(N, Cout * G) @ M).reshape(N, Cin, G)
        worst = max(worst, _rel(dx_fn(dy, w), dx_ref))
    return worst


def pin_fft(bwd) -> float:
    dx_fn, dw_fn = bwd
    worst = 0.0
    for N, Cin, Cout, G in SHAPES:
        x, w, dy = _rand(N, Cin, Cout, G)
        Xf, Wf, Yf = (np.fft.fft(a, axis=-1) for a in (x, w, dy))
        dx_ref = np.fft.ifft(np.einsum("oik,nok->nik", np.conj(Wf), Yf), axis=-1).real
        dw_ref = np.fft.ifft(np.einsum("nok,nik->oik", Yf, np.conj(Xf)), axis=-1).real
        dw, db = dw_fn(dy, x)
        worst = max(worst, _rel(dx_fn(dy, w), dx_ref), _rel(dw, dw_ref),
                    _rel(db, dy.sum(axis=(0, 2))))
    return worst


def pin_finite_difference(bwd) -> float:
    dx_fn, dw_fn = bwd
    worst = 0.0
    for N, Cin, Cout, G in [(2, 2, 3, 4), (3, 3, 2, 3), (2, 2, 2, 8)]:
        x, w, dy = _rand(N, Cin, Cout, G)
        b = RNG.standard_normal(Cout)

        def loss(xx, ww, bb):
            return float((oracle.forward(xx, ww, bb) * dy).sum())

        eps = 0.5  # the loss is affine in each argument: any step is exact
        gx = np.zeros_like(x)
        for k in np.ndindex(*x.shape):
            e = np.zeros_like(x)
            e[k] = eps
            gx[k] = (loss(x + e, w, b) - loss(x - e, w, b)) / (2 * eps)
        gw = np.zeros_like(w)
        for k in np.ndindex(*w.shape):
            e = np.zeros_like(w)
            e[k] = eps
            gw[k] = (loss(x, w + e, b) - loss(x, w - e, b)) / (2 * eps)
        gb = np.array([(loss(x, w, b + eps * np.eye(Cout)[o]) - loss(x, w, b - eps * np.eye(Cout)[o]))
                       / (2 * eps) for o in range(Cout)])
        dw, db = dw_fn(dy, x)
        worst = max(worst, _rel(dx_fn(dy, w), gx), _rel(dw, gw), _rel(db, gb))
    return worst


def pin_hand_examples(bwd) -> float:
    dx_fn, dw_fn = bwd
    path = os.path.join(os.path.dirname(__file__), "golden", "hand_backward.txt")
    worst = 0.0
    for blk in parse_blocks(path):
        G, Cin, Cout = int(blk["G"][0]), int(blk["Cin"][0]), int(blk["Cout"][0])
        w = np.array(blk["w"]).reshape(Cout, Cin, G)
        x = np.array(blk["x"]).reshape(-1, Cin, G)
        dy = np.array(blk["dy"]).reshape(-1, Cout, G)
        dw, db = dw_fn(dy, x)
        worst = max(worst,
                    float(np.abs(dx_fn(dy, w) - np.array(blk["dx"]).reshape(x.shape)).max()),
                    float(np.abs(dw - np.array(blk["dw"]).reshape(w.shape)).max()),
                    float(np.abs(db - np.array(blk["dbias"])).max()))
    return worst


def pin_invariants(bwd) -> float:
    dx_fn, dw_fn = bwd
    worst = 0.0
    for N, Cin, Cout, G in SHAPES:
        x, w, dy = _rand(N, Cin, Cout, G)
        dx = dx_fn(dy, w)
        # adjoint identity: <W x, dy> = <x, W^T dy>
        lhs = float((oracle.forward(x, w) * dy).sum())
        rhs = float((x * dx).sum())
        worst = max(worst, abs(lhs - rhs) / max(abs(lhs), 1.0))
        # dx commutes with cyclic shifts along the group axis
        for s in range(G):
            worst = max(worst, _rel(dx_fn(np.roll(dy, s, axis=-1), w), np.roll(dx, s, axis=-1)))
        # dw, summed over its group index, is the G=1 weight gradient of the
        # group-summed signals (sum_m dw[o,i,m] = sum_n (sum_g dy)(sum_h x))
        dw, _ = dw_fn(dy, x)
        worst = max(worst, _rel(dw.sum(-1), dy.sum(-1).T @ x.sum(-1)))
    # G = 1: the plain linear layer y = x W^T
    x, w, dy = _rand(6, 5, 4, 1)
    dw, db = dw_fn(dy, x)
    worst = max(worst, _rel(dx_fn(dy, w)[:, :, 0], dy[:, :, 0] @ w[:, :, 0]),
                _rel(dw[:, :, 0], dy[:, :, 0].T @ x[:, :, 0]), _rel(db, dy[:, :, 0].sum(0)))
    return worst


PINS = {
    "autograd": (pin_autograd, 1e-12),
    "circulant": (pin_circulant, 1e-12),
    "fft": (pin_fft, 1e-12),
    "finite_difference": (pin_finite_difference, 1e-9),
    "hand": (pin_hand_examples, 1e-12),
    "invariants": (pin_invariants, 1e-12),
}


@pytest.mark.parametrize("pin", sorted(PINS))
def test_backward_oracle_passes_pin(pin):
    fn, tol = PINS[pin]
    err = fn(ORACLE_BWD)
    assert err <= tol, f"pin {pin}: {err}"


def test_backward_empty_batch():
    w = RNG.standard_normal((3, 2, 4))
    assert oracle.backward_dx(np.zeros((0, 3, 4)), w).shape == (0, 2, 4)
    dw, db = oracle.backward_dw(np.zeros((0, 3, 4)), np.zeros((0, 2, 4)))
    assert not dw.any() and not db.any()


def test_backward_thread_count_does_not_change_result():
    x, w, dy = _rand(37, 6, 5, 8)
    assert np.array_equal(oracle.backward_dx(dy, w, threads=1), oracle.backward_dx(dy, w, threads=4))
    a = oracle.backward_dw(dy, x, threads=1)
    b = oracle.backward_dw(dy, x, threads=4)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_backward_bad_arguments_are_rejected():
    with pytest.raises(ValueError):
        oracle.backward_dx(np.zeros((2, 3, 4)), np.zeros((2, 3, 4)))
    with pytest.raises(ValueError):
        oracle.backward_dw(np.zeros((2, 3, 4)), np.zeros((3, 3, 4)))


# ------------------------------------------------------------ mutant check

def _dx_loop(dy, w, index):
    N, Cout, G = dy.shape
    Cin = w.shape[1]
    dx = np.zeros((N, Cin, G))
    for i, h in itertools.product(range(Cin), range(G)):
        for o in range(Cout):
            for g in range(G):
                dx[:, i, h] += w[o, i, index(g, h, G)] * dy[:, o, g]
    return dx


def _dw_loop(dy, x, index, with_bias=True, tokens=None):
    N, Cout, G = dy.shape
    Cin = x.shape[1]
    ns = slice(None) if tokens is None else tokens(N)
    dw = np.zeros((Cout, Cin, G))
    for o, i, m in itertools.product(range(Cout), range(Cin), range(G)):
        dw[o, i, m] = sum((dy[ns, o, g] * x[ns, i, index(g, m, G)]).sum() for g in range(G))
    db = dy[ns].sum(axis=(0, 2)) if with_bias else np.zeros(Cout)
    return dw, db


_DX_OK = lambda dy, w: _dx_loop(dy, w, lambda g, h, G: (g - h) % G)  # noqa: E731
_DW_OK = lambda dy, x: _dw_loop(dy, x, lambda g, m, G: (g - m) % G)  # noqa: E731

BACKWARD_MUTANTS = {
    # dx taken as a convolution (forward index) instead of the correlation
    "dx_convolution": (lambda dy, w: _dx_loop(dy, w, lambda g, h, G: (h - g) % G), _DW_OK),
    # dx with the weight's group axis not shifted at all
    "dx_no_shift": (lambda dy, w: _dx_loop(dy, w, lambda g, h, G: g % G), _DW_OK),
    # dw with the shift the wrong way round
    "dw_wrong_shift": (_DX_OK, lambda dy, x: _dw_loop(dy, x, lambda g, m, G: (g + m) % G)),
    # dw off by one
    "dw_off_by_one": (_DX_OK, lambda dy, x: _dw_loop(dy, x, lambda g, m, G: (g - m + 1) % G)),
    # dbias not computed
    "dbias_dropped": (_DX_OK, lambda dy, x: _dw_loop(dy, x, lambda g, m, G: (g - m) % G,
                                                     with_bias=False)),
    # last token dropped from the reduction over the batch
    "dw_dropped_token": (_DX_OK, lambda dy, x: _dw_loop(dy, x, lambda g, m, G: (g - m) % G,
                                                        tokens=lambda N: slice(0, max(N - 1, 1)))),
    # dx through the forward weight (no transpose): only shapes Cin == Cout run
    "dx_untransposed": (lambda dy, w: (_dx_loop(dy, np.swapaxes(w, 0, 1), lambda g, h, G: (h - g) % G)
                                       if w.shape[0] == w.shape[1] else
                                       np.full((dy.shape[0], w.shape[1], dy.shape[2]), np.nan)), _DW_OK),
}


def test_mutant_helpers_reproduce_the_oracle():
    x, w, dy = _rand(4, 3, 2, 4)
    assert _rel(_DX_OK(dy, w), oracle.backward_dx(dy, w)) < 1e-13
    a, b = _DW_OK(dy, x), oracle.backward_dw(dy, x)
    assert _rel(a[0], b[0]) < 1e-13 and _rel(a[1], b[1]) < 1e-13


@pytest.mark.parametrize("mutant", sorted(BACKWARD_MUTANTS))
def test_backward_pins_reject_mutants(mutant):
    bwd = BACKWARD_MUTANTS[mutant]
    failed = []
    for name, (fn, tol) in PINS.items():
        if name == "finite_difference":
            continue  # slow; the other pins are enough to score the mutants
        with np.errstate(all="ignore"):
            err = fn(bwd)
        if not (err <= tol):
            failed.append(name)
    assert failed, f"mutant {mutant} passed every pin"
