"""Pins for the float64 oracle, against things other than the oracle itself.

The CUDA path is judged against ``oracle``; these tests judge the oracle:

* scipy's ``linalg.circulant`` (a library definition of a circulant matrix)
  builds the naive dense block-circulant weight -- brute force;
* numpy's FFT gives the circular convolution by the convolution theorem
  (closed form, "Enfoque Algoritmico" on the page "Flash EQ-Linear: ...");
* hand-worked examples in tests/golden/hand_examples.txt;
* the p4 dyadic coefficient set, the six real products and the MAC model the
  page states (tests/golden/page_facts.txt);
* invariants: cyclic-shift equivariance ("Garantias Teoricas"), G = 1 is a
  plain linear layer (numpy matmul), zero input gives the bias, constant
  input stays constant along G.

``test_pins_reject_mutants`` plants plausible mistakes in copies of the
definition (on the CPU) and checks that each one fails at least one pin.
"""
from __future__ import annotations

import itertools
import os

import numpy as np
import pytest
import scipy.linalg

import oracle
from conftest import parse_blocks, parse_facts

RNG = np.random.default_rng(1234)

SHAPES = [  # (N, Cin, Cout, G)
    (3, 1, 1, 1), (4, 3, 2, 1), (5, 2, 3, 2), (4, 3, 2, 3), (6, 4, 5, 4),
    (3, 2, 2, 5), (4, 3, 4, 8), (2, 5, 3, 16), (7, 8, 8, 4), (3, 6, 2, 6),
]


def _rand(N, Cin, Cout, G, rng=RNG):
    return (rng.standard_normal((N, Cin, G)), rng.standard_normal((Cout, Cin, G)),
            rng.standard_normal(Cout))


# ---------------------------------------------------------------- pin functions
# Each takes a forward function f(x, w, bias) -> y and returns the worst
# relative error it finds (so mutants can be scored with the same code).

def _rel(a, b):
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


def pin_circulant(fwd) -> float:
    worst = 0.0
    for N, Cin, Cout, G in SHAPES:
        x, w, b = _rand(N, Cin, Cout, G)
        # scipy.linalg.circulant(c)[g, h] = c[(g - h) mod G]
        M = np.block([[scipy.linalg.circulant(w[o, i]) for i in range(Cin)]
                      for o in range(Cout)])
        y_ref = (x.reshape(N, Cin * G) @ M.T).reshape(N, Cout, G) + b[None, :, None]
        worst = max(worst, _rel(fwd(x, w, b), y_ref))
    return worst


def pin_fft(fwd) -> float:
    worst = 0.0
    for N, Cin, Cout, G in SHAPES:
        x, w, b = _rand(N, Cin, Cout, G)
        # convolution theorem: circular conv = ifft(fft(w) * fft(x))
        Xf = np.fft.fft(x, axis=-1)                    # [N, Cin, G]
        Wf = np.fft.fft(w, axis=-1)                    # [Cout, Cin, G]
        Yf = np.einsum("oik,nik->nok", Wf, Xf)
        y_ref = np.fft.ifft(Yf, axis=-1).real + b[None, :, None]
        worst = max(worst, _rel(fwd(x, w, b), y_ref))
    return worst


def pin_hand_examples(fwd) -> float:
    path = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.txt")
    worst = 0.0
    for blk in parse_blocks(path):
        G, Cin, Cout = int(blk["G"][0]), int(blk["Cin"][0]), int(blk["Cout"][0])
        w = np.array(blk["w"]).reshape(Cout, Cin, G)
        x = np.array(blk["x"]).reshape(-1, Cin, G)
        b = np.array(blk["bias"])
        y = np.array(blk["y"]).reshape(x.shape[0], Cout, G)
        got = fwd(x, w, b)
        worst = max(worst, float(np.abs(got - y).max()))
    return worst


def pin_equivariance(fwd) -> float:
    worst = 0.0
    for N, Cin, Cout, G in SHAPES:
        x, w, b = _rand(N, Cin, Cout, G)
        y = fwd(x, w, b)
        for s in range(G):
            ys = fwd(np.roll(x, s, axis=-1), w, b)
            worst = max(worst, _rel(ys, np.roll(y, s, axis=-1)))
    return worst


def pin_special_cases(fwd) -> float:
    worst = 0.0
    for N, Cin, Cout, G in SHAPES:
        x, w, b = _rand(N, Cin, Cout, G)
        # zero input -> bias everywhere
        y0 = fwd(np.zeros_like(x), w, b)
        worst = max(worst, float(np.abs(y0 - b[None, :, None]).max()))
        # constant along G -> constant along G, equal to (sum_m w) . x + b
        xc = np.repeat(x[:, :, :1], G, axis=-1)
        yc = fwd(xc, w, b)
        ref = x[:, :, 0] @ w.sum(-1).T + b
        worst = max(worst, _rel(yc, np.repeat(ref[:, :, None], G, axis=-1)))
        # filter supported at m = 0 only -> independent linear map per g
        w0 = np.zeros_like(w)
        w0[:, :, 0] = w[:, :, 0]
        yd = fwd(x, w0, b)
        ref = np.einsum("nig,oi->nog", x, w[:, :, 0]) + b[None, :, None]
        worst = max(worst, _rel(yd, ref))
    # G = 1 is a plain linear layer
    x, w, b = _rand(9, 7, 5, 1)
    worst = max(worst, _rel(fwd(x, w, b)[:, :, 0], x[:, :, 0] @ w[:, :, 0].T + b))
    return worst


PINS = {
    "circulant": (pin_circulant, 1e-12),
    "fft": (pin_fft, 1e-12),
    "hand": (pin_hand_examples, 1e-12),
    "equivariance": (pin_equivariance, 1e-12),
    "special": (pin_special_cases, 1e-12),
}


# ----------------------------------------------------------------- the oracle

@pytest.mark.parametrize("pin", sorted(PINS))
def test_definition_passes_pin(pin):
    fn, tol = PINS[pin]
    assert fn(oracle.forward) <= tol


@pytest.mark.parametrize("pin", sorted(PINS))
def test_fourier_path_passes_pin(pin):
    fn, tol = PINS[pin]
    assert fn(oracle.forward_fourier) <= tol


def test_dense_weight_is_block_circulant():
    for _, Cin, Cout, G in SHAPES:
        w = RNG.standard_normal((Cout, Cin, G))
        M = oracle.dense_weight(w)
        ref = np.block([[scipy.linalg.circulant(w[o, i]) for i in range(Cin)]
                        for o in range(Cout)])
        assert np.array_equal(M, ref)


def test_dense_product_matches_definition():
    for N, Cin, Cout, G in SHAPES:
        x, w, b = _rand(N, Cin, Cout, G)
        M = oracle.dense_weight(w)
        y = (x.reshape(N, -1) @ M.T).reshape(N, Cout, G) + b[None, :, None]
        assert _rel(oracle.forward(x, w, b), y) < 1e-13


def test_fourier_path_equals_definition():
    for N, Cin, Cout, G in SHAPES:
        x, w, b = _rand(N, Cin, Cout, G)
        assert _rel(oracle.forward_fourier(x, w, b), oracle.forward(x, w, b)) < 1e-12


def test_none_bias_is_zero():
    x, w, b = _rand(4, 3, 2, 4)
    assert np.array_equal(oracle.forward(x, w, None), oracle.forward(x, w, np.zeros(2)))


def test_empty_batch():
    x = np.zeros((0, 3, 4))
    w = RNG.standard_normal((2, 3, 4))
    assert oracle.forward(x, w, None).shape == (0, 2, 4)
    assert oracle.forward_fourier(x, w, None).shape == (0, 2, 4)


def test_thread_count_does_not_change_result():
    x, w, b = _rand(64, 5, 3, 8)
    y1 = oracle.forward(x, w, b, threads=1)
    y4 = oracle.forward(x, w, b, threads=4)
    assert np.array_equal(y1, y4)


def test_bad_arguments_are_rejected():
    with pytest.raises(ValueError):
        oracle.forward(np.zeros((2, 3, 4)), np.zeros((2, 5, 4)), None)


# ------------------------------------------------------- DFT and page facts

@pytest.mark.parametrize("G", [1, 2, 3, 4, 5, 8, 16])
def test_rdft_matches_numpy_rfft(G):
    v = RNG.standard_normal((6, G))
    re, im = oracle.rdft(v)
    ref = np.fft.rfft(v, axis=-1) / np.sqrt(G)
    assert np.abs(re - ref.real).max() < 1e-13
    assert np.abs(im - ref.imag).max() < 1e-13


@pytest.mark.parametrize("G", [1, 2, 3, 4, 5, 8, 16])
def test_half_spectrum_is_hermitian_and_invertible(G):
    v = RNG.standard_normal((6, G))
    full = np.fft.fft(v, axis=-1) / np.sqrt(G)
    for k in range(1, G):
        assert np.abs(full[:, G - k] - np.conj(full[:, k])).max() < 1e-13
    re, im = oracle.rdft(v)
    assert np.abs(oracle.irdft(re, im, G) - v).max() < 1e-13


def _p4_matrices():
    G = 4
    eye = np.eye(G)
    re, im = oracle.rdft(eye)             # column h of the forward matrix
    K = G // 2 + 1
    fwd = np.empty((2 * K, G))
    fwd[0::2], fwd[1::2] = re.T, im.T    # rows: Re X_k, Im X_k
    inv = np.empty((G, 2 * K))
    for j in range(2 * K):               # column j of the inverse matrix
        s = np.zeros(2 * K)
        s[j] = 1.0
        inv[:, j] = oracle.irdft(s[0::2][None], s[1::2][None], G)[0]
    return fwd, inv


def test_p4_transform_coefficients_are_dyadic(golden_dir):
    facts = parse_facts(os.path.join(golden_dir, "page_facts.txt"))
    allowed = np.array(facts["p4_transform_entries"])
    fwd, inv = _p4_matrices()
    # drop the identically-zero rows/columns (Im of the real frequencies)
    K = 3
    fwd_used = np.delete(fwd, [1, 2 * K - 1], axis=0)
    inv_used = np.delete(inv, [1, 2 * K - 1], axis=1)
    entries = np.concatenate([fwd_used.ravel(), inv_used.ravel()])
    dist = np.abs(entries[:, None] - allowed[None, :]).min(axis=1)
    assert dist.max() < 1e-15
    # and every coefficient of the stated set actually occurs
    for a in allowed:
        assert np.abs(entries - a).min() < 1e-15


def test_operation_counts_match_page(golden_dir):
    facts = parse_facts(os.path.join(golden_dir, "page_facts.txt"))
    assert oracle.fourier_real_gemm_blocks(4) == facts["p4_real_matrix_products"][0]
    gain = oracle.dense_flops(1, 1, 1, 4) / oracle.fourier_flops(1, 1, 1, 4)
    assert gain == pytest.approx(16 / 6)
    assert round(gain, 2) == facts["p4_theoretical_gain"][0]
    # MAC ratio (Fourier / naive) approaches 2/T for large T
    for G in (64, 256, 1024):
        r = oracle.fourier_flops(1, 1, 1, G) / oracle.dense_flops(1, 1, 1, G)
        assert r * G == pytest.approx(facts["mac_ratio_asymptote_times_T"][0], rel=2.0 / G)
    # the page's 0.134 GFLOP naive figure is 2^27 exactly (e.g. 256 tokens,
    # Cin*G = Cout*G = 512); the 6/16 Fourier share of it is ~0.050 GFLOP and
    # the page's 0.052 G (x2.6) leaves ~0.002 G for the transforms and bias.
    naive = oracle.dense_flops(256, 128, 128, 4)
    assert naive / 1e9 == pytest.approx(facts["naive_gflops"][0], abs=5e-4)
    fourier = oracle.fourier_flops(256, 128, 128, 4)
    assert fourier < facts["flash_gflops"][0] * 1e9 < 1.05 * fourier
    assert naive / (facts["flash_gflops"][0] * 1e9) == pytest.approx(
        facts["flop_reduction"][0], abs=0.05)


# ------------------------------------------------------------ mutant check

def _conv_loop(x, w, b, index, use_bias=True, h_range=None):
    N, Cin, G = x.shape
    Cout = w.shape[0]
    y = np.zeros((N, Cout, G))
    hs = range(G) if h_range is None else h_range(G)
    for o, g in itertools.product(range(Cout), range(G)):
        acc = np.zeros(N)
        for i in range(Cin):
            for h in hs:
                acc += w[o, i, index(g, h, G)] * x[:, i, h]
        y[:, o, g] = acc + (b[o] if use_bias else 0.0)
    return y


MUTANTS = {
    # correlation instead of convolution (wrong shift sign)
    "correlation": lambda x, w, b: _conv_loop(x, w, b, lambda g, h, G: (h - g) % G),
    # off-by-one shift
    "off_by_one": lambda x, w, b: _conv_loop(x, w, b, lambda g, h, G: (g - h + 1) % G),
    # bias dropped
    "no_bias": lambda x, w, b: _conv_loop(x, w, b, lambda g, h, G: (g - h) % G, use_bias=False),
    # last group element dropped from the sum
    "dropped_term": lambda x, w, b: _conv_loop(
        x, w, b, lambda g, h, G: (g - h) % G, h_range=lambda G: range(max(G - 1, 1))),
    # filter index taken from h alone (no circulant structure)
    "no_shift": lambda x, w, b: _conv_loop(x, w, b, lambda g, h, G: h % G),
    # output and input channels swapped in the weight (square shapes only)
    "transposed_channels": lambda x, w, b: (
        _conv_loop(x, np.swapaxes(w, 0, 1), b, lambda g, h, G: (g - h) % G)
        if w.shape[0] == w.shape[1] else np.full((x.shape[0], w.shape[0], x.shape[2]), np.nan)),
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_reject_mutants(mutant):
    fwd = MUTANTS[mutant]
    failed = []
    for name, (fn, tol) in PINS.items():
        with np.errstate(all="ignore"):
            err = fn(fwd)
        if not (err <= tol):
            failed.append(name)
    assert failed, f"mutant {mutant} passed every pin"
