"""CPU float64 oracle for EQ-Linear over the cyclic group C_G.

TEST INFRASTRUCTURE ONLY.  This package is the slow, obviously-correct
reference the CUDA path is checked against.  Only the tests, the package
smoke check (``__graft_entry__.smoke``) and the CPU-baseline leg of
``bench.py`` may import it; the product package never does, and this package
never imports the product.

The arithmetic lives in ``eqlin_oracle.c`` (plain C, float64 loops); this
module only marshals numpy arrays to it.  Functions:

* :func:`forward`          -- the definition, y = bias + block-circulant(w) x
  (page "Flash EQ-Linear: ...", section "Percepcion Central");
* :func:`dense_weight`     -- the naive replicated dense matrix
  (section "Declaracion del Problema");
* :func:`rdft`, :func:`irdft` -- unitary real DFT along the group axis,
  half spectrum (section "Enfoque Algoritmico", conjugate symmetry);
* :func:`forward_fourier`  -- the method's algorithm: DFT, per-frequency
  complex contraction, inverse DFT, bias (section "Enfoque Algoritmico");
* :func:`backward_dx`, :func:`backward_dw` -- the gradients of a loss with
  respect to x, and to w and bias, by the chain rule on the definition (the
  backward pass of section "Implementacion");
* :func:`gelu`, :func:`mlp_forward` -- the MLP block y = L2(GELU(L1(x))) of the
  network-level results (section "A Nivel de Red"), GELU(v) = v * Phi(v);
* :func:`dense_flops`, :func:`fourier_flops` -- the operation counts of the
  naive and the Fourier-domain contraction (sections "Enfoque Algoritmico",
  "Especializacion para el Grupo de Rotacion p4").
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        i64, dp, ip = ctypes.c_int64, ctypes.POINTER(ctypes.c_double), ctypes.c_int
        lib.eqlin_oracle_forward_f64.argtypes = [dp, dp, dp, i64, i64, i64, i64, dp, ip]
        lib.eqlin_oracle_forward_fourier_f64.argtypes = [dp, dp, dp, i64, i64, i64, i64, dp, ip]
        lib.eqlin_oracle_dense_weight_f64.argtypes = [dp, i64, i64, i64, dp]
        lib.eqlin_oracle_rdft_f64.argtypes = [dp, i64, i64, dp, dp]
        lib.eqlin_oracle_irdft_f64.argtypes = [dp, dp, i64, i64, dp]
        lib.eqlin_oracle_backward_dx_f64.argtypes = [dp, dp, i64, i64, i64, i64, dp, ip]
        lib.eqlin_oracle_backward_dw_f64.argtypes = [dp, dp, i64, i64, i64, i64, dp, dp, ip]
        lib.eqlin_oracle_gelu_f64.argtypes = [dp, i64, dp]
        lib.eqlin_oracle_mlp_f64.argtypes = [dp, dp, dp, dp, dp, i64, i64, i64, i64, i64, dp, ip]
        lib.eqlin_oracle_num_freqs.argtypes = [i64]
        lib.eqlin_oracle_num_freqs.restype = i64
        lib.eqlin_oracle_max_threads.restype = ctypes.c_int
        for f in ("eqlin_oracle_forward_f64", "eqlin_oracle_forward_fourier_f64",
                  "eqlin_oracle_dense_weight_f64", "eqlin_oracle_rdft_f64",
                  "eqlin_oracle_irdft_f64", "eqlin_oracle_backward_dx_f64",
                  "eqlin_oracle_backward_dw_f64", "eqlin_oracle_gelu_f64", "eqlin_oracle_mlp_f64"):
            getattr(lib, f).restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    """Any array-like (numpy, torch CPU tensor of any float dtype) -> contiguous float64."""
    if hasattr(a, "detach"):  # torch tensor: upcast exactly (bf16/fp32 -> f64)
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def max_threads() -> int:
    """Threads an OpenMP region of the oracle uses by default."""
    return int(_load().eqlin_oracle_max_threads())


def _check(status: int, what: str) -> None:
    if status != 0:
        raise ValueError(f"oracle {what} rejected its arguments (status {status})")


def forward(x, w, bias=None, threads: int = 0) -> np.ndarray:
    """Definition of EQ-Linear in float64.

    x [N, Cin, G], w [Cout, Cin, G], bias [Cout] or None -> y [N, Cout, G].
    """
    x, w = _f64(x), _f64(w)
    N, Cin, G = x.shape
    Cout = w.shape[0]
    if w.shape != (Cout, Cin, G):
        raise ValueError(f"w shape {w.shape} does not match x shape {x.shape}")
    b = None if bias is None else _f64(bias).reshape(Cout)
    y = np.empty((N, Cout, G), dtype=np.float64)
    st = _load().eqlin_oracle_forward_f64(
        _ptr(x), _ptr(w), None if b is None else _ptr(b), N, Cin, Cout, G, _ptr(y), int(threads))
    _check(st, "forward")
    return y


def forward_fourier(x, w, bias=None, threads: int = 0) -> np.ndarray:
    """The method's algorithm (rDFT, per-frequency contraction, irDFT) in float64."""
    x, w = _f64(x), _f64(w)
    N, Cin, G = x.shape
    Cout = w.shape[0]
    if w.shape != (Cout, Cin, G):
        raise ValueError(f"w shape {w.shape} does not match x shape {x.shape}")
    b = None if bias is None else _f64(bias).reshape(Cout)
    y = np.empty((N, Cout, G), dtype=np.float64)
    st = _load().eqlin_oracle_forward_fourier_f64(
        _ptr(x), _ptr(w), None if b is None else _ptr(b), N, Cin, Cout, G, _ptr(y), int(threads))
    _check(st, "forward_fourier")
    return y


def backward_dx(dy, w, threads: int = 0) -> np.ndarray:
    """Gradient with respect to x: dx[n,i,h] = sum_{o,g} w[o,i,(g-h) mod G] dy[n,o,g].

    dy [N, Cout, G], w [Cout, Cin, G] -> dx [N, Cin, G], float64.
    """
    dy, w = _f64(dy), _f64(w)
    N, Cout, G = dy.shape
    Cin = w.shape[1]
    if w.shape != (Cout, Cin, G):
        raise ValueError(f"w shape {w.shape} does not match dy shape {dy.shape}")
    dx = np.empty((N, Cin, G), dtype=np.float64)
    st = _load().eqlin_oracle_backward_dx_f64(_ptr(dy), _ptr(w), N, Cin, Cout, G, _ptr(dx), int(threads))
    _check(st, "backward_dx")
    return dx


def backward_dw(dy, x, threads: int = 0) -> tuple[np.ndarray, np.ndarray]:
    """Gradients with respect to w and bias:
    dw[o,i,m] = sum_{n,g} dy[n,o,g] x[n,i,(g-m) mod G], dbias[o] = sum_{n,g} dy[n,o,g].

    dy [N, Cout, G], x [N, Cin, G] -> (dw [Cout, Cin, G], dbias [Cout]), float64.
    """
    dy, x = _f64(dy), _f64(x)
    N, Cout, G = dy.shape
    if x.shape[0] != N or x.shape[2] != G:
        raise ValueError(f"x shape {x.shape} does not match dy shape {dy.shape}")
    Cin = x.shape[1]
    dw = np.empty((Cout, Cin, G), dtype=np.float64)
    db = np.empty((Cout,), dtype=np.float64)
    st = _load().eqlin_oracle_backward_dw_f64(_ptr(dy), _ptr(x), N, Cin, Cout, G, _ptr(dw), _ptr(db),
                                              int(threads))
    _check(st, "backward_dw")
    return dw, db


def gelu(v) -> np.ndarray:
    """GELU(v) = v * Phi(v) elementwise, Phi the standard normal CDF (erf form), float64."""
    v = _f64(v)
    out = np.empty_like(v)
    _check(_load().eqlin_oracle_gelu_f64(_ptr(v), v.size, _ptr(out)), "gelu")
    return out


def mlp_forward(x, w1, b1, w2, b2, threads: int = 0) -> np.ndarray:
    """MLP block y = L2(GELU(L1(x))): x [N, Cin, G], w1 [H, Cin, G], b1 [H] or None,
    w2 [Cout, H, G], b2 [Cout] or None -> y [N, Cout, G], float64."""
    x, w1, w2 = _f64(x), _f64(w1), _f64(w2)
    N, Cin, G = x.shape
    H, Cout = w1.shape[0], w2.shape[0]
    if w1.shape != (H, Cin, G) or w2.shape != (Cout, H, G):
        raise ValueError("w1 must be [H, Cin, G] and w2 [Cout, H, G]")
    c1 = None if b1 is None else _f64(b1).reshape(H)
    c2 = None if b2 is None else _f64(b2).reshape(Cout)
    y = np.empty((N, Cout, G), dtype=np.float64)
    st = _load().eqlin_oracle_mlp_f64(_ptr(x), _ptr(w1), None if c1 is None else _ptr(c1), _ptr(w2),
                                      None if c2 is None else _ptr(c2), N, Cin, H, Cout, G, _ptr(y), int(threads))
    _check(st, "mlp_forward")
    return y


def dense_weight(w) -> np.ndarray:
    """Naive replicated matrix M[(o,g),(i,h)] = w[o,i,(g-h) mod G], [Cout*G, Cin*G]."""
    w = _f64(w)
    Cout, Cin, G = w.shape
    M = np.empty((Cout * G, Cin * G), dtype=np.float64)
    _check(_load().eqlin_oracle_dense_weight_f64(_ptr(w), Cout, Cin, G, _ptr(M)), "dense_weight")
    return M


def rdft(v) -> tuple[np.ndarray, np.ndarray]:
    """Unitary real DFT along the last axis: [..., G] -> (re, im) each [..., G//2+1]."""
    v = _f64(v)
    G = v.shape[-1]
    rows = int(np.prod(v.shape[:-1], dtype=np.int64))
    K = G // 2 + 1
    re = np.empty(v.shape[:-1] + (K,), dtype=np.float64)
    im = np.empty_like(re)
    _check(_load().eqlin_oracle_rdft_f64(_ptr(v), rows, G, _ptr(re), _ptr(im)), "rdft")
    return re, im


def irdft(re, im, G: int) -> np.ndarray:
    """Inverse of :func:`rdft` for real signals: (re, im) [..., G//2+1] -> [..., G]."""
    re, im = _f64(re), _f64(im)
    K = G // 2 + 1
    if re.shape[-1] != K or im.shape != re.shape:
        raise ValueError("spectrum shape does not match G")
    rows = int(np.prod(re.shape[:-1], dtype=np.int64))
    v = np.empty(re.shape[:-1] + (G,), dtype=np.float64)
    _check(_load().eqlin_oracle_irdft_f64(_ptr(re), _ptr(im), rows, G, _ptr(v)), "irdft")
    return v


def dense_flops(N: int, Cin: int, Cout: int, G: int) -> int:
    """FLOPs of the naive dense product: 2 * N * (Cout*G) * (Cin*G)
    ("Declaracion del Problema": replicate, then multiply densely)."""
    return 2 * N * (Cout * G) * (Cin * G)


def fourier_real_gemm_blocks(G: int) -> int:
    """Real [Cout x Cin] matrix products per token in the Fourier domain.

    The half spectrum of a real length-G signal (G even) has two real
    frequencies (k = 0 and k = G/2) and G/2 - 1 complex ones; a complex
    product is four real ones.  For p4 (G = 4) this is 2 + 4 = 6, the count
    the p4 section states.  Odd G: one real frequency and (G-1)/2 complex.
    """
    if G % 2 == 0:
        return 2 + 4 * (G // 2 - 1)
    return 1 + 4 * ((G - 1) // 2)


def fourier_flops(N: int, Cin: int, Cout: int, G: int) -> int:
    """FLOPs of the per-frequency contractions: 2 * N * Cin * Cout * blocks(G)."""
    return 2 * N * Cin * Cout * fourier_real_gemm_blocks(G)
