"""B200-native (sm_100a) EQ-Linear forward over the cyclic group C_G.

y[n,o,g] = bias[o] + sum_{i,h} w[o,i,(g-h) mod G] x[n,i,h], computed as a real
DFT over the group axis, per-frequency contractions on tcgen05 tensor cores
(half spectrum) and an inverse DFT, fused in one kernel; and its backward
(input, weight and bias gradients) the same way.

Usage::

    import cyclic_group_dft_b200 as eq
    h = eq.prepare(w, bias)          # w [Cout, Cin, G] CUDA tensor (bf16 or fp32)
    y = h.forward(x)                 # x [N, Cin, G] -> y [N, Cout, G]

    hb = eq.prepare(w, bias, backward=True)
    dx = hb.backward_dx(dy)          # dy [N, Cout, G] -> dx [N, Cin, G]
    dw, dbias = hb.backward_dw(x, dy)  # fp32 [Cout, Cin, G], [Cout]

The functions with the C ABI's names (eqlin_prepare_weights, eqlin_forward,
eqlin_destroy, ...) are the same calls with explicit arguments.

The CUDA library (libeqlin.so) is loaded on first use of any of these names, not
at package import: the submodule ``workloads`` (seeded synthetic inputs, no
arithmetic of the layer) can be imported by a process that never runs the layer
on a GPU.  The first use fails with ImportError when the library is missing --
there is no fallback path.
"""
from __future__ import annotations

import importlib

_EXPORTS = (
    "ATTRS",
    "EQLIN_BF16",
    "EQLIN_ERR_CUDA",
    "EQLIN_ERR_INVALID_ARG",
    "EQLIN_ERR_MISALIGNED",
    "EQLIN_ERR_OOM",
    "EQLIN_ERR_TIMEOUT",
    "EQLIN_ERR_UNSUPPORTED",
    "EQLIN_F16",
    "EQLIN_F32",
    "EQLIN_OK",
    "EQLIN_PREPARE_BACKWARD",
    "EQLIN_PREPARE_GELU",
    "LIB_PATH",
    "PATH_NAMES",
    "EqlinError",
    "Handle",
    "eqlin_backward_dw",
    "eqlin_backward_dw_workspace_size",
    "eqlin_backward_dx",
    "eqlin_check_shape",
    "eqlin_copy_freq_weights",
    "eqlin_destroy",
    "eqlin_device_status",
    "eqlin_forward",
    "eqlin_forward_noalloc",
    "eqlin_forward_host",
    "query_plan",
    "eqlin_last_error",
    "eqlin_prepare_weights",
    "eqlin_status_string",
    "eqlin_version",
    "header_functions",
    "library",
    "mlp_block",
    "MlpHandle",
    "eqlin_mlp_prepare",
    "eqlin_mlp_forward",
    "eqlin_mlp_query",
)

__all__ = list(_EXPORTS) + ["prepare", "workloads"]


def __getattr__(name: str):
    if name in _EXPORTS or name == "prepare":
        capi = importlib.import_module("._capi", __name__)
        value = capi.eqlin_prepare_weights if name == "prepare" else getattr(capi, name)
        globals()[name] = value
        return value
    if name == "workloads":
        return importlib.import_module(".workloads", __name__)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")


def __dir__():
    return sorted(set(globals()) | set(__all__))
