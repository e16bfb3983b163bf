"""ctypes binding of libeqlin.so (C ABI in include/eqlin.h).

Argument marshalling only: every step of the forward and backward runs in the
library's kernels.  torch supplies device memory and streams.  Importing this module
fails loudly if the library has not been built -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libeqlin.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "eqlin.h")

EQLIN_F32 = 0
EQLIN_BF16 = 1
EQLIN_F16 = 2

EQLIN_OK = 0
EQLIN_ERR_INVALID_ARG = -1
EQLIN_ERR_UNSUPPORTED = -2
EQLIN_ERR_MISALIGNED = -3
EQLIN_ERR_CUDA = -4
EQLIN_ERR_OOM = -5
EQLIN_ERR_TIMEOUT = -6

EQLIN_PREPARE_BACKWARD = 1
EQLIN_PREPARE_GELU = 2

ATTRS = {
    "G": 0, "Cin": 1, "Cout": 2, "io_dtype": 3, "path": 4, "tokens_per_tile": 5,
    "stages": 6, "smem_bytes": 7, "max_grid": 8, "weight_bytes": 9, "activation": 10,
    "y_staging": 11, "dw_tile_rows": 12, "dw_tile_cols": 13, "dw_raw_stages": 14, "dw_tokens": 15,
}
PATH_NAMES = {0: "tcgen05_tokens_on_n_resident_weights", 1: "tcgen05_tokens_on_n_streamed_weights",
              2: "fp32_fp64_arithmetic", 3: "tcgen05_tokens_on_m_resident_weights",
              4: "tcgen05_tokens_on_m_streamed_weights", 5: "tcgen05_tokens_on_n_resident_input"}

_TORCH_TO_EQLIN = {torch.float32: EQLIN_F32, torch.bfloat16: EQLIN_BF16, torch.float16: EQLIN_F16}
_EQLIN_TO_TORCH = {v: k for k, v in _TORCH_TO_EQLIN.items()}

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build the CUDA library first "
        "(python -m cyclic_group_dft_b200.build); there is no fallback path")

_lib = ctypes.CDLL(LIB_PATH)
_vp, _i64, _int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
_lib.eqlin_prepare_weights.argtypes = [_vp, _vp, _i64, _i64, _i64, _int, _int, _vp, ctypes.POINTER(_vp)]
_lib.eqlin_forward.argtypes = [_vp, _vp, _vp, _i64, _vp]
_lib.eqlin_forward_host.argtypes = [_vp, _vp, _vp, _i64, _vp]
_lib.eqlin_query_plan.argtypes = [_i64, _i64, _i64, _int, _int, ctypes.POINTER(_i64)]
_lib.eqlin_destroy.argtypes = [_vp]
_lib.eqlin_device_status.argtypes = [_vp, ctypes.POINTER(_int)]
_lib.eqlin_get_attr.argtypes = [_vp, _int, ctypes.POINTER(_i64)]
_lib.eqlin_copy_freq_weights.argtypes = [_vp, ctypes.POINTER(ctypes.c_float), _i64]
_lib.eqlin_check_shape.argtypes = [_i64, _i64, _i64, _int, _int]
_lib.eqlin_forward_noalloc.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _int, _vp]
_lib.eqlin_prepare_weights_ex.argtypes = [_vp, _vp, _i64, _i64, _i64, _int, _int, ctypes.c_uint, _vp,
                                          ctypes.POINTER(_vp)]
_lib.eqlin_backward_dx.argtypes = [_vp, _vp, _vp, _i64, _vp]
_lib.eqlin_backward_dw_workspace_size.argtypes = [_vp, _i64, ctypes.POINTER(ctypes.c_size_t)]
_lib.eqlin_backward_dw.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _vp, ctypes.c_size_t, _vp]
_lib.eqlin_mlp_prepare.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _int, _int, _vp, ctypes.POINTER(_vp)]
_lib.eqlin_mlp_forward.argtypes = [_vp, _vp, _vp, _i64, _vp]
_lib.eqlin_mlp_device_status.argtypes = [_vp, ctypes.POINTER(_int)]
_lib.eqlin_mlp_destroy.argtypes = [_vp]
_lib.eqlin_mlp_query.argtypes = [_i64, _i64, _i64, _i64, _int, ctypes.POINTER(_i64), ctypes.POINTER(_i64)]
_lib.eqlin_status_string.argtypes = [_int]
_lib.eqlin_status_string.restype = ctypes.c_char_p
_lib.eqlin_last_error.argtypes = []
_lib.eqlin_last_error.restype = ctypes.c_char_p
_lib.eqlin_version.argtypes = []
for _f in ("eqlin_prepare_weights", "eqlin_forward", "eqlin_forward_host", "eqlin_query_plan", "eqlin_destroy",
           "eqlin_device_status",
           "eqlin_get_attr", "eqlin_copy_freq_weights", "eqlin_check_shape", "eqlin_version",
           "eqlin_forward_noalloc", "eqlin_prepare_weights_ex", "eqlin_backward_dx",
           "eqlin_backward_dw_workspace_size", "eqlin_backward_dw", "eqlin_mlp_prepare", "eqlin_mlp_forward",
           "eqlin_mlp_device_status", "eqlin_mlp_destroy", "eqlin_mlp_query"):
    getattr(_lib, _f).restype = _int


class EqlinError(RuntimeError):
    """A C-ABI call returned a negative eqlin_status."""

    def __init__(self, status: int, what: str):
        self.status = status
        msg = _lib.eqlin_last_error().decode(errors="replace")
        super().__init__(f"{what}: {eqlin_status_string(status)} ({status}): {msg}")


def _check(status: int, what: str) -> None:
    if status != EQLIN_OK:
        raise EqlinError(status, what)


def library() -> ctypes.CDLL:
    """The loaded libeqlin.so."""
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/eqlin.h declares."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return re.findall(r"^EQLIN_API\s+[\w\s\*]+?\b(eqlin_\w+)\s*\(", text, flags=re.M)


def eqlin_status_string(status: int) -> str:
    return _lib.eqlin_status_string(int(status)).decode()


def eqlin_last_error() -> str:
    return _lib.eqlin_last_error().decode(errors="replace")


def eqlin_version() -> int:
    return int(_lib.eqlin_version())


def eqlin_check_shape(Cout: int, Cin: int, G: int, w_dtype=EQLIN_BF16, io_dtype=EQLIN_BF16) -> int:
    """Host-only shape check; returns the status prepare's validation would give."""
    return int(_lib.eqlin_check_shape(Cout, Cin, G, _as_code(w_dtype), _as_code(io_dtype)))


def _as_code(dt) -> int:
    if isinstance(dt, torch.dtype):
        return _TORCH_TO_EQLIN[dt]
    return int(dt)


def _stream_ptr(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


class Handle:
    """Frequency-domain weights prepared on one device (owns device memory)."""

    def __init__(self, ptr: int, device: torch.device):
        self._ptr = ptr
        self.device = device
        self.G = self.attr("G")
        self.Cin = self.attr("Cin")
        self.Cout = self.attr("Cout")
        self.io_dtype = _EQLIN_TO_TORCH[self.attr("io_dtype")]

    @property
    def ptr(self) -> int:
        if not self._ptr:
            raise EqlinError(EQLIN_ERR_INVALID_ARG, "handle already destroyed")
        return self._ptr

    def attr(self, name: str) -> int:
        v = ctypes.c_int64()
        _check(_lib.eqlin_get_attr(self.ptr, ATTRS[name], ctypes.byref(v)), f"eqlin_get_attr({name})")
        return int(v.value)

    @property
    def path(self) -> str:
        return PATH_NAMES[self.attr("path")]

    def forward(self, x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        return eqlin_forward(self, x, out, stream)

    def backward_dx(self, dy: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """dx = dL/dx from dy (the handle must be prepared with backward=True)."""
        return eqlin_backward_dx(self, dy, out, stream)

    def backward_dw(self, x: torch.Tensor, dy: torch.Tensor, with_bias: bool = True,
                    stream=None) -> tuple[torch.Tensor, torch.Tensor | None]:
        """(dw [Cout, Cin, G], dbias [Cout] or None) = dL/dw, dL/dbias, both fp32."""
        return eqlin_backward_dw(self, x, dy, with_bias, stream)

    def forward_host(self, x_host: torch.Tensor, out_host: torch.Tensor | None = None,
                     stream=None) -> torch.Tensor:
        """Forward from and to host memory through eqlin_forward_host (chunked copies in
        and out overlapping the kernels); returns once y is in host memory."""
        return eqlin_forward_host(self, x_host, out_host, stream)

    def device_status(self) -> int:
        return eqlin_device_status(self)

    def freq_weights(self) -> torch.Tensor:
        return eqlin_copy_freq_weights(self)

    def close(self) -> None:
        if self._ptr:
            p, self._ptr = self._ptr, None
            _check(_lib.eqlin_destroy(p), "eqlin_destroy")

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            if self._ptr and _lib is not None:
                _lib.eqlin_destroy(self._ptr)
                self._ptr = None
        except Exception:
            pass


def eqlin_prepare_weights(w: torch.Tensor, bias: torch.Tensor | None = None,
                          io_dtype: torch.dtype | None = None, stream=None, backward: bool = False,
                          activation: str | None = None) -> Handle:
    """Transform w [Cout, Cin, G] (and bias [Cout]) to the frequency domain on w's device.
    backward=True also prepares the input-gradient weights (eqlin_prepare_weights_ex with
    EQLIN_PREPARE_BACKWARD), for Handle.backward_dx.  activation="gelu" makes the forward
    apply GELU after the bias (EQLIN_PREPARE_GELU)."""
    if activation not in (None, "gelu"):
        raise ValueError(f"unsupported activation {activation!r}")
    if w.dim() != 3:
        raise ValueError("w must be [Cout, Cin, G]")
    if w.device.type != "cuda":
        raise ValueError("w must be a CUDA tensor")
    if w.dtype not in _TORCH_TO_EQLIN:
        raise ValueError(f"unsupported weight dtype {w.dtype}")
    w = w.contiguous()
    Cout, Cin, G = w.shape
    if bias is not None:
        if bias.shape != (Cout,) or bias.device != w.device:
            raise ValueError("bias must be [Cout] on w's device")
        bias = bias.to(w.dtype).contiguous()
    io = _TORCH_TO_EQLIN[w.dtype if io_dtype is None else io_dtype]
    out = ctypes.c_void_p()
    with torch.cuda.device(w.device):
        st = _lib.eqlin_prepare_weights_ex(
            w.data_ptr(), None if bias is None else bias.data_ptr(), Cout, Cin, G,
            _TORCH_TO_EQLIN[w.dtype], io,
            (EQLIN_PREPARE_BACKWARD if backward else 0) | (EQLIN_PREPARE_GELU if activation == "gelu" else 0),
            _stream_ptr(stream), ctypes.byref(out))
    _check(st, "eqlin_prepare_weights_ex")
    return Handle(out.value, w.device)


def eqlin_forward(h: Handle, x: torch.Tensor, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y [N, Cout, G] = EQ-Linear(x [N, Cin, G]) on the handle's device."""
    if x.dim() != 3 or x.shape[1] != h.Cin or x.shape[2] != h.G:
        raise ValueError(f"x must be [N, {h.Cin}, {h.G}], got {tuple(x.shape)}")
    if x.device != h.device or x.dtype != h.io_dtype:
        raise ValueError(f"x must be {h.io_dtype} on {h.device}")
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")
    N = x.shape[0]
    if y is None:
        y = torch.empty((N, h.Cout, h.G), dtype=h.io_dtype, device=h.device)
    elif y.shape != (N, h.Cout, h.G) or y.dtype != h.io_dtype or y.device != h.device \
            or not y.is_contiguous():
        raise ValueError("y has the wrong shape, dtype, device or layout")
    with torch.cuda.device(h.device):
        _check(_lib.eqlin_forward(h.ptr, x.data_ptr(), y.data_ptr(), N, _stream_ptr(stream)),
               "eqlin_forward")
    return y


def query_plan(Cout: int, Cin: int, G: int, io_dtype=torch.bfloat16) -> dict:
    """The kernel plan eqlin_prepare_weights would choose for these sizes on a B200 (host
    only, no GPU): {attribute name: value} via eqlin_query_plan."""
    io = _TORCH_TO_EQLIN[io_dtype]
    out = {}
    v = _i64()
    for name, a in ATTRS.items():
        if name == "activation":
            continue
        _check(_lib.eqlin_query_plan(Cout, Cin, G, io, a, ctypes.byref(v)), "eqlin_query_plan")
        out[name] = v.value
    out["path_name"] = PATH_NAMES.get(out["path"], str(out["path"]))
    return out


def eqlin_forward_host(h: Handle, x_host: torch.Tensor, y_host: torch.Tensor | None = None,
                       stream=None) -> torch.Tensor:
    """y_host [N, Cout, G] = EQ-Linear(x_host [N, Cin, G]), both in host memory (pinned
    for overlapped copies).  Synchronises the stream before returning."""
    if x_host.device.type != "cpu":
        raise ValueError("eqlin_forward_host takes CPU tensors")
    if x_host.dim() != 3 or x_host.shape[1] != h.Cin or x_host.shape[2] != h.G:
        raise ValueError(f"x must be [N, {h.Cin}, {h.G}], got {tuple(x_host.shape)}")
    if x_host.dtype != h.io_dtype or not x_host.is_contiguous():
        raise ValueError(f"x must be contiguous {h.io_dtype}")
    N = x_host.shape[0]
    if y_host is None:
        y_host = torch.empty((N, h.Cout, h.G), dtype=h.io_dtype, pin_memory=x_host.is_pinned())
    elif y_host.shape != (N, h.Cout, h.G) or y_host.dtype != h.io_dtype or y_host.device.type != "cpu" \
            or not y_host.is_contiguous():
        raise ValueError("y has the wrong shape, dtype, device or layout")
    with torch.cuda.device(h.device):
        ptr = _stream_ptr(stream)
        _check(_lib.eqlin_forward_host(h.ptr, x_host.data_ptr(), y_host.data_ptr(), N, ptr),
               "eqlin_forward_host")
        _synchronize(stream, ptr)
    return y_host


def _synchronize(stream, ptr: int) -> None:
    """Block until the work queued on the call's stream is done.  A torch Stream (or None,
    the current stream) synchronises itself; a raw pointer goes through ExternalStream,
    except 0, the legacy default stream, which ExternalStream(0) does not wait for (measured
    on B200: the call returned before its copies out in 99 of 100 trials)."""
    if isinstance(stream, torch.cuda.Stream):
        stream.synchronize()
    elif stream is None:
        torch.cuda.current_stream().synchronize()
    elif ptr == 0:
        torch.cuda.default_stream().synchronize()
    else:
        torch.cuda.ExternalStream(ptr).synchronize()


def _check_rows(t: torch.Tensor, name: str, C: int, h: Handle) -> None:
    if t.dim() != 3 or t.shape[1] != C or t.shape[2] != h.G:
        raise ValueError(f"{name} must be [N, {C}, {h.G}], got {tuple(t.shape)}")
    if t.device != h.device or t.dtype != h.io_dtype:
        raise ValueError(f"{name} must be {h.io_dtype} on {h.device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def eqlin_backward_dx(h: Handle, dy: torch.Tensor, dx: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """dx [N, Cin, G] = dL/dx for the upstream gradient dy [N, Cout, G]."""
    _check_rows(dy, "dy", h.Cout, h)
    N = dy.shape[0]
    if dx is None:
        dx = torch.empty((N, h.Cin, h.G), dtype=h.io_dtype, device=h.device)
    elif dx.shape != (N, h.Cin, h.G) or dx.dtype != h.io_dtype or dx.device != h.device \
            or not dx.is_contiguous():
        raise ValueError("dx has the wrong shape, dtype, device or layout")
    with torch.cuda.device(h.device):
        _check(_lib.eqlin_backward_dx(h.ptr, dy.data_ptr(), dx.data_ptr(), N, _stream_ptr(stream)),
               "eqlin_backward_dx")
    return dx


def eqlin_backward_dw_workspace_size(h: Handle, N: int) -> int:
    v = ctypes.c_size_t()
    _check(_lib.eqlin_backward_dw_workspace_size(h.ptr, N, ctypes.byref(v)), "eqlin_backward_dw_workspace_size")
    return int(v.value)


def eqlin_backward_dw(h: Handle, x: torch.Tensor, dy: torch.Tensor, with_bias: bool = True,
                      stream=None, dw: torch.Tensor | None = None, dbias: torch.Tensor | None = None,
                      workspace: torch.Tensor | None = None) -> tuple[torch.Tensor, torch.Tensor | None]:
    """(dw [Cout, Cin, G] fp32, dbias [Cout] fp32 or None) for the forward input x and
    the upstream gradient dy.  The workspace (a uint8 CUDA tensor) is allocated by torch
    when not given."""
    _check_rows(x, "x", h.Cin, h)
    _check_rows(dy, "dy", h.Cout, h)
    N = x.shape[0]
    if dy.shape[0] != N:
        raise ValueError("x and dy must have the same number of tokens")
    if dw is None:
        dw = torch.empty((h.Cout, h.Cin, h.G), dtype=torch.float32, device=h.device)
    elif dw.shape != (h.Cout, h.Cin, h.G) or dw.dtype != torch.float32 or not dw.is_contiguous():
        raise ValueError("dw must be a contiguous fp32 [Cout, Cin, G] tensor")
    if with_bias and dbias is None:
        dbias = torch.empty((h.Cout,), dtype=torch.float32, device=h.device)
    need = eqlin_backward_dw_workspace_size(h, N)
    if workspace is None:
        workspace = torch.empty((max(need, 16),), dtype=torch.uint8, device=h.device)
    with torch.cuda.device(h.device):
        _check(_lib.eqlin_backward_dw(h.ptr, x.data_ptr(), dy.data_ptr(), dw.data_ptr(),
                                      None if dbias is None else dbias.data_ptr(), N,
                                      workspace.data_ptr(), workspace.numel(), _stream_ptr(stream)),
               "eqlin_backward_dw")
    return dw, dbias


def mlp_block(h1: Handle, h2: Handle, x: torch.Tensor, hidden: torch.Tensor | None = None,
              out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """The equivariant MLP block y = L2(GELU(L1(x))): a forward of h1 (prepared with
    activation="gelu") into `hidden` [N, H, G], then a forward of h2.  Two launches on one
    stream; the second one's prologue overlaps the first one's tail."""
    if h1.attr("activation") != 1:
        raise ValueError("h1 must be prepared with activation='gelu'")
    if h1.Cout != h2.Cin or h1.G != h2.G or h1.io_dtype != h2.io_dtype or h1.device != h2.device:
        raise ValueError("h1's outputs must match h2's inputs (channels, G, dtype, device)")
    hidden = eqlin_forward(h1, x, hidden, stream)
    return eqlin_forward(h2, hidden, out, stream)


class MlpHandle:
    """Both weight sets of an equivariant MLP block y = L2(GELU(L1(x))), transformed for
    the single fused kernel (eqlin_mlp_prepare; owns device memory)."""

    def __init__(self, ptr: int, device: torch.device, Cin: int, H: int, Cout: int, G: int, io_dtype: torch.dtype):
        self._ptr = ptr
        self.device = device
        self.Cin, self.H, self.Cout, self.G, self.io_dtype = Cin, H, Cout, G, io_dtype

    @property
    def ptr(self) -> int:
        if not self._ptr:
            raise EqlinError(EQLIN_ERR_INVALID_ARG, "MLP handle already destroyed")
        return self._ptr

    def forward(self, x: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        return eqlin_mlp_forward(self, x, out, stream)

    def device_status(self) -> int:
        v = ctypes.c_int()
        with torch.cuda.device(self.device):
            _check(_lib.eqlin_mlp_device_status(self.ptr, ctypes.byref(v)), "eqlin_mlp_device_status")
        return int(v.value)

    def close(self) -> None:
        if self._ptr:
            p, self._ptr = self._ptr, None
            _check(_lib.eqlin_mlp_destroy(p), "eqlin_mlp_destroy")

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        self.close()

    def __del__(self):
        try:
            if self._ptr and _lib is not None:
                _lib.eqlin_mlp_destroy(self._ptr)
                self._ptr = None
        except Exception:
            pass


def eqlin_mlp_query(Cin: int, H: int, Cout: int, G: int, io_dtype=torch.bfloat16) -> dict | None:
    """Host only: {"stages", "smem_bytes"} of the fused MLP block's kernel for these sizes on
    a B200, or None when the fused block does not support them."""
    st, sm = _i64(), _i64()
    s = _lib.eqlin_mlp_query(Cin, H, Cout, G, _as_code(io_dtype), ctypes.byref(st), ctypes.byref(sm))
    if s != EQLIN_OK:
        return None
    return {"stages": int(st.value), "smem_bytes": int(sm.value)}


def eqlin_mlp_prepare(w1: torch.Tensor, b1: torch.Tensor | None, w2: torch.Tensor, b2: torch.Tensor | None,
                      io_dtype: torch.dtype | None = None, stream=None) -> MlpHandle:
    """Transform the weights of y = L2(GELU(L1(x))) for the fused kernel: w1 [H, Cin, G],
    b1 [H] or None, w2 [Cout, H, G], b2 [Cout] or None, all CUDA tensors of one dtype."""
    if w1.dim() != 3 or w2.dim() != 3 or w2.shape[1] != w1.shape[0] or w2.shape[2] != w1.shape[2]:
        raise ValueError("w1 must be [H, Cin, G] and w2 [Cout, H, G]")
    if w1.device.type != "cuda" or w2.device != w1.device:
        raise ValueError("w1 and w2 must be CUDA tensors on one device")
    if w1.dtype not in _TORCH_TO_EQLIN or w2.dtype != w1.dtype:
        raise ValueError("w1 and w2 must share a supported dtype")
    H, Cin, G = w1.shape
    Cout = w2.shape[0]
    w1, w2 = w1.contiguous(), w2.contiguous()
    bs = []
    for b, n in ((b1, H), (b2, Cout)):
        if b is not None:
            if b.shape != (n,) or b.device != w1.device:
                raise ValueError("biases must be [H] and [Cout] on the weights' device")
            b = b.to(w1.dtype).contiguous()
        bs.append(b)
    io = w1.dtype if io_dtype is None else io_dtype
    out = ctypes.c_void_p()
    with torch.cuda.device(w1.device):
        st = _lib.eqlin_mlp_prepare(w1.data_ptr(), None if bs[0] is None else bs[0].data_ptr(), w2.data_ptr(),
                                    None if bs[1] is None else bs[1].data_ptr(), Cin, H, Cout, G,
                                    _TORCH_TO_EQLIN[w1.dtype], _TORCH_TO_EQLIN[io], _stream_ptr(stream),
                                    ctypes.byref(out))
    _check(st, "eqlin_mlp_prepare")
    return MlpHandle(out.value, w1.device, Cin, H, Cout, G, io)


def eqlin_mlp_forward(m: MlpHandle, x: torch.Tensor, y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y [N, Cout, G] = L2(GELU(L1(x [N, Cin, G]))) in one fused launch."""
    if x.dim() != 3 or x.shape[1] != m.Cin or x.shape[2] != m.G:
        raise ValueError(f"x must be [N, {m.Cin}, {m.G}], got {tuple(x.shape)}")
    if x.device != m.device or x.dtype != m.io_dtype or not x.is_contiguous():
        raise ValueError(f"x must be a contiguous {m.io_dtype} tensor on {m.device}")
    N = x.shape[0]
    if y is None:
        y = torch.empty((N, m.Cout, m.G), dtype=m.io_dtype, device=m.device)
    elif y.shape != (N, m.Cout, m.G) or y.dtype != m.io_dtype or y.device != m.device or not y.is_contiguous():
        raise ValueError("y has the wrong shape, dtype, device or layout")
    with torch.cuda.device(m.device):
        _check(_lib.eqlin_mlp_forward(m.ptr, x.data_ptr(), y.data_ptr(), N, _stream_ptr(stream)),
               "eqlin_mlp_forward")
    return y


def eqlin_destroy(h: Handle) -> None:
    h.close()


def eqlin_device_status(h: Handle) -> int:
    v = ctypes.c_int()
    with torch.cuda.device(h.device):
        _check(_lib.eqlin_device_status(h.ptr, ctypes.byref(v)), "eqlin_device_status")
    return int(v.value)


def eqlin_copy_freq_weights(h: Handle) -> torch.Tensor:
    """fp32 frequency-domain weights [G, Cin, Cout] (scaled; see include/eqlin.h)."""
    out = torch.empty((h.G, h.Cin, h.Cout), dtype=torch.float32)
    with torch.cuda.device(h.device):
        dst = ctypes.cast(out.data_ptr(), ctypes.POINTER(ctypes.c_float))
        _check(_lib.eqlin_copy_freq_weights(h.ptr, dst, out.numel()), "eqlin_copy_freq_weights")
    return out


def eqlin_forward_noalloc(x: torch.Tensor, w: torch.Tensor, bias: torch.Tensor | None = None,
                          y: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Weight transform + forward in one call that allocates no device memory in the
    library (for callers that must not allocate); x, w, bias and y share one dtype.
    Calls that overlap on the GPU share the library's fixed scratch array: serialise
    them.  (The y tensor, when not given, is allocated here by torch.)"""
    if w.dim() != 3 or x.dim() != 3 or x.shape[1:] != w.shape[1:]:
        raise ValueError("x must be [N, Cin, G] and w [Cout, Cin, G]")
    if x.dtype not in _TORCH_TO_EQLIN or w.dtype != x.dtype or x.device != w.device:
        raise ValueError("x and w must share a supported dtype and a device")
    if not (x.is_contiguous() and w.is_contiguous()):
        raise ValueError("x and w must be contiguous")
    N, Cin, G = x.shape
    Cout = w.shape[0]
    if bias is not None and (bias.shape != (Cout,) or bias.dtype != x.dtype or not bias.is_contiguous()):
        raise ValueError("bias must be a contiguous [Cout] tensor of x's dtype")
    if y is None:
        y = torch.empty((N, Cout, G), dtype=x.dtype, device=x.device)
    elif y.shape != (N, Cout, G) or y.dtype != x.dtype or y.device != x.device or not y.is_contiguous():
        raise ValueError(f"y must be a contiguous [{N}, {Cout}, {G}] tensor of x's dtype on x's device")
    if bias is not None and bias.device != x.device:
        raise ValueError("bias must be on x's device")
    with torch.cuda.device(x.device):
        _check(_lib.eqlin_forward_noalloc(x.data_ptr(), w.data_ptr(), None if bias is None else bias.data_ptr(),
                                          y.data_ptr(), N, Cout, Cin, G, _TORCH_TO_EQLIN[x.dtype],
                                          _stream_ptr(stream)), "eqlin_forward_noalloc")
    return y
