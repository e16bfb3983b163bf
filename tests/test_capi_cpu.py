"""C-ABI checks that need no GPU: the library loads, exports every function
include/eqlin.h declares, and rejects bad arguments on the host before any
CUDA work (so these return codes are the same with or without a device)."""
from __future__ import annotations

import ctypes
import subprocess

import pytest
import torch

import cyclic_group_dft_b200 as eq
from cyclic_group_dft_b200 import _capi


def test_exports_every_declared_function():
    declared = eq.header_functions()
    assert len(declared) >= 10
    lib = eq.library()
    for name in declared:
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", eq.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert exported == set(declared), exported ^ set(declared)


def test_version_and_status_strings():
    assert eq.eqlin_version() >= 100
    assert eq.eqlin_status_string(0) == "ok"
    for code in range(-6, 0):
        assert eq.eqlin_status_string(code) not in ("", "unknown status")
    assert eq.eqlin_status_string(-99) == "unknown status"


@pytest.mark.parametrize("shape,expected", [
    ((96, 96, 4, eq.EQLIN_BF16, eq.EQLIN_BF16), eq.EQLIN_OK),
    ((768, 192, 4, eq.EQLIN_BF16, eq.EQLIN_BF16), eq.EQLIN_OK),
    ((64, 64, 8, eq.EQLIN_BF16, eq.EQLIN_BF16), eq.EQLIN_OK),
    ((32, 32, 16, eq.EQLIN_BF16, eq.EQLIN_BF16), eq.EQLIN_OK),
    ((16, 16, 4, eq.EQLIN_F32, eq.EQLIN_F32), eq.EQLIN_OK),
    ((16, 16, 2, eq.EQLIN_F32, eq.EQLIN_BF16), eq.EQLIN_OK),
    ((96, 96, 4, eq.EQLIN_F16, eq.EQLIN_F16), eq.EQLIN_OK),
    ((32, 32, 16, eq.EQLIN_F32, eq.EQLIN_F16), eq.EQLIN_OK),
    ((3, 3, 2, eq.EQLIN_F16, eq.EQLIN_F16), eq.EQLIN_ERR_UNSUPPORTED),     # Cin*G % 8
    ((96, 96, 3, eq.EQLIN_BF16, eq.EQLIN_BF16), eq.EQLIN_ERR_UNSUPPORTED),
    ((96, 96, 32, eq.EQLIN_BF16, eq.EQLIN_BF16), eq.EQLIN_ERR_UNSUPPORTED),
    ((3, 3, 2, eq.EQLIN_BF16, eq.EQLIN_BF16), eq.EQLIN_ERR_UNSUPPORTED),   # Cin*G % 8
    ((3, 3, 2, eq.EQLIN_F32, eq.EQLIN_F32), eq.EQLIN_OK),                  # fine for fp32
    ((3, 8, 2, eq.EQLIN_BF16, eq.EQLIN_BF16), eq.EQLIN_ERR_UNSUPPORTED),   # Cout*G % 8
    ((0, 4, 4, eq.EQLIN_BF16, eq.EQLIN_BF16), eq.EQLIN_ERR_INVALID_ARG),
    ((4, -1, 4, eq.EQLIN_BF16, eq.EQLIN_BF16), eq.EQLIN_ERR_INVALID_ARG),
    ((4, 4, 4, 7, eq.EQLIN_BF16), eq.EQLIN_ERR_INVALID_ARG),
    ((4, 4, 4, eq.EQLIN_BF16, 9), eq.EQLIN_ERR_INVALID_ARG),
    ((1 << 17, 8, 4, eq.EQLIN_BF16, eq.EQLIN_BF16), eq.EQLIN_ERR_UNSUPPORTED),
])
def test_check_shape(shape, expected):
    assert eq.eqlin_check_shape(*shape) == expected


def _prepare_raw(w_ptr, Cout=8, Cin=8, G=4, wd=eq.EQLIN_BF16, io=eq.EQLIN_BF16, out=True):
    h = ctypes.c_void_p(1234)
    st = eq.library().eqlin_prepare_weights(w_ptr, None, Cout, Cin, G, wd, io, None,
                                            ctypes.byref(h) if out else None)
    return st, h.value


def test_prepare_rejects_bad_arguments_on_host():
    lib = eq.library()
    assert _prepare_raw(None)[0] == eq.EQLIN_ERR_INVALID_ARG
    st, h = _prepare_raw(None)
    assert h is None  # *out cleared on failure
    assert _prepare_raw(16, out=False)[0] == eq.EQLIN_ERR_INVALID_ARG
    assert _prepare_raw(16, G=5)[0] == eq.EQLIN_ERR_UNSUPPORTED
    assert _prepare_raw(16, Cout=0)[0] == eq.EQLIN_ERR_INVALID_ARG
    assert _prepare_raw(17)[0] == eq.EQLIN_ERR_MISALIGNED        # bf16 w at an odd address
    assert _prepare_raw(18, wd=eq.EQLIN_F32, io=eq.EQLIN_F32)[0] == eq.EQLIN_ERR_MISALIGNED
    assert "aligned" in eq.eqlin_last_error()
    assert lib.eqlin_destroy(None) == eq.EQLIN_OK


def test_forward_rejects_bad_arguments_on_host():
    lib = eq.library()
    assert lib.eqlin_forward(None, 16, 16, 4, None) == eq.EQLIN_ERR_INVALID_ARG
    assert "NULL" in eq.eqlin_last_error()
    v = ctypes.c_int64()
    assert lib.eqlin_get_attr(None, 0, ctypes.byref(v)) == eq.EQLIN_ERR_INVALID_ARG
    s = ctypes.c_int()
    assert lib.eqlin_device_status(None, ctypes.byref(s)) == eq.EQLIN_ERR_INVALID_ARG
    assert lib.eqlin_copy_freq_weights(None, None, 0) == eq.EQLIN_ERR_INVALID_ARG
    assert lib.eqlin_forward_host(None, 16, 16, 4, None) == eq.EQLIN_ERR_INVALID_ARG
    assert "NULL" in eq.eqlin_last_error()


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks behaviour without a GPU")
def test_prepare_without_gpu_reports_cuda_error():
    # an aligned fake pointer passes host validation; the device query then fails
    st, h = _prepare_raw(256)
    assert st == eq.EQLIN_ERR_CUDA
    assert h is None


def test_binding_validates_before_calling():
    with pytest.raises(ValueError):
        eq.eqlin_prepare_weights(torch.zeros(4, 4))          # not 3-D
    with pytest.raises(ValueError):
        eq.eqlin_prepare_weights(torch.zeros(4, 4, 4))       # not on a GPU


def test_header_matches_binding_constants():
    text = open(_capi.HEADER_PATH).read()
    for name in ("EQLIN_ERR_INVALID_ARG = -1", "EQLIN_ERR_UNSUPPORTED = -2", "EQLIN_ERR_MISALIGNED = -3",
                 "EQLIN_ERR_CUDA = -4", "EQLIN_ERR_OOM = -5", "EQLIN_ERR_TIMEOUT = -6",
                 "EQLIN_F32 = 0", "EQLIN_BF16 = 1", "EQLIN_F16 = 2"):
        assert name in text
    for attr, code in eq.ATTRS.items():
        assert f"= {code}" in text


def test_backward_entry_points_reject_bad_arguments_on_host():
    lib = eq.library()
    assert lib.eqlin_backward_dx(None, 16, 16, 4, None) == eq.EQLIN_ERR_INVALID_ARG
    n = ctypes.c_size_t()
    assert lib.eqlin_backward_dw_workspace_size(None, 4, ctypes.byref(n)) == eq.EQLIN_ERR_INVALID_ARG
    assert lib.eqlin_backward_dw(None, 16, 16, 16, None, 4, 16, 1 << 20, None) == eq.EQLIN_ERR_INVALID_ARG
    h = ctypes.c_void_p(1234)
    # unknown flag bits are rejected before anything else is looked at
    st = lib.eqlin_prepare_weights_ex(16, None, 8, 8, 4, eq.EQLIN_BF16, eq.EQLIN_BF16, 0x80, None,
                                      ctypes.byref(h))
    assert st == eq.EQLIN_ERR_INVALID_ARG and h.value is None
    assert "flag" in eq.eqlin_last_error()
    st = lib.eqlin_prepare_weights_ex(None, None, 8, 8, 4, eq.EQLIN_BF16, eq.EQLIN_BF16,
                                      eq.EQLIN_PREPARE_BACKWARD, None, ctypes.byref(h))
    assert st == eq.EQLIN_ERR_INVALID_ARG


def test_header_declares_the_backward_flag():
    text = open(_capi.HEADER_PATH).read()
    assert f"#define EQLIN_PREPARE_BACKWARD {eq.EQLIN_PREPARE_BACKWARD}u" in text


def test_gelu_flag_is_declared_and_accepted_on_host():
    text = open(_capi.HEADER_PATH).read()
    assert f"#define EQLIN_PREPARE_GELU {eq.EQLIN_PREPARE_GELU}u" in text
    assert "EQLIN_ATTR_ACTIVATION = 10" in text
    lib = eq.library()
    h = ctypes.c_void_p(1234)
    # both flags together pass the flag check (then fail on the NULL weight pointer)
    st = lib.eqlin_prepare_weights_ex(None, None, 8, 8, 4, eq.EQLIN_BF16, eq.EQLIN_BF16,
                                      eq.EQLIN_PREPARE_BACKWARD | eq.EQLIN_PREPARE_GELU, None,
                                      ctypes.byref(h))
    assert st == eq.EQLIN_ERR_INVALID_ARG and "NULL" in eq.eqlin_last_error()


# ---------------------------------------------------------------- planner (host only)
@pytest.mark.parametrize("Cout,Cin,G,path,ystore", [
    (96, 96, 4, "tcgen05_tokens_on_n_resident_weights", "tma"),      # headline: staged TMA stores
    (96, 96, 2, "tcgen05_tokens_on_n_resident_weights", "tma"),
    (384, 96, 4, "tcgen05_tokens_on_n_streamed_weights", "tma"),     # 3 input chunks: no resident input
    (512, 128, 4, "tcgen05_tokens_on_n_resident_input", "tma"),      # from 4 input chunks on
    (768, 192, 4, "tcgen05_tokens_on_n_resident_input", "direct"),   # direct stores deepen the ring
    (96, 384, 4, "tcgen05_tokens_on_n_streamed_weights", "direct"),  # 12 input chunks: direct stores
    (64, 224, 4, "tcgen05_tokens_on_n_resident_weights", "tma"),     # 7 input chunks: staged
    (64, 256, 4, "tcgen05_tokens_on_n_resident_weights", "direct"),  # 8 input chunks: direct
    (64, 64, 8, "tcgen05_tokens_on_m_resident_weights", "none"),
    (32, 32, 16, "tcgen05_tokens_on_m_resident_weights", "none"),
])
def test_planner_kernel_choice(Cout, Cin, G, path, ystore):
    """The kernel form and store mode the planner picks, from the measured rules."""
    q = eq.query_plan(Cout, Cin, G)
    assert q["path_name"] == path
    mode = {-1: "none", 0: "direct"}.get(q["y_staging"], "tma")
    assert mode == ystore, q


def test_planner_fits_shared_memory_and_tiles():
    for shape in [(96, 96, 4), (768, 192, 4), (64, 64, 8), (32, 32, 16), (1024, 1024, 4), (1, 1, 8), (8, 16, 2)]:
        for io in (torch.bfloat16, torch.float16):
            q = eq.query_plan(*shape, io_dtype=io)
            assert 0 < q["smem_bytes"] <= 232448
            assert q["stages"] >= 2 and q["tokens_per_tile"] in (16, 32, 64, 128)
            assert q["max_grid"] == 148


@pytest.mark.parametrize("G,tokens", [(2, 32), (4, 32), (8, 16), (16, 16)])
def test_planner_weight_gradient_chunks(G, tokens):
    """Weight-gradient chunks: 32 tokens up to G = 4, 16 from G = 8 on (a deeper raw ring)."""
    q = eq.query_plan(32, 32, G)
    assert q["dw_tokens"] == tokens
    assert q["dw_raw_stages"] >= 2
    assert q["dw_tile_rows"] % 16 == 0 and q["dw_tile_cols"] % 16 == 0


@pytest.mark.parametrize("Cout,Cin,G,rows,cols", [(96, 96, 4, 96, 96), (768, 192, 4, 128, 96),
                                                    (192, 768, 4, 96, 128), (64, 64, 8, 64, 64),
                                                    (32, 32, 16, 32, 32)])
def test_planner_weight_gradient_tiles(Cout, Cin, G, rows, cols):
    """Weight-gradient tiles: the fewest units, then the least padded area (192 input
    channels as 2 x 96, not 128 + 64)."""
    q = eq.query_plan(Cout, Cin, G)
    assert (q["dw_tile_rows"], q["dw_tile_cols"]) == (rows, cols)


def test_planner_tokens_on_m_weight_image():
    """Tokens-on-M weight image: the G planes in plane order up to G = 8 (p8 C64: 64 KB, so
    four 32 KB ring stages fit), the pair slots at G = 16 (C16 C32: 23 slots, 46 KB)."""
    q = eq.query_plan(64, 64, 8)
    assert "tokens_on_m" in q["path_name"] and q["weight_bytes"] == 8 * 64 * 32 * 4 and q["stages"] == 4
    q = eq.query_plan(32, 32, 16)
    assert "tokens_on_m" in q["path_name"] and q["weight_bytes"] == 23 * 32 * 32 * 2


def test_planner_y_staging_only_for_used_lane_quarters():
    """Tokens-on-N with one output chunk: Cout = 96 uses 3 of the 4 TMEM lane quarters, so
    only 3 x 2 warps get y staging and the input ring gets a fifth stage."""
    q = eq.query_plan(96, 96, 4)
    assert q["path_name"] == "tcgen05_tokens_on_n_resident_weights"
    assert q["stages"] == 5 and q["y_staging"] == 2


def test_planner_environment_overrides(monkeypatch):
    monkeypatch.setenv("EQLIN_KERNEL", "tm")
    assert "tokens_on_m" in eq.query_plan(96, 96, 4)["path_name"]
    monkeypatch.setenv("EQLIN_KERNEL", "tn")
    assert eq.query_plan(768, 192, 4)["path_name"] == "tcgen05_tokens_on_n_streamed_weights"
    monkeypatch.delenv("EQLIN_KERNEL")
    monkeypatch.setenv("EQLIN_YSTORE", "direct")
    assert eq.query_plan(96, 96, 4)["y_staging"] == 0
    monkeypatch.setenv("EQLIN_YSTORE", "tma")
    assert eq.query_plan(768, 192, 4)["y_staging"] in (1, 2)


def test_planner_query_errors():
    lib = eq.library()
    v = ctypes.c_int64()
    assert lib.eqlin_query_plan(96, 96, 3, eq.EQLIN_BF16, 4, ctypes.byref(v)) == eq.EQLIN_ERR_UNSUPPORTED
    assert lib.eqlin_query_plan(96, 96, 4, eq.EQLIN_BF16, 999, ctypes.byref(v)) == eq.EQLIN_ERR_INVALID_ARG
    assert lib.eqlin_query_plan(96, 96, 4, eq.EQLIN_BF16, 4, None) == eq.EQLIN_ERR_INVALID_ARG
    q = eq.query_plan(16, 16, 4, io_dtype=torch.float32)
    assert q["path_name"] == "fp32_fp64_arithmetic" and q["dw_tokens"] == -1


def test_planner_over_random_shapes():
    """Every accepted 16-bit shape gets a plan inside the 227 KB opt-in shared memory with at
    least two ring stages, a tile the kernels support, and a weight-gradient tiling."""
    import random
    rnd = random.Random(7)
    lib = eq.library()
    checked = 0
    for _ in range(300):
        G = rnd.choice([2, 4, 8, 16])
        step = max(1, 8 // G)                  # 16-byte rows: C*G a multiple of 8
        Cout = step * rnd.randint(1, 1024 // step)
        Cin = step * rnd.randint(1, 1024 // step)
        io = rnd.choice([torch.bfloat16, torch.float16])
        if lib.eqlin_check_shape(Cout, Cin, G, eq.EQLIN_BF16, eq.EQLIN_BF16) != eq.EQLIN_OK:
            continue
        q = eq.query_plan(Cout, Cin, G, io_dtype=io)
        assert 0 < q["smem_bytes"] <= 232448, (Cout, Cin, G, q)
        assert q["stages"] >= 1 and q["tokens_per_tile"] in (16, 32, 64, 128), (Cout, Cin, G, q)
        assert q["dw_tile_rows"] > 0 and q["dw_tile_cols"] > 0 and q["dw_raw_stages"] >= 2, (Cout, Cin, G, q)
        checked += 1
    assert checked > 250


def test_fused_mlp_block_planner():
    """eqlin_mlp_query (host only): the fused MLP block's supported sizes and its ring."""
    for Cin, H, Cout, G in [(96, 384, 96, 4), (64, 256, 64, 8), (32, 128, 32, 16), (48, 80, 24, 2), (256, 64, 16, 2)]:
        for io in (torch.bfloat16, torch.float16):
            q = eq.eqlin_mlp_query(Cin, H, Cout, G, io)
            assert q is not None and 2 <= q["stages"] <= 12 and q["smem_bytes"] <= 232448, (Cin, H, Cout, G, q)
        assert eq.eqlin_mlp_query(Cin, H, Cout, G, torch.float32) is not None
    # one output chunk only; the input spectrum of a tile must stay in shared memory
    assert eq.eqlin_mlp_query(96, 384, 136, 4) is None
    assert eq.eqlin_mlp_query(288, 64, 64, 4) is None
    assert eq.eqlin_mlp_query(256, 64, 64, 16) is None
    # the single-layer shape rules apply to both layers
    assert eq.eqlin_mlp_query(96, 382, 96, 4) is not None       # H*G = 1528, a multiple of 8
    assert eq.eqlin_mlp_query(96, 381, 96, 2) is None           # H*G = 762 is not
    assert eq.eqlin_mlp_query(96, 384, 96, 3) is None
    # fp32: 8 tokens' spectra of the input and the hidden layer in shared memory
    assert eq.eqlin_mlp_query(96, 384, 96, 4, torch.float32) is not None
    assert eq.eqlin_mlp_query(512, 4096, 96, 4, torch.float32) is None
