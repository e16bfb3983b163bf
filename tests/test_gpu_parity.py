"""GPU parity: the CUDA path (called through the C ABI) against the float64 oracle
on identical seeded inputs.

* every workload at a small N that spans several tiles plus a ragged tail,
  compared element by element, seeds 0-2;
* every workload at its full size, on sampled tokens (tokens are independent,
  so the oracle computes just those rows);
* edge cases: N = 1, N = 0, non-multiple-of-32 channel counts, Cout > 128
  (weights streamed), every supported G, fp32 / bf16 / fp16 weights and I/O,
  no bias;
* properties: cyclic-shift equivariance, guard bands around y untouched,
  the device status word stays OK, the prepared weights equal the oracle's DFT.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import cyclic_group_dft_b200 as eq
import oracle
from cyclic_group_dft_b200 import workloads
from parity_util import BF16_DERIVED, TOL_BF16_NORMWISE, TOL_F32_MAXREL, check

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _prep(w, bias, dtype):
    return eq.prepare(w.to(DEV), None if bias is None else bias.to(DEV), io_dtype=dtype)


def _run(x, w, bias, dtype):
    h = _prep(w, bias, dtype)
    y = h.forward(x.to(DEV))
    torch.cuda.synchronize()
    assert h.device_status() == eq.EQLIN_OK
    return y.cpu(), h


def _ref(x, w, bias):
    return oracle.forward(x, w, bias)


def _assert_parity(dtype, y, ref, label):
    r = check(dtype, y, ref)
    assert r["ok"], f"{label}: {r}"
    return r


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_workload_small_n(name, seed):
    wl = workloads.WORKLOADS[name]
    N = 1031 if name != "tiny_p4_fp32" else wl.N + 37
    x, w, bias = workloads.make_inputs(wl, seed=seed, N=N)
    y, h = _run(x, w, bias, wl.torch_dtype)
    _assert_parity(wl.torch_dtype, y, _ref(x, w, bias), f"{name} seed {seed} N {N}")
    h.close()


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_workload_full_size_sampled(name):
    wl = workloads.WORKLOADS[name]
    x, w, bias = workloads.make_inputs(wl)
    y, h = _run(x, w, bias, wl.torch_dtype)
    idx = workloads.sample_tokens(wl.N, 768, seed=7)
    ref = _ref(x[idx], w, bias)
    _assert_parity(wl.torch_dtype, y[idx], ref, f"{name} full N={wl.N}")
    assert torch.isfinite(y.float()).all()
    h.close()


@pytest.mark.parametrize("N", [1, 2, 127, 128, 129, 255, 257, 1000])
def test_ragged_token_counts(N):
    wl = workloads.WORKLOADS["p4_c96_bf16"]
    x, w, bias = workloads.make_inputs(wl, seed=3, N=N)
    y, h = _run(x, w, bias, wl.torch_dtype)
    _assert_parity(wl.torch_dtype, y, _ref(x, w, bias), f"N={N}")
    h.close()


SHAPES = [  # (Cout, Cin, G): odd channel counts, streamed weights (Cout > 128), every G
    (8, 16, 2), (96, 96, 2), (50, 40, 4), (100, 64, 4), (200, 32, 4), (130, 96, 4),
    (24, 8, 8), (64, 64, 8), (136, 64, 8), (32, 32, 16), (16, 8, 16), (160, 16, 16),
    (128, 128, 4), (256, 96, 4),
]


@pytest.mark.parametrize("io", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("Cout,Cin,G", SHAPES)
def test_shapes_every_group_order(Cout, Cin, G, io):
    gen = torch.Generator().manual_seed(Cout * 1000 + Cin * 10 + G)
    N = 300
    x = torch.randn(N, Cin, G, generator=gen).to(io)
    w = (torch.randn(Cout, Cin, G, generator=gen) / np.sqrt(Cin * G)).to(io)
    bias = (torch.randn(Cout, generator=gen) * 0.3).to(io)
    y, h = _run(x, w, bias, io)
    _assert_parity(io, y, _ref(x, w, bias), f"Cout={Cout} Cin={Cin} G={G} {io} path={h.path}")
    h.close()


@pytest.mark.parametrize("io", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("kernel", ["tn", "tm", "tnr"])
@pytest.mark.parametrize("Cout,Cin,G", SHAPES)
def test_shapes_both_fused_kernels(Cout, Cin, G, kernel, io, monkeypatch):
    """Each fused 16-bit kernel (tokens on N, tokens on M, tokens on N with the input
    spectrum resident -- which falls back to tokens on N where it does not apply) is
    correct for every shape, whichever one the planner would pick by default."""
    monkeypatch.setenv("EQLIN_KERNEL", kernel)
    gen = torch.Generator().manual_seed(Cout * 1000 + Cin * 10 + G + 5)
    N = 517
    x = torch.randn(N, Cin, G, generator=gen).to(io)
    w = (torch.randn(Cout, Cin, G, generator=gen) / np.sqrt(Cin * G)).to(io)
    bias = (torch.randn(Cout, generator=gen) * 0.3).to(io)
    y, h = _run(x, w, bias, io)
    assert f"tokens_on_{kernel[1]}" in h.path, h.path
    _assert_parity(io, y, _ref(x, w, bias), f"Cout={Cout} Cin={Cin} G={G} {kernel} {io}")
    h.close()


@pytest.mark.parametrize("Cout,Cin,G,path", [
    (96, 96, 4, "tcgen05_tokens_on_n_resident_weights"), (384, 96, 4, "tcgen05_tokens_on_n_streamed_weights"),
    (768, 192, 4, "tcgen05_tokens_on_n_resident_input"), (512, 128, 4, "tcgen05_tokens_on_n_resident_input"),
    (96, 384, 4, "tcgen05_tokens_on_n_streamed_weights"), (64, 64, 8, "tcgen05_tokens_on_m_resident_weights"),
])
def test_default_kernel_choice(Cout, Cin, G, path):
    """The planner's default for 16-bit I/O, so the parity cases cover each form."""
    w = torch.zeros(Cout, Cin, G, dtype=torch.bfloat16, device=DEV)
    h = eq.prepare(w, None)
    assert h.path == path
    h.close()


EDGE_SHAPES = [  # (Cout, Cin, G): the fewest channels 16-byte rows allow, and large layers
    (1, 1, 8), (1, 1, 16), (2, 2, 4), (4, 4, 2), (8, 4, 2), (4, 1, 8), (3, 5, 8),
    (1024, 1024, 4), (2048, 64, 8), (64, 2048, 4), (512, 512, 16),
]


@pytest.mark.parametrize("kernel", ["default", "tn", "tm", "tnr"])
@pytest.mark.parametrize("Cout,Cin,G", EDGE_SHAPES)
def test_edge_channel_counts(Cout, Cin, G, kernel, monkeypatch):
    """Smallest channel counts (a 16-byte row), where one 32- or 16-channel chunk is mostly
    padding, and large layers with many weight chunks, on each fused kernel."""
    if kernel != "default":
        monkeypatch.setenv("EQLIN_KERNEL", kernel)
    gen = torch.Generator().manual_seed(Cout * 7 + Cin * 3 + G)
    N = 333 if Cout * Cin < 2 ** 17 else 97   # the oracle's definition loop stays a few seconds
    x = torch.randn(N, Cin, G, generator=gen).to(torch.bfloat16)
    w = (torch.randn(Cout, Cin, G, generator=gen) / np.sqrt(Cin * G)).to(torch.bfloat16)
    bias = (torch.randn(Cout, generator=gen) * 0.3).to(torch.bfloat16)
    y, h = _run(x, w, bias, torch.bfloat16)
    _assert_parity(torch.bfloat16, y, _ref(x, w, bias), f"Cout={Cout} Cin={Cin} G={G} {kernel} path={h.path}")
    h.close()


@pytest.mark.parametrize("ystore", ["tma", "direct"])
@pytest.mark.parametrize("Cout,Cin,G", [(50, 40, 4), (96, 96, 4), (200, 32, 4), (130, 96, 4), (96, 96, 2),
                                        (136, 64, 8), (768, 192, 4), (70, 64, 4), (16, 32, 16)])
def test_tokens_on_n_store_modes(Cout, Cin, G, ystore, monkeypatch):
    """Both ways the tokens-on-N epilogues write y (TMA stores of a staged group, plain
    coalesced stores), for both tokens-on-N kernels, with a ragged token tail.  Cout = 50,
    70, 96 and 16 leave TMEM lane quarters empty, which get no staging."""
    monkeypatch.setenv("EQLIN_KERNEL", "tnr")
    monkeypatch.setenv("EQLIN_YSTORE", ystore)
    gen = torch.Generator().manual_seed(Cout * 1000 + Cin * 10 + G + 17)
    N = 1031
    x = torch.randn(N, Cin, G, generator=gen).to(torch.bfloat16)
    w = (torch.randn(Cout, Cin, G, generator=gen) / np.sqrt(Cin * G)).to(torch.bfloat16)
    bias = (torch.randn(Cout, generator=gen) * 0.3).to(torch.bfloat16)
    y, h = _run(x, w, bias, torch.bfloat16)
    assert "tokens_on_n" in h.path, h.path
    _assert_parity(torch.bfloat16, y, _ref(x, w, bias), f"Cout={Cout} Cin={Cin} G={G} {ystore} path={h.path}")
    h.close()


@pytest.mark.parametrize("kernel", ["tn", "tm", "tnr"])
@pytest.mark.parametrize("name", ["p4_c96_bf16", "p8_c64_bf16", "p4_mlp_bf16", "c16_c32_bf16"])
def test_workloads_both_fused_kernels(name, kernel, monkeypatch):
    monkeypatch.setenv("EQLIN_KERNEL", kernel)
    wl = workloads.WORKLOADS[name]
    x, w, bias = workloads.make_inputs(wl, seed=11, N=2 * 148 * 128 + 77)
    y, h = _run(x, w, bias, wl.torch_dtype)
    idx = workloads.sample_tokens(x.shape[0], 512, seed=13)
    _assert_parity(wl.torch_dtype, y[idx], _ref(x[idx], w, bias), f"{name} {kernel} path={h.path}")
    h.close()


@pytest.mark.parametrize("G", [2, 4, 8, 16])
def test_fp32_weights_bf16_io(G):
    gen = torch.Generator().manual_seed(G)
    Cout, Cin, N = 48, 32, 200
    x = torch.randn(N, Cin, G, generator=gen).to(torch.bfloat16)
    w = torch.randn(Cout, Cin, G, generator=gen) / np.sqrt(Cin * G)
    bias = torch.randn(Cout, generator=gen) * 0.3
    y, h = _run(x, w, bias, torch.bfloat16)
    _assert_parity(torch.bfloat16, y, _ref(x, w, bias), f"fp32 weights G={G}")
    h.close()


def test_no_bias_equals_zero_bias():
    wl = workloads.WORKLOADS["p4_c96_bf16"]
    x, w, bias = workloads.make_inputs(wl, N=300)
    y0, h0 = _run(x, w, None, wl.torch_dtype)
    y1, h1 = _run(x, w, torch.zeros_like(bias), wl.torch_dtype)
    assert torch.equal(y0, y1)
    h0.close()
    h1.close()


@pytest.mark.parametrize("name", ["p4_c96_bf16", "p8_c64_bf16", "c16_c32_bf16", "tiny_p4_fp32"])
def test_cyclic_shift_equivariance(name):
    wl = workloads.WORKLOADS[name]
    x, w, bias = workloads.make_inputs(wl, N=257)
    h = _prep(w, bias, wl.torch_dtype)
    y = h.forward(x.to(DEV)).float().cpu().numpy()
    for s in range(1, wl.G):
        ys = h.forward(torch.roll(x, s, dims=-1).contiguous().to(DEV)).float().cpu().numpy()
        ref = np.roll(y, s, axis=-1)
        err = np.linalg.norm(ys - ref) / np.linalg.norm(ref)
        tol = 1e-6 if wl.io_dtype == "f32" else BF16_DERIVED
        assert err <= tol, (s, err)
    h.close()


def test_prepared_weights_equal_oracle_dft():
    for G in (2, 4, 8, 16):
        for wdt in (torch.float32, torch.bfloat16):
            gen = torch.Generator().manual_seed(100 + G)
            Cout, Cin = 24, 40
            w = torch.randn(Cout, Cin, G, generator=gen).to(wdt)
            h = eq.prepare(w.to(DEV), None, io_dtype=torch.bfloat16 if G * Cin % 8 == 0 else torch.float32)
            got = h.freq_weights().numpy()                  # [G, Cin, Cout]
            re, im = oracle.rdft(w)                          # [Cout, Cin, G/2+1], unitary
            K = G // 2
            s = 1.0 / np.sqrt(G)
            exp = np.empty((G, Cin, Cout))
            exp[0] = (s * re[..., 0]).T
            exp[1] = (s * re[..., K]).T
            for k in range(1, K):
                exp[2 * k] = (2 * s * re[..., k]).T
                exp[2 * k + 1] = (2 * s * im[..., k]).T
            err = np.abs(got - exp).max() / np.abs(exp).max()
            assert err < 1e-6, (G, wdt, err)
            h.close()


def test_empty_batch_is_noop():
    wl = workloads.WORKLOADS["p4_c96_bf16"]
    _, w, bias = workloads.make_inputs(wl, N=1)
    h = _prep(w, bias, wl.torch_dtype)
    x = torch.empty(0, wl.Cin, wl.G, dtype=torch.bfloat16, device=DEV)
    y = h.forward(x)
    assert y.shape == (0, wl.Cout, wl.G)
    assert eq.library().eqlin_forward(h.ptr, None, None, 0, None) == eq.EQLIN_OK
    h.close()


def test_misaligned_and_wrong_arguments_rejected():
    wl = workloads.WORKLOADS["p4_c96_bf16"]
    x, w, bias = workloads.make_inputs(wl, N=64)
    h = _prep(w, bias, wl.torch_dtype)
    buf = torch.zeros(x.numel() + 8, dtype=torch.bfloat16, device=DEV)
    y = torch.empty(64, wl.Cout, wl.G, dtype=torch.bfloat16, device=DEV)
    lib = eq.library()
    st = lib.eqlin_forward(h.ptr, buf.data_ptr() + 2, y.data_ptr(), 64, None)
    assert st == eq.EQLIN_ERR_MISALIGNED
    st = lib.eqlin_forward(h.ptr, buf.data_ptr(), y.data_ptr() + 8, 64, None)
    assert st == eq.EQLIN_ERR_MISALIGNED
    assert lib.eqlin_forward(h.ptr, buf.data_ptr(), y.data_ptr(), -1, None) == eq.EQLIN_ERR_INVALID_ARG
    with pytest.raises(ValueError):
        h.forward(x.to(DEV).float())
    h.close()


def test_output_guard_bands_untouched():
    wl = workloads.WORKLOADS["p8_c64_bf16"]
    N = 1000
    x, w, bias = workloads.make_inputs(wl, N=N)
    h = _prep(w, bias, wl.torch_dtype)
    n_out = N * wl.Cout * wl.G
    pad = 4096
    big = torch.full((pad + n_out + pad,), 12345.0, dtype=torch.bfloat16, device=DEV)
    y = big[pad:pad + n_out].view(N, wl.Cout, wl.G)
    h.forward(x.to(DEV), out=y)
    torch.cuda.synchronize()
    canary = torch.tensor(12345.0, dtype=torch.bfloat16)
    assert (big[:pad].cpu() == canary).all()
    assert (big[pad + n_out:].cpu() == canary).all()
    _assert_parity(torch.bfloat16, y.cpu(), _ref(x, w, bias), "guard band run")
    h.close()


def test_repeated_calls_are_deterministic():
    wl = workloads.WORKLOADS["p4_c96_bf16"]
    x, w, bias = workloads.make_inputs(wl, N=5000)
    h = _prep(w, bias, wl.torch_dtype)
    xd = x.to(DEV)
    ys = [h.forward(xd).cpu() for _ in range(3)]
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[1], ys[2])
    assert h.device_status() == eq.EQLIN_OK
    h.close()


def test_host_buffer_forward_matches_device_forward():
    wl = workloads.WORKLOADS["p4_c96_bf16"]
    x, w, bias = workloads.make_inputs(wl, N=2048)
    h = _prep(w, bias, wl.torch_dtype)
    y_dev = h.forward(x.to(DEV)).cpu()
    y_host = h.forward_host(x.pin_memory())
    assert torch.equal(y_dev, y_host)
    h.close()


@pytest.mark.parametrize("which", ["none", "torch_stream", "raw_default_pointer"])
def test_host_buffer_forward_returns_with_y_in_place(which):
    """The binding's forward_host returns only once y is in host memory, whichever way the
    stream is given (None = the current stream, a torch Stream, or the raw pointer 0 of the
    legacy default stream): a NaN-filled pinned output holds the device forward's values
    right after the call, with no synchronisation by the caller."""
    wl = workloads.WORKLOADS["p4_c96_bf16"]
    x, w, bias = workloads.make_inputs(wl, seed=61, N=2048)
    h = _prep(w, bias, wl.torch_dtype)
    ref = h.forward(x.to(DEV)).cpu()
    xp = x.pin_memory()
    side = torch.cuda.Stream(DEV)
    stream = {"none": None, "torch_stream": side, "raw_default_pointer": 0}[which]
    for _ in range(20):
        yp = torch.full((2048, wl.Cout, wl.G), float("nan"), dtype=wl.torch_dtype).pin_memory()
        torch.cuda.synchronize()
        out = h.forward_host(xp, yp, stream=stream)
        snap = out.clone()                      # before any synchronisation of ours
        assert torch.equal(snap, ref)
    h.close()


def test_host_buffer_forward_on_two_streams():
    """Two host-buffer calls on one handle, issued on two streams without a synchronisation
    between them, each over more chunks than the handle has staging buffers: the second
    call's copies must wait for the first call's use of the shared buffers, so both
    results equal the device-buffer forward."""
    wl = workloads.WORKLOADS["p4_c96_bf16"]
    N = 6 * 10880 + 300                       # 10880 tokens per full chunk at p4 C96: > 4 chunks
    x1, w, bias = workloads.make_inputs(wl, seed=31, N=N)
    x2, _, _ = workloads.make_inputs(wl, seed=32, N=N)
    h = _prep(w, bias, wl.torch_dtype)
    ref1, ref2 = h.forward(x1.to(DEV)).cpu(), h.forward(x2.to(DEV)).cpu()
    xs = [x1.pin_memory(), x2.pin_memory()]
    ys = [torch.empty(N, wl.Cout, wl.G, dtype=wl.torch_dtype, pin_memory=True) for _ in range(2)]
    streams = [torch.cuda.Stream(DEV), torch.cuda.Stream(DEV)]
    lib = eq.library()
    torch.cuda.synchronize()
    for k in range(2):
        st = lib.eqlin_forward_host(h.ptr, xs[k].data_ptr(), ys[k].data_ptr(), N, streams[k].cuda_stream)
        assert st == eq.EQLIN_OK
    for s_ in streams:
        s_.synchronize()
    assert h.device_status() == eq.EQLIN_OK
    assert torch.equal(ys[0], ref1) and torch.equal(ys[1], ref2)
    h.close()


@pytest.mark.parametrize("name", ["p4_c96_bf16", "p8_c64_bf16", "p4_mlp_bf16"])
def test_concurrent_forwards_of_one_handle_on_two_streams(name):
    """A prepared handle is read-only on the forward path (weights, bias, plan), so
    forwards of one handle issued on two streams at once, with no synchronisation between
    them, give the same outputs as the same calls made one after the other."""
    wl = workloads.WORKLOADS[name]
    N = 3 * 148 * 64 + 123
    xa, w, bias = workloads.make_inputs(wl, seed=51, N=N)
    xb, _, _ = workloads.make_inputs(wl, seed=52, N=N)
    h = _prep(w, bias, wl.torch_dtype)
    xs = [xa.to(DEV), xb.to(DEV)]
    serial = [h.forward(t).clone() for t in xs]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(DEV), torch.cuda.Stream(DEV)]
    outs = [torch.empty_like(serial[0]) for _ in range(2)]
    for rep in range(3):
        for k in range(2):
            h.forward(xs[k], out=outs[k], stream=streams[k])
        for s_ in streams:
            s_.synchronize()
        assert torch.equal(outs[0], serial[0]) and torch.equal(outs[1], serial[1])
    assert h.device_status() == eq.EQLIN_OK
    h.close()


def test_tolerances_are_the_stated_ones():
    assert TOL_F32_MAXREL == 1e-5 and TOL_BF16_NORMWISE == 2e-2


def test_handles_sharing_a_kernel_keep_their_shared_memory():
    """Two handles of one kernel with different shared-memory plans: preparing the second
    must not shrink what the first one launches with (the limit is per kernel)."""
    gen = torch.Generator().manual_seed(91)
    shapes = [(128, 128, 4), (32, 32, 4)]
    hs, refs, xs = [], [], []
    for Cout, Cin, G in shapes:
        x = torch.randn(300, Cin, G, generator=gen).to(torch.bfloat16)
        w = (torch.randn(Cout, Cin, G, generator=gen) / np.sqrt(Cin * G)).to(torch.bfloat16)
        hs.append(eq.prepare(w.to(DEV), None))
        xs.append(x)
        refs.append(_ref(x, w, None))
    assert hs[0].path == hs[1].path and hs[0].attr("smem_bytes") != hs[1].attr("smem_bytes")
    for h, x, ref in zip(hs, xs, refs):
        y = h.forward(x.to(DEV))
        torch.cuda.synchronize()
        _assert_parity(torch.bfloat16, y, ref, f"path={h.path} smem={h.attr('smem_bytes')}")
        h.close()


@pytest.mark.parametrize("pinned", [True, False])
@pytest.mark.parametrize("name,N", [("p4_c96_bf16", 3 * 10880 + 517), ("p4_c96_bf16", 300), ("p4_mlp_bf16", 20000),
                                    ("c16_c32_bf16", 40000), ("tiny_p4_fp32", 5000)])
def test_forward_from_host_buffers(name, N, pinned):
    """eqlin_forward_host: chunked copies in and out around the fused kernel, several
    chunks with a ragged last one, pinned or pageable host memory; equal to the
    device-buffer forward bit for bit, and to the oracle within the tolerance."""
    wl = workloads.WORKLOADS[name]
    x, w, bias = workloads.make_inputs(wl, seed=21, N=N)
    h = eq.prepare(w.to(DEV), None if bias is None else bias.to(DEV), io_dtype=wl.torch_dtype)
    xh = x.pin_memory() if pinned else x.clone()
    y_host = h.forward_host(xh)
    y_dev = h.forward(x.to(DEV)).cpu()
    assert h.device_status() == eq.EQLIN_OK
    assert torch.equal(y_host, y_dev)
    idx = workloads.sample_tokens(N, 256, seed=4)
    _assert_parity(wl.torch_dtype, y_host[idx], _ref(x[idx], w, bias), f"{name} N={N} pinned={pinned}")
    y2 = h.forward_host(xh, y_host)            # again, into the same output, staging reused
    assert torch.equal(y2, y_dev)
    h.close()
