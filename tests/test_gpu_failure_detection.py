"""Failure detection on the GPU without a GPU fault.

Every wait inside the fused kernels is bounded (global timer); when one runs out
the kernel records EQLIN_ERR_TIMEOUT in the handle's device status word, every role
leaves its loop, in-flight copies and MMAs are drained with bounded waits, TMEM is
freed and the kernel returns.  The test makes a wait run out on purpose through the
test hook EQLIN_TEST_STOP_AFTER (read at prepare): the producer stops issuing input
chunks after k of them, so the consumers wait for a chunk that never comes.  No
fault, trap or unbounded wait is involved.  The test then checks that the status
comes back to the host and that the same process keeps computing correct results.
"""
from __future__ import annotations

import pytest
import torch

import cyclic_group_dft_b200 as eq
import oracle
from cyclic_group_dft_b200 import workloads
from parity_util import check

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.mark.parametrize("kernel,name", [("tn", "p4_c96_bf16"), ("tm", "c16_c32_bf16"), ("tnr", "p4_mlp_bf16")])
def test_wait_timeout_is_reported_and_the_gpu_stays_usable(kernel, name, monkeypatch):
    wl = workloads.WORKLOADS[name]
    x, w, bias = workloads.make_inputs(wl, N=4 * 148 * 128)
    xd = x.to(DEV)
    monkeypatch.setenv("EQLIN_KERNEL", kernel)
    monkeypatch.setenv("EQLIN_WAIT_TIMEOUT_MS", "200")
    monkeypatch.setenv("EQLIN_TEST_STOP_AFTER", "3")
    bd = None if bias is None else bias.to(DEV)
    h = eq.prepare(w.to(DEV), bd, io_dtype=wl.torch_dtype)
    h.forward(xd)
    torch.cuda.synchronize()                   # the kernel returns: no hang, no fault
    assert h.device_status() == eq.EQLIN_ERR_TIMEOUT
    assert h.device_status() == eq.EQLIN_OK    # reading the word clears it
    h.close()

    monkeypatch.delenv("EQLIN_TEST_STOP_AFTER")
    h = eq.prepare(w.to(DEV), bd, io_dtype=wl.torch_dtype)
    y = h.forward(xd)
    torch.cuda.synchronize()
    assert h.device_status() == eq.EQLIN_OK
    idx = workloads.sample_tokens(x.shape[0], 256, seed=3)
    r = check(wl.torch_dtype, y.cpu()[idx], oracle.forward(x[idx], w, bias))
    assert r["ok"], r
    h.close()


def test_sync_check_returns_the_timeout(monkeypatch):
    """With EQLIN_SYNC_CHECK=1 the forward itself synchronises and returns the status."""
    wl = workloads.WORKLOADS["p4_c96_bf16"]
    x, w, bias = workloads.make_inputs(wl, N=148 * 64 * 4)
    monkeypatch.setenv("EQLIN_WAIT_TIMEOUT_MS", "200")
    monkeypatch.setenv("EQLIN_TEST_STOP_AFTER", "1")
    monkeypatch.setenv("EQLIN_SYNC_CHECK", "1")
    h = eq.prepare(w.to(DEV), bias.to(DEV))
    with pytest.raises(eq.EqlinError) as e:
        h.forward(x.to(DEV))
    assert e.value.status == eq.EQLIN_ERR_TIMEOUT
    h.close()
