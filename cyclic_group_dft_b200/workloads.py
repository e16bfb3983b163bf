"""Seeded synthetic workloads for the EQ-Linear forward.

This module holds shapes, dtypes, distributions and seeds only -- none of the
layer's arithmetic -- so both the CUDA path and the float64 oracle can be fed
identical inputs from it.

Six workloads, all EQ-Linear over the cyclic group C_G with layout
x [N, Cin, G], w [Cout, Cin, G], y [N, Cout, G] (G fastest):

===================  =======  ====  =====  ===  =====  =====================
name                 N        Cin   Cout   G    I/O    role
===================  =======  ====  =====  ===  =====  =====================
tiny_p4_fp32         256      16    16     4    fp32   small parity case
p4_c96_bf16          200704   96    96     4    bf16   headline (64*56*56)
p8_c64_bf16          25088    64    64     8    bf16   p8 group (32*28*28)
p4_mlp_bf16          65536    192   768    4    bf16   MLP expansion, no bias
c16_c32_bf16         262144   32    32     16   bf16   C16 group
p4_c96_f16           200704   96    96     4    fp16   headline shape, FP16 I/O
===================  =======  ====  =====  ===  =====  =====================

Distributions: x ~ N(0, 1); w ~ N(0, 1/(Cin*G)); bias ~ N(0, 0.1), where the
second parameter is read as the variance (std = sqrt).  The p4 MLP workload
has no bias.  Values are drawn in fp32 from one CPU ``torch.Generator`` seeded
with the workload seed, in the order w, bias, x (weights first, so they do not
depend on N), then rounded to the I/O dtype (round-to-nearest-even).
"""
from __future__ import annotations

import dataclasses
import math

import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    N: int
    Cin: int
    Cout: int
    G: int
    io_dtype: str          # "f32", "bf16" or "f16"
    w_var: float           # variance of w
    bias_var: float | None  # variance of bias; None = no bias (zero)
    seed: int = 0
    about: str = ""

    @property
    def torch_dtype(self) -> torch.dtype:
        return DTYPES[self.io_dtype]

    @property
    def elem_bytes(self) -> int:
        return 4 if self.io_dtype == "f32" else 2

    def with_n(self, N: int) -> "Workload":
        return dataclasses.replace(self, N=int(N))


WORKLOADS: dict[str, Workload] = {
    w.name: w for w in [
        Workload("tiny_p4_fp32", 256, 16, 16, 4, "f32", 1.0 / (16 * 4), 0.1, 0,
                 "tiny p4 EQ-Linear, fp32 I/O"),
        Workload("p4_c96_bf16", 64 * 56 * 56, 96, 96, 4, "bf16", 1.0 / (96 * 4), 0.1, 0,
                 "p4 EQ-Linear sized like a visual-Mamba projection, bf16 I/O"),
        Workload("p8_c64_bf16", 32 * 28 * 28, 64, 64, 8, "bf16", 1.0 / (64 * 8), 0.1, 0,
                 "p8 EQ-Linear, bf16 I/O"),
        Workload("p4_mlp_bf16", 65536, 192, 768, 4, "bf16", 1.0 / (192 * 4), None, 0,
                 "p4 MLP-expansion EQ-Linear, bf16 I/O, no bias"),
        Workload("c16_c32_bf16", 262144, 32, 32, 16, "bf16", 1.0 / (32 * 16), 0.1, 0,
                 "C16 EQ-Linear, bf16 I/O"),
        Workload("p4_c96_f16", 64 * 56 * 56, 96, 96, 4, "f16", 1.0 / (96 * 4), 0.1, 0,
                 "the headline p4 shape with FP16 I/O"),
    ]
}

HEADLINE = "p4_c96_bf16"


def _draw_weights(wl: Workload, gen: torch.Generator):
    w = torch.randn(wl.Cout, wl.Cin, wl.G, generator=gen) * math.sqrt(wl.w_var)
    bias = None
    if wl.bias_var is not None:
        bias = torch.randn(wl.Cout, generator=gen) * math.sqrt(wl.bias_var)
    return w.to(wl.torch_dtype), (None if bias is None else bias.to(wl.torch_dtype))


def make_weights(wl: Workload, seed: int | None = None):
    """(w, bias) as CPU tensors in the I/O dtype; bias is None for no-bias workloads."""
    gen = torch.Generator(device="cpu").manual_seed(wl.seed if seed is None else int(seed))
    return _draw_weights(wl, gen)


def make_inputs(wl: Workload, seed: int | None = None, N: int | None = None):
    """(x, w, bias) as CPU tensors in the I/O dtype.

    ``N`` overrides the token count (weights are unaffected by it).
    """
    gen = torch.Generator(device="cpu").manual_seed(wl.seed if seed is None else int(seed))
    w, bias = _draw_weights(wl, gen)
    n = wl.N if N is None else int(N)
    x = torch.randn(n, wl.Cin, wl.G, generator=gen).to(wl.torch_dtype)
    return x, w, bias


def sample_tokens(N: int, count: int, seed: int = 0) -> torch.Tensor:
    """Sorted token indices for sampled checks: first, last, and random ones."""
    if N <= count:
        return torch.arange(N)
    gen = torch.Generator(device="cpu").manual_seed(seed)
    idx = torch.randperm(N, generator=gen)[: max(count - 2, 0)]
    idx = torch.cat([idx, torch.tensor([0, N - 1])])
    return torch.unique(idx)


def make_mlp_weights(wl: Workload, hidden: int, seed: int | None = None):
    """(w1 [H, Cin, G], b1 [H], w2 [Cout, H, G], b2 [Cout]) for the equivariant MLP block
    L2(GELU(L1(x))) at the workload's channels, as CPU tensors in the I/O dtype:
    w1 ~ N(0, 1/(Cin*G)), w2 ~ N(0, 1/(H*G)), biases ~ N(0, 0.1) (second parameter the
    variance), drawn in that order from one generator (seed + 1000 by default, so
    they differ from the single-layer weights)."""
    gen = torch.Generator(device="cpu").manual_seed((wl.seed if seed is None else int(seed)) + 1000)
    G, H = wl.G, int(hidden)
    w1 = torch.randn(H, wl.Cin, G, generator=gen) * math.sqrt(1.0 / (wl.Cin * G))
    b1 = torch.randn(H, generator=gen) * math.sqrt(0.1)
    w2 = torch.randn(wl.Cout, H, G, generator=gen) * math.sqrt(1.0 / (H * G))
    b2 = torch.randn(wl.Cout, generator=gen) * math.sqrt(0.1)
    dt = wl.torch_dtype
    return w1.to(dt), b1.to(dt), w2.to(dt), b2.to(dt)
