"""Parity helpers shared by the GPU tests: run the CUDA path, run the oracle on
the same inputs, compare with the tolerances the spec states.

Tolerances
  fp32 I/O : max_j |y_j - o_j| / max(|o_j|, 1e-3 * max|o|) <= 1e-5
  bf16 / fp16 I/O : ||y - o||_2 / ||o||_2 <= 2e-2 (normwise over the whole output)
plus, for bf16, a tighter bound derived from the arithmetic (bf16 rounding of
the input spectrum, of the weight spectrum and of y, each relative error
<= 2^-9, fp32 accumulation): normwise <= BF16_DERIVED (~3x the expected
~2e-3), used to catch structural mistakes the loose spec bound would hide;
for fp16 I/O the same derivation with 2^-11 gives F16_DERIVED (~3x the
expected ~5e-4).
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TOL_F32_MAXREL = 1e-5
TOL_BF16_NORMWISE = 2e-2
BF16_DERIVED = 6e-3
F16_DERIVED = 1.5e-3


def f32_maxrel(y, ref) -> float:
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    floor = 1e-3 * np.abs(ref).max()
    return float((np.abs(y - ref) / np.maximum(np.abs(ref), floor)).max())


def normwise(y, ref) -> float:
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    return float(np.linalg.norm(y - ref) / max(np.linalg.norm(ref), 1e-300))


def oracle_forward(x, w, bias, threads: int = 0) -> np.ndarray:
    return oracle.forward(x, w, bias, threads=threads)


def check(dtype: torch.dtype, y_gpu: torch.Tensor, ref: np.ndarray) -> dict:
    y = y_gpu.detach().float().cpu().numpy()
    out = {"normwise": normwise(y, ref), "f32_maxrel": f32_maxrel(y, ref),
           "max_abs": float(np.abs(y - ref).max()) if ref.size else 0.0}
    if dtype == torch.float32:
        out["ok"] = out["f32_maxrel"] <= TOL_F32_MAXREL
    else:
        derived = F16_DERIVED if dtype == torch.float16 else BF16_DERIVED
        out["ok"] = out["normwise"] <= TOL_BF16_NORMWISE and out["normwise"] <= derived
    return out
