"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench.

This module holds no attention arithmetic: it only draws random numbers,
rounds them once to bf16 and moves bit patterns around, so that the CUDA
path and the CPU oracle receive identical inputs.

Recipe (the workloads are shaped like the MiniMax-01 attention layers: 64 heads
of dimension 128, contexts up to 1M tokens):
  * q, k, v: iid N(0, 1) in fp32, times ``scale`` (default 128**-0.5), rounded
    once to bf16 (round-to-nearest-even, torch's conversion), drawn in the
    order q, k, v from one ``torch.Generator`` seeded with ``seed``.
  * packed varlen lengths: ``numpy.random.default_rng(seed).integers(lo, hi+1, n)``.
  * decode step s of a run seeded ``seed`` uses seed ``seed * 1_000_003 + s``.
"""
from __future__ import annotations

import numpy as np
import torch

DEFAULT_SCALE = 128 ** -0.5


def qkv(shape, seed: int, device="cpu", scale: float = DEFAULT_SCALE):
    """Three bf16 tensors of ``shape`` (e.g. [T, H, d] or [B, N, H, d])."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    out = []
    for _ in range(3):
        x = torch.randn(tuple(shape), generator=gen, device=device, dtype=torch.float32)
        out.append((x * scale).to(torch.bfloat16))
    return tuple(out)


def varlen_lengths(n: int, lo: int, hi: int, seed: int) -> np.ndarray:
    """``n`` sequence lengths uniform in [lo, hi] (inclusive)."""
    return np.random.default_rng(int(seed)).integers(lo, hi + 1, n).astype(np.int64)


def cu_seqlens_from_lengths(lengths) -> np.ndarray:
    """int32 prefix offsets [0, l0, l0+l1, ...]."""
    cu = np.zeros(len(lengths) + 1, dtype=np.int64)
    cu[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64))
    return cu.astype(np.int32)


def decode_seed(seed: int, step: int) -> int:
    return int(seed) * 1_000_003 + int(step)


def bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor (any device) -> numpy uint16 bit patterns, same shape."""
    if t.dtype != torch.bfloat16:
        raise TypeError("expected a bf16 tensor")
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def from_bits(b: np.ndarray) -> torch.Tensor:
    """numpy uint16 bit patterns -> CPU bf16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(b, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)


def bf16_exact(values) -> np.ndarray:
    """Bit patterns of values that bf16 represents exactly (raises otherwise)."""
    a = np.asarray(values, dtype=np.float32)
    b = torch.from_numpy(a).to(torch.bfloat16)
    if not np.array_equal(b.to(torch.float32).numpy(), a):
        raise ValueError("value not exactly representable in bf16")
    return bits(b)
