"""Prefill of inputs that live in host memory (la_prefill_from_host).

When q, k, v are resident on the host (pinned), the host link, not the
kernel, sets the pace: at B=1, H=64, N=32768 the inputs are 1.61 GB and the
output 0.54 GB, tens of milliseconds over the link against half a
millisecond of compute.  The C entry point la_prefill_from_host cuts the
sequence into chunks of tokens and pipelines them over three CUDA streams --
copy in chunk c+1, scan chunk c, copy out chunk c-1 -- carrying the state
from chunk to chunk (a prefill of chunk c from the state after chunk c-1 is
the prefill of the longer sequence, the state-carry identity of the method),
so the copies in both directions overlap each other and the compute.  This
module only checks and marshals arguments: the pipeline, its copies, events
and scans are the library's.
"""
from __future__ import annotations

import ctypes

import torch

from . import _binding

D = _binding.D


def prefill_from_host(q, k, v, chunk_tokens: int = 4096, state_in=None, out=None, state_out=None,
                      out_dtype=torch.bfloat16, device=None, buffers=None):
    """la_prefill_from_host on pinned host tensors q, k, v [B, N, H, d] (bf16).

    Returns (out, state): out is a pinned host tensor [B, N, H, d] (or
    `out`), state the final fp32 state [B, H, d, d] on the device (or
    `state_out`, a device tensor or a pinned host tensor).  state_in:
    optional fp32 [B, H, d, d] device tensor.  `buffers`: the device buffers
    and streams of make_buffers(B, chunk_tokens, H, ...), reused across calls
    so that no device memory is allocated per call (made per call when None).
    The call returns once every copy has been enqueued; work queued on the
    current stream afterwards sees every result, and the caller synchronises
    (for example torch.cuda.synchronize()) before reading `out` on the host.
    """
    if q.dim() != 4:
        raise ValueError("q must be [B, N, H, d]")
    B, N, H, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.is_cuda or t.dtype != torch.bfloat16 or tuple(t.shape) != (B, N, H, d) or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous host bf16 tensor of shape {(B, N, H, d)}")
        if t.numel() and not t.is_pinned():
            raise ValueError(f"{name} must be in pinned host memory")
    if chunk_tokens <= 0:
        raise ValueError("chunk_tokens must be positive")
    if buffers is not None:
        device = buffers["state"].device
    elif device is None:
        device = torch.device("cuda", torch.cuda.current_device())
    else:
        device = torch.device(device)
    if out is None:
        out = torch.empty((B, N, H, d), dtype=out_dtype, pin_memory=True)
    if out.is_cuda or tuple(out.shape) != (B, N, H, d) or not out.is_contiguous():
        raise ValueError("out must be a contiguous host tensor of the shape of q")
    if out.numel() and not out.is_pinned():
        raise ValueError("out must be in pinned host memory")
    code = _binding._out_code(out.dtype)
    bufs = buffers if buffers is not None else make_buffers(B, chunk_tokens, H, out.dtype, device)
    if bufs["B"] != B or bufs["H"] != H or bufs["out_dtype"] != out.dtype or bufs["chunk_tokens"] < chunk_tokens:
        raise ValueError("buffers were made for another shape")
    if state_in is not None:
        _binding._need(state_in, "state_in", torch.float32, (B, H, d, d))
    if state_out is None:
        state_out = torch.empty((B, H, d, d), dtype=torch.float32, device=device)
    if tuple(state_out.shape) != (B, H, d, d) or state_out.dtype != torch.float32 or not state_out.is_contiguous():
        raise ValueError("state_out must be a contiguous fp32 tensor [B, H, d, d]")
    if not state_out.is_cuda and not state_out.is_pinned():
        raise ValueError("a host state_out must be in pinned memory")
    s_in, s_out = bufs["streams"]
    compute = torch.cuda.current_stream(device)
    ptr = lambda t: None if t is None or t.numel() == 0 else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    sh = lambda s: ctypes.c_void_p(s.cuda_stream)  # noqa: E731
    nbytes = bufs["buffer"].numel()
    with torch.cuda.device(device):
        st = _binding.lib().la_prefill_from_host(ptr(q), ptr(k), ptr(v), B, N, H, d, int(chunk_tokens), ptr(state_in),
                                                 ptr(out), code, ptr(state_out), ptr(bufs["buffer"]), nbytes,
                                                 sh(s_in), sh(compute), sh(s_out))
    _binding._check(st, "la_prefill_from_host")
    return out, state_out


def make_buffers(B: int, chunk_tokens: int, H: int, out_dtype=torch.bfloat16, device=None):
    """Device scratch for prefill_from_host (la_prefill_from_host_buffer_size
    bytes: two chunk slots of q, k, v and out, the running state, a prefill
    workspace) and the two copy streams."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    C = int(chunk_tokens)
    nbytes = int(_binding.lib().la_prefill_from_host_buffer_size(B, C, H, D, _binding._out_code(out_dtype)))
    if nbytes == 0:
        raise ValueError("invalid shape for prefill_from_host buffers")
    return {
        "B": B, "H": H, "chunk_tokens": C, "out_dtype": out_dtype,
        "buffer": torch.empty(nbytes, dtype=torch.uint8, device=device),
        "state": torch.empty((1,), dtype=torch.float32, device=device),  # marks the device of the buffers
        "streams": tuple(torch.cuda.Stream(device) for _ in range(2)),
    }
