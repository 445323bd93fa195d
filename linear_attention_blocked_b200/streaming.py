"""Prefill of inputs that live in host memory.

When q, k, v are resident on the host (pinned), the host link, not the
kernel, sets the pace: at B=1, H=64, N=32768 the inputs are 1.61 GB and the
output 0.54 GB, tens of milliseconds over the link against half a
millisecond of compute.  prefill_from_host cuts the sequence into chunks of
tokens and pipelines them over three CUDA streams -- copy in chunk c+1,
scan chunk c, copy out chunk c-1 -- carrying the state from chunk to chunk
(a prefill of chunk c from the state after chunk c-1 is the prefill of the
longer sequence, the state-carry identity of the method), so the copies in
both directions overlap each other and the compute.  The scans are
la_prefill calls; the copies are plain cudaMemcpyAsync through torch.
"""
from __future__ import annotations

import torch

from . import _binding

D = _binding.D


def prefill_from_host(q, k, v, chunk_tokens: int = 4096, state_in=None, out=None, state_out=None,
                      out_dtype=torch.bfloat16, device=None, buffers=None):
    """la_prefill of pinned host tensors q, k, v [B, N, H, d] (bf16).

    Returns (out, state): out is a pinned host tensor [B, N, H, d] (or
    `out`), state the final fp32 state [B, H, d, d] on the device (or
    `state_out`, which may be a device tensor or pinned host tensor).
    state_in: optional fp32 [B, H, d, d] device tensor.  `buffers`: the
    device buffers of make_buffers(B, chunk_tokens, H, ...), reused across
    calls to avoid allocating device memory per call (made per call when
    None).  The call returns once every copy has been enqueued; the caller
    synchronises (for example torch.cuda.synchronize()) before reading
    `out`.
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
    bufs = buffers if buffers is not None else make_buffers(B, min(chunk_tokens, max(N, 1)), H, out.dtype, device)
    C = bufs["chunk_tokens"]  # the chunk length the buffers were made for
    if C < min(chunk_tokens, N) or bufs["B"] != B or bufs["H"] != H or bufs["out_dtype"] != out.dtype:
        raise ValueError("buffers were made for another shape")
    state = bufs["state"]
    s_in, s_cmp, s_out = bufs["streams"]
    main = torch.cuda.current_stream(device)
    # the state starts as state_in (or zero) on the compute stream
    s_cmp.wait_stream(main)
    with torch.cuda.stream(s_cmp):
        if state_in is not None:
            _binding.state_prefix(None, 0, state_in, out=state)
        else:
            _binding.state_prefix(None, 0, None, out=state)
    s_in.wait_stream(main)
    s_out.wait_stream(main)
    nchunks = (N + C - 1) // C if N > 0 else 0
    if nchunks:
        # a shorter last chunk may use shorter segments and more scratch than a full one
        need = max(_binding.workspace_size(B, min(C, N), H, d), _binding.workspace_size(B, N - (nchunks - 1) * C, H, d))
        if bufs["workspace"].numel() < need:
            bufs["workspace"] = torch.empty(need, dtype=torch.uint8, device=device)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for c in range(nchunks):
        j = c & 1
        t0, t1 = c * C, min(N, (c + 1) * C)
        n = t1 - t0
        qd, kd, vd, od = (bufs[x][j][:, :n] for x in ("q", "k", "v", "out"))
        # copy in: slot j is free once the chunk two before has been copied out
        with torch.cuda.stream(s_in):
            if c >= 2:
                s_in.wait_event(ev_out[j])
                s_in.wait_event(ev_cmp[j])
            for b in range(B):
                qd[b].copy_(q[b, t0:t1], non_blocking=True)
                kd[b].copy_(k[b, t0:t1], non_blocking=True)
                vd[b].copy_(v[b, t0:t1], non_blocking=True)
            ev_in[j].record(s_in)
        # scan the chunk from the carried state (in place)
        with torch.cuda.stream(s_cmp):
            s_cmp.wait_event(ev_in[j])
            if c >= 2:
                s_cmp.wait_event(ev_out[j])  # the output slot has been copied out
            qc, kc, vc, oc = (x if n == C else x.contiguous() for x in (qd, kd, vd, od))
            _binding.prefill(qc, kc, vc, state_in=state, out=oc, state_out=state,
                             workspace=bufs["workspace"], stream=s_cmp)
            if oc is not od:
                od.copy_(oc)
            ev_cmp[j].record(s_cmp)
        # copy out
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[j])
            for b in range(B):
                out[b, t0:t1].copy_(od[b], non_blocking=True)
            ev_out[j].record(s_out)
    # the caller's stream sees every result
    main.wait_stream(s_cmp)
    main.wait_stream(s_out)
    if state_out is not None:
        state_out.copy_(state, non_blocking=True)
        return out, state_out
    return out, state.clone()


def make_buffers(B: int, chunk_tokens: int, H: int, out_dtype=torch.bfloat16, device=None):
    """Device buffers for prefill_from_host: two slots of q, k, v and out
    chunks, the running state, a prefill workspace and three streams."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    C = int(chunk_tokens)
    shape = (B, C, H, D)
    mk = lambda dt: [torch.empty(shape, dtype=dt, device=device) for _ in range(2)]  # noqa: E731
    return {
        "B": B, "H": H, "chunk_tokens": C, "out_dtype": out_dtype,
        "q": mk(torch.bfloat16), "k": mk(torch.bfloat16), "v": mk(torch.bfloat16), "out": mk(out_dtype),
        "state": torch.empty((B, H, D, D), dtype=torch.float32, device=device),
        "workspace": torch.empty(max(256, _binding.workspace_size(B, C, H, D)), dtype=torch.uint8, device=device),
        "streams": tuple(torch.cuda.Stream(device) for _ in range(3)),
    }
