"""ctypes binding of the C ABI in include/lightning_attn.h.

Argument marshalling only: shapes, dtypes and pointers are checked and handed
to the CUDA library, which does every step of the computation on the GPU.
PyTorch provides device memory (outputs, workspace) and the current stream.
There is no CPU fallback: if the library or a GPU is missing, calls raise.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import _build

LA_OK, LA_ERR_INVALID_ARGUMENT, LA_ERR_UNSUPPORTED, LA_ERR_CUDA, LA_ERR_TIMEOUT, LA_ERR_WORKSPACE = range(6)
LA_BF16, LA_FP32 = 0, 1
LA_INJECT_NONE, LA_INJECT_SKIP_PUBLISH = 0, 1
D = 128
DEFAULT_BLOCK = 128

EXPORTED = ("la_prefill_workspace_size", "la_prefill", "la_prefill_varlen_workspace_size",
            "la_prefill_varlen", "la_decode_step", "la_get_device_status", "la_status_string",
            "la_set_wait_limit_ns", "la_set_segment_len", "la_debug_inject",
            "la_last_segment_len", "la_kernel_launches", "la_prefill_noalloc",
            "la_prefill_varlen_slots", "la_decode_step_slots", "la_mixed_step",
            "la_kv_aggregate_workspace_size", "la_kv_aggregate", "la_state_prefix",
            "la_prefill_backward_workspace_size", "la_prefill_backward", "la_prefill_decay",
            "la_prefill_varlen_decay", "la_decode_step_decay", "la_prefill_from_host_buffer_size",
            "la_prefill_from_host", "la_prefill_backward_varlen_workspace_size", "la_prefill_backward_varlen")


class LAError(RuntimeError):
    """A non-OK status from the library."""

    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {status_string(status)} (status {status})")


_lib = None


def library_path() -> str:
    return _build.LIB_PATH


def lib():
    """Load the in-tree shared library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        path = _build.LIB_PATH
        if not os.path.exists(path):
            raise ImportError(f"CUDA library not built: {path} is missing "
                              "(run linear_attention_blocked_b200._build.build())")
        L = ctypes.CDLL(path)
        vp, c_int, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.la_prefill_workspace_size.argtypes = [c_int] * 5
        L.la_prefill_workspace_size.restype = sz
        L.la_prefill.argtypes = [vp, vp, vp, c_int, c_int, c_int, c_int, c_int, vp, vp, c_int, vp, vp, sz, vp]
        L.la_prefill.restype = c_int
        L.la_prefill_varlen_workspace_size.argtypes = [c_int] * 6
        L.la_prefill_varlen_workspace_size.restype = sz
        L.la_prefill_varlen.argtypes = [vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_int,
                                        vp, vp, c_int, vp, vp, sz, vp]
        L.la_prefill_varlen.restype = c_int
        L.la_prefill_noalloc.argtypes = [vp, vp, vp, c_int, c_int, c_int, c_int, c_int, vp, vp, c_int, vp, vp]
        L.la_prefill_noalloc.restype = c_int
        L.la_decode_step.argtypes = [vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, vp]
        L.la_decode_step.restype = c_int
        L.la_prefill_decay.argtypes = [vp, vp, vp, c_int, c_int, c_int, c_int, c_int, vp, vp, vp, c_int, vp, vp,
                                       sz, vp]
        L.la_prefill_decay.restype = c_int
        L.la_prefill_varlen_decay.argtypes = [vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_int, vp,
                                              vp, vp, c_int, vp, vp, sz, vp]
        L.la_prefill_varlen_decay.restype = c_int
        L.la_decode_step_decay.argtypes = [vp, vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, vp]
        L.la_decode_step_decay.restype = c_int
        L.la_prefill_from_host_buffer_size.argtypes = [c_int, c_int, c_int, c_int, c_int]
        L.la_prefill_from_host_buffer_size.restype = sz
        L.la_prefill_from_host.argtypes = [vp, vp, vp, c_int, c_int, c_int, c_int, c_int, vp, vp, c_int, vp, vp, sz,
                                           vp, vp, vp]
        L.la_prefill_from_host.restype = c_int
        L.la_prefill_varlen_slots.argtypes = [vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_int, c_int,
                                              vp, c_int, vp, c_int, vp, sz, vp]
        L.la_prefill_varlen_slots.restype = c_int
        L.la_decode_step_slots.argtypes = [vp, vp, vp, vp, c_int, vp, vp, c_int, c_int, c_int, c_int, vp]
        L.la_decode_step_slots.restype = c_int
        L.la_mixed_step.argtypes = [vp, vp, vp, vp, vp, c_int, c_int, c_int, vp, c_int, c_int, c_int, vp, c_int,
                                    vp, c_int, vp, sz, vp, vp]
        L.la_mixed_step.restype = c_int
        L.la_kv_aggregate_workspace_size.argtypes = [c_int] * 4
        L.la_kv_aggregate_workspace_size.restype = sz
        L.la_kv_aggregate.argtypes = [vp, vp, c_int, c_int, c_int, c_int, vp, vp, sz, vp]
        L.la_kv_aggregate.restype = c_int
        L.la_state_prefix.argtypes = [vp, c_int, vp, vp, c_int, c_int, vp]
        L.la_state_prefix.restype = c_int
        L.la_prefill_backward_workspace_size.argtypes = [c_int] * 4
        L.la_prefill_backward_workspace_size.restype = sz
        L.la_prefill_backward.argtypes = [vp, vp, vp, vp, c_int, c_int, c_int, c_int, vp, vp, vp, vp, vp, c_int, vp,
                                          vp, sz, vp]
        L.la_prefill_backward.restype = c_int
        L.la_prefill_backward_varlen_workspace_size.argtypes = [c_int] * 5
        L.la_prefill_backward_varlen_workspace_size.restype = sz
        L.la_prefill_backward_varlen.argtypes = [vp, vp, vp, vp, vp, c_int, c_int, c_int, c_int, c_int, vp, vp, vp,
                                                 vp, vp, c_int, vp, vp, sz, vp]
        L.la_prefill_backward_varlen.restype = c_int
        L.la_get_device_status.argtypes = [vp]
        L.la_get_device_status.restype = c_int
        L.la_status_string.argtypes = [c_int]
        L.la_status_string.restype = ctypes.c_char_p
        L.la_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
        L.la_set_wait_limit_ns.restype = c_int
        L.la_set_segment_len.argtypes = [c_int]
        L.la_set_segment_len.restype = c_int
        L.la_debug_inject.argtypes = [c_int]
        L.la_debug_inject.restype = c_int
        L.la_last_segment_len.argtypes = []
        L.la_last_segment_len.restype = c_int
        L.la_kernel_launches.argtypes = []
        L.la_kernel_launches.restype = ctypes.c_ulonglong
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().la_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != LA_OK:
        raise LAError(status, where)


def _stream_handle(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _out_code(dtype):
    if dtype == torch.bfloat16:
        return LA_BF16
    if dtype == torch.float32:
        return LA_FP32
    raise TypeError("out dtype must be torch.bfloat16 or torch.float32")


def _need(t, name, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def workspace_size(B: int, N: int, H: int, d: int = D, block: int = 0) -> int:
    return int(lib().la_prefill_workspace_size(B, N, H, d, block))


def varlen_workspace_size(nseq: int, total_tokens: int, max_seqlen: int, H: int, d: int = D,
                          block: int = 0) -> int:
    return int(lib().la_prefill_varlen_workspace_size(nseq, total_tokens, max_seqlen, H, d, block))


def _alloc_workspace(nbytes, device):
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def _need_decay(decay, H, device):
    if decay is None:
        return None
    _need(decay, "decay", torch.float32, (H,))
    if decay.device != device:
        raise ValueError("decay must be on the device of q")
    return decay


def prefill(q, k, v, block: int = 0, state_in=None, out=None, out_dtype=torch.bfloat16,
            state_out=None, want_state: bool = True, workspace=None, stream=None, decay=None):
    """la_prefill on [B, N, H, d] bf16 tensors (la_prefill_decay when `decay`,
    a device fp32 [H] tensor of per-head decays in (0, 1], is given).
    Returns (out, state_out or None)."""
    if q.dim() != 4:
        raise ValueError("q must be [B, N, H, d]")
    B, N, H, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, torch.bfloat16, (B, N, H, d))
    if out is None:
        out = torch.empty((B, N, H, d), dtype=out_dtype, device=q.device)
    _need(out, "out", out.dtype, (B, N, H, d))
    if state_in is not None:
        _need(state_in, "state_in", torch.float32, (B, H, d, d))
    if state_out is None and want_state:
        state_out = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device)
    if state_out is not None:
        _need(state_out, "state_out", torch.float32, (B, H, d, d))
    decay = _need_decay(decay, H, q.device)
    ws_bytes = workspace_size(B, N, H, d, block)
    if workspace is None:
        workspace = _alloc_workspace(ws_bytes, q.device)
    if decay is None:
        st = lib().la_prefill(_ptr(q), _ptr(k), _ptr(v), B, N, H, d, block, _ptr(state_in), _ptr(out),
                              _out_code(out.dtype), _ptr(state_out), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream_handle(stream))
        _check(st, "la_prefill")
    else:
        st = lib().la_prefill_decay(_ptr(q), _ptr(k), _ptr(v), B, N, H, d, block, _ptr(decay), _ptr(state_in),
                                    _ptr(out), _out_code(out.dtype), _ptr(state_out), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream_handle(stream))
        _check(st, "la_prefill_decay")
    return out, state_out


def prefill_varlen(q, k, v, cu_seqlens, max_seqlen: int, block: int = 0, state_in=None, out=None,
                   out_dtype=torch.bfloat16, state_out=None, want_state: bool = True, workspace=None,
                   stream=None, decay=None):
    """la_prefill_varlen on packed [T, H, d] tensors with device int32 cu_seqlens
    (la_prefill_varlen_decay when `decay`, device fp32 [H], is given)."""
    if q.dim() != 3:
        raise ValueError("q must be [T, H, d]")
    T, H, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, torch.bfloat16, (T, H, d))
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    nseq = cu_seqlens.numel() - 1
    if nseq < 0:
        raise ValueError("cu_seqlens must hold nseq + 1 entries")
    if out is None:
        out = torch.empty((T, H, d), dtype=out_dtype, device=q.device)
    _need(out, "out", out.dtype, (T, H, d))
    if state_in is not None:
        _need(state_in, "state_in", torch.float32, (nseq, H, d, d))
    if state_out is None and want_state:
        state_out = torch.empty((nseq, H, d, d), dtype=torch.float32, device=q.device)
    if state_out is not None:
        _need(state_out, "state_out", torch.float32, (nseq, H, d, d))
    decay = _need_decay(decay, H, q.device)
    ws_bytes = varlen_workspace_size(nseq, T, max_seqlen, H, d, block)
    if workspace is None:
        workspace = _alloc_workspace(ws_bytes, q.device)
    if decay is None:
        st = lib().la_prefill_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), nseq, T, int(max_seqlen),
                                     H, d, block, _ptr(state_in), _ptr(out), _out_code(out.dtype),
                                     _ptr(state_out), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(), _stream_handle(stream))
        _check(st, "la_prefill_varlen")
    else:
        st = lib().la_prefill_varlen_decay(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), nseq, T, int(max_seqlen),
                                           H, d, block, _ptr(decay), _ptr(state_in), _ptr(out),
                                           _out_code(out.dtype), _ptr(state_out), _ptr(workspace),
                                           workspace.numel() * workspace.element_size(), _stream_handle(stream))
        _check(st, "la_prefill_varlen_decay")
    return out, state_out


def decode_step(q, k, v, state, out=None, out_dtype=torch.bfloat16, stream=None, decay=None):
    """la_decode_step on [B, H, d] bf16 tensors; `state` [B, H, d, d] fp32 is updated in place
    (la_decode_step_decay when `decay`, device fp32 [H], is given)."""
    if q.dim() != 3:
        raise ValueError("q must be [B, H, d]")
    B, H, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, torch.bfloat16, (B, H, d))
    _need(state, "state", torch.float32, (B, H, d, d))
    if out is None:
        out = torch.empty((B, H, d), dtype=out_dtype, device=q.device)
    _need(out, "out", out.dtype, (B, H, d))
    decay = _need_decay(decay, H, q.device)
    if decay is None:
        st = lib().la_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(state), _ptr(out), _out_code(out.dtype),
                                  B, H, d, _stream_handle(stream))
        _check(st, "la_decode_step")
    else:
        st = lib().la_decode_step_decay(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(state), _ptr(out),
                                        _out_code(out.dtype), B, H, d, _stream_handle(stream))
        _check(st, "la_decode_step_decay")
    return out


def _need_pool(state_pool, H, d):
    if state_pool.dim() != 4:
        raise ValueError("state_pool must be [n_slots, H, d, d]")
    _need(state_pool, "state_pool", torch.float32, (state_pool.shape[0], H, d, d))
    return int(state_pool.shape[0])


def prefill_varlen_slots(q, k, v, cu_seqlens, slots, max_seqlen: int, state_pool, out=None,
                         out_dtype=torch.bfloat16, workspace=None, stream=None):
    """la_prefill_varlen_slots: sequence i starts from state_pool[slots[i]] and
    leaves its final state there.  slots: device int32 [nseq]."""
    if q.dim() != 3:
        raise ValueError("q must be [T, H, d]")
    T, H, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, torch.bfloat16, (T, H, d))
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    nseq = cu_seqlens.numel() - 1
    _need(slots, "slots", torch.int32, (nseq,))
    n_slots = _need_pool(state_pool, H, d)
    if out is None:
        out = torch.empty((T, H, d), dtype=out_dtype, device=q.device)
    _need(out, "out", out.dtype, (T, H, d))
    ws_bytes = varlen_workspace_size(nseq, T, max_seqlen, H, d)
    if workspace is None:
        workspace = _alloc_workspace(ws_bytes, q.device)
    st = lib().la_prefill_varlen_slots(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), _ptr(slots), nseq, T,
                                       int(max_seqlen), H, d, 0, _ptr(state_pool), n_slots, _ptr(out),
                                       _out_code(out.dtype), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _check(st, "la_prefill_varlen_slots")
    return out


def decode_step_slots(q, k, v, state_pool, slots, out=None, out_dtype=torch.bfloat16, stream=None):
    """la_decode_step_slots: row b updates state_pool[slots[b]] in place."""
    if q.dim() != 3:
        raise ValueError("q must be [B, H, d]")
    B, H, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, torch.bfloat16, (B, H, d))
    _need(slots, "slots", torch.int32, (B,))
    n_slots = _need_pool(state_pool, H, d)
    if out is None:
        out = torch.empty((B, H, d), dtype=out_dtype, device=q.device)
    _need(out, "out", out.dtype, (B, H, d))
    st = lib().la_decode_step_slots(_ptr(q), _ptr(k), _ptr(v), _ptr(state_pool), n_slots, _ptr(slots),
                                    _ptr(out), _out_code(out.dtype), B, H, d, _stream_handle(stream))
    _check(st, "la_decode_step_slots")
    return out


def mixed_step(q, k, v, cu_seqlens, prefill_slots, max_seqlen: int, decode_slots, state_pool, out=None,
               out_dtype=torch.bfloat16, workspace=None, prefill_stream=None, decode_stream=None):
    """la_mixed_step on one packed batch: rows [0, T_p) are prefill chunks
    (cu_seqlens, prefill_slots), the last n_decode rows one decode token each
    (decode_slots).  Prefill runs on prefill_stream, decode on decode_stream;
    prefill_stream then waits for the decode."""
    if q.dim() != 3:
        raise ValueError("q must be [T, H, d]")
    T, H, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _need(t, name, torch.bfloat16, (T, H, d))
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    n_prefill = cu_seqlens.numel() - 1
    _need(prefill_slots, "prefill_slots", torch.int32, (n_prefill,))
    _need(decode_slots, "decode_slots", torch.int32)
    n_decode = decode_slots.numel()
    T_p = T - n_decode
    if T_p < 0:
        raise ValueError("fewer rows than decode tokens")
    n_slots = _need_pool(state_pool, H, d)
    if out is None:
        out = torch.empty((T, H, d), dtype=out_dtype, device=q.device)
    _need(out, "out", out.dtype, (T, H, d))
    ws_bytes = varlen_workspace_size(max(n_prefill, 1), T_p, max_seqlen, H, d)
    if workspace is None:
        workspace = _alloc_workspace(ws_bytes, q.device)
    if prefill_stream is None:
        prefill_stream = torch.cuda.current_stream()
    if decode_stream is None:
        decode_stream = prefill_stream
    st = lib().la_mixed_step(_ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens), _ptr(prefill_slots), n_prefill, T_p,
                             int(max_seqlen), _ptr(decode_slots), n_decode, H, d, _ptr(state_pool), n_slots,
                             _ptr(out), _out_code(out.dtype), _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream_handle(prefill_stream),
                             _stream_handle(decode_stream))
    _check(st, "la_mixed_step")
    return out


def kv_aggregate(k, v, out=None, workspace=None, stream=None):
    """la_kv_aggregate on [B, N, H, d] bf16 k, v: returns fp32 [B, H, d, d]
    with A[b, h] = sum over the N tokens of k_t^T v_t."""
    if k.dim() != 4:
        raise ValueError("k must be [B, N, H, d]")
    B, N, H, d = k.shape
    _need(k, "k", torch.bfloat16, (B, N, H, d))
    _need(v, "v", torch.bfloat16, (B, N, H, d))
    if out is None:
        out = torch.empty((B, H, d, d), dtype=torch.float32, device=k.device)
    _need(out, "out", torch.float32, (B, H, d, d))
    ws_bytes = int(lib().la_kv_aggregate_workspace_size(B, N, H, d))
    if workspace is None:
        workspace = _alloc_workspace(ws_bytes, k.device)
    st = lib().la_kv_aggregate(_ptr(k), _ptr(v), B, N, H, d, _ptr(out), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _check(st, "la_kv_aggregate")
    return out


def state_prefix(parts, count: int, state_in=None, out=None, stream=None):
    """la_state_prefix: (state_in or 0) + parts[0] + ... + parts[count-1].
    parts: fp32 [W, ...states..., d, d] with W >= count, or None when count is
    0 (then the call copies state_in into out, or zeroes out).  Returns fp32
    states of the shape of one part (or of state_in / out)."""
    if parts is not None:
        if parts.dim() < 3:
            raise ValueError("parts must be [W, ..., d, d]")
        shape = tuple(parts.shape[1:])
        _need(parts, "parts", torch.float32, (parts.shape[0],) + shape)
        if not 0 <= count <= parts.shape[0]:
            raise ValueError("count must lie in [0, W]")
        device = parts.device
    else:
        if count != 0:
            raise ValueError("count must be 0 without parts")
        ref = state_in if state_in is not None else out
        if ref is None:
            raise ValueError("need parts, state_in or out to know the shape")
        shape = tuple(ref.shape)
        device = ref.device
    if len(shape) < 2 or shape[-1] != shape[-2]:
        raise ValueError("states must be square")
    d = shape[-1]
    nstates = 1
    for x in shape[:-2]:
        nstates *= int(x)
    if state_in is not None:
        _need(state_in, "state_in", torch.float32, shape)
    if out is None:
        out = torch.empty(shape, dtype=torch.float32, device=device)
    _need(out, "out", torch.float32, shape)
    st = lib().la_state_prefix(_ptr(parts) if count > 0 else None, int(count), _ptr(state_in), _ptr(out),
                               nstates, d, _stream_handle(stream))
    _check(st, "la_state_prefix")
    return out


def backward_workspace_size(B: int, N: int, H: int, d: int = D) -> int:
    return int(lib().la_prefill_backward_workspace_size(B, N, H, d))


def prefill_backward(q, k, v, dout, state_in=None, dstate_out=None, grad_dtype=torch.bfloat16,
                     want_dstate_in: bool = True, dq=None, dk=None, dv=None, workspace=None, stream=None):
    """la_prefill_backward on [B, N, H, d] bf16 tensors: gradients of
    la_prefill for dL/dout and dL/dstate_out.  Returns (dq, dk, dv,
    dstate_in or None)."""
    if q.dim() != 4:
        raise ValueError("q must be [B, N, H, d]")
    B, N, H, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("dout", dout)):
        _need(t, name, torch.bfloat16, (B, N, H, d))
    for name, t in (("state_in", state_in), ("dstate_out", dstate_out)):
        if t is not None:
            _need(t, name, torch.float32, (B, H, d, d))
    grads = []
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        if t is None:
            t = torch.empty((B, N, H, d), dtype=grad_dtype, device=q.device)
        _need(t, name, t.dtype, (B, N, H, d))
        grads.append(t)
    if len({t.dtype for t in grads}) != 1:
        raise TypeError("dq, dk and dv must share one dtype")
    dsin = torch.empty((B, H, d, d), dtype=torch.float32, device=q.device) if want_dstate_in else None
    ws_bytes = backward_workspace_size(B, N, H, d)
    if workspace is None:
        workspace = _alloc_workspace(ws_bytes, q.device)
    st = lib().la_prefill_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), B, N, H, d, _ptr(state_in),
                                   _ptr(dstate_out), _ptr(grads[0]), _ptr(grads[1]), _ptr(grads[2]),
                                   _out_code(grads[0].dtype), _ptr(dsin), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream_handle(stream))
    _check(st, "la_prefill_backward")
    return grads[0], grads[1], grads[2], dsin


def backward_varlen_workspace_size(nseq: int, total_tokens: int, max_seqlen: int, H: int, d: int = D) -> int:
    return int(lib().la_prefill_backward_varlen_workspace_size(nseq, total_tokens, max_seqlen, H, d))


def prefill_backward_varlen(q, k, v, dout, cu_seqlens, max_seqlen: int, state_in=None, dstate_out=None,
                            grad_dtype=torch.bfloat16, want_dstate_in: bool = True, dq=None, dk=None, dv=None,
                            workspace=None, stream=None):
    """la_prefill_backward_varlen on packed [T, H, d] bf16 tensors with device
    int32 cu_seqlens: gradients of la_prefill_varlen for dL/dout and
    dL/dstate_out.  Returns (dq, dk, dv, dstate_in or None)."""
    if q.dim() != 3:
        raise ValueError("q must be [T, H, d]")
    T, H, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v), ("dout", dout)):
        _need(t, name, torch.bfloat16, (T, H, d))
    _need(cu_seqlens, "cu_seqlens", torch.int32)
    nseq = cu_seqlens.numel() - 1
    if nseq < 0:
        raise ValueError("cu_seqlens must hold nseq + 1 entries")
    for name, t in (("state_in", state_in), ("dstate_out", dstate_out)):
        if t is not None:
            _need(t, name, torch.float32, (nseq, H, d, d))
    grads = []
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        if t is None:
            t = torch.empty((T, H, d), dtype=grad_dtype, device=q.device)
        _need(t, name, t.dtype, (T, H, d))
        grads.append(t)
    if len({t.dtype for t in grads}) != 1:
        raise TypeError("dq, dk and dv must share one dtype")
    dsin = torch.empty((nseq, H, d, d), dtype=torch.float32, device=q.device) if want_dstate_in else None
    ws_bytes = backward_varlen_workspace_size(nseq, T, max_seqlen, H, d)
    if workspace is None:
        workspace = _alloc_workspace(ws_bytes, q.device)
    st = lib().la_prefill_backward_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(cu_seqlens), nseq, T,
                                          int(max_seqlen), H, d, _ptr(state_in), _ptr(dstate_out), _ptr(grads[0]),
                                          _ptr(grads[1]), _ptr(grads[2]), _out_code(grads[0].dtype), _ptr(dsin),
                                          _ptr(workspace), workspace.numel() * workspace.element_size(),
                                          _stream_handle(stream))
    _check(st, "la_prefill_backward_varlen")
    return grads[0], grads[1], grads[2], dsin


def get_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the sticky device status."""
    return int(lib().la_get_device_status(_stream_handle(stream)))


def set_wait_limit_ns(ns: int):
    _check(lib().la_set_wait_limit_ns(int(ns)), "la_set_wait_limit_ns")


def set_segment_len(tokens: int):
    _check(lib().la_set_segment_len(int(tokens)), "la_set_segment_len")


def debug_inject(mode: int):
    _check(lib().la_debug_inject(int(mode)), "la_debug_inject")


def last_segment_len() -> int:
    return int(lib().la_last_segment_len())


def kernel_launches() -> int:
    return int(lib().la_kernel_launches())
