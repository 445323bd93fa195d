"""Sequence parallelism across ranks for the prefill (LASP+).

"MiniMax-01技术报告解读", §3.2 item 3 (LASP+): every rank holds a contiguous
part of the sequence; it forms the local prefix of its part (the sum of
k_t^T v_t over its tokens), the local prefixes are all-gathered, each rank adds
up those of the ranks before it (the global prefix) and then runs its own
blocked scan starting from that state.  One process per GPU; the exchange is
one AllGather of a d x d fp32 matrix per (sequence, head) -- 4 MiB per rank at
64 heads -- over the process group (NCCL over NVLink between GPUs).

Rank r of `group` holds tokens [n_0 + ... + n_{r-1}, + n_r) of every sequence
of the batch as [B, n_r, H, 128] tensors; the parts may differ in length.  The
rank's output equals the rows of the single-GPU prefill of the whole sequences
for its tokens, and every rank returns the final state of the whole sequences.

The device steps run in the CUDA library (la_kv_aggregate, la_state_prefix,
la_prefill); the collective is torch.distributed's.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

from . import _binding


class DeviceOps:
    """The three device steps of one rank, as this library's CUDA entry points."""

    @staticmethod
    def kv_aggregate(k, v):
        return _binding.kv_aggregate(k, v)

    @staticmethod
    def state_prefix(parts, count, state_in):
        return _binding.state_prefix(parts, count, state_in)

    @staticmethod
    def prefill(q, k, v, state_in, out_dtype):
        out, _ = _binding.prefill(q, k, v, state_in=state_in, out_dtype=out_dtype, want_state=False)
        return out


def lasp_prefill(q, k, v, group=None, state_in=None, out_dtype=torch.bfloat16, want_state: bool = True,
                 ops=DeviceOps):
    """Prefill of this rank's part [B, n_r, H, d] of every sequence.

    state_in: fp32 [B, H, d, d] state before the first rank's tokens (the same
    on every rank), or None for zero.  Returns (out [B, n_r, H, d], final state
    [B, H, d, d] of the whole sequences, or None when want_state is False).
    `ops` supplies the device steps; the default is the CUDA library (a test
    may pass host implementations to check the exchange on CPU ranks).
    """
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if q.dim() != 4:
        raise ValueError("q must be [B, n_r, H, d]")
    B, _, H, d = q.shape
    local = ops.kv_aggregate(k, v)  # A_r = sum over this rank's tokens of k_t^T v_t
    if tuple(local.shape) != (B, H, d, d):
        raise ValueError("local prefix has the wrong shape")
    gathered = local.new_empty((world * B, H, d, d))  # rank-major, the layout every backend accepts
    dist.all_gather_into_tensor(gathered, local.contiguous(), group=group)
    parts = gathered.view(world, B, H, d, d)
    prefix = ops.state_prefix(parts, rank, state_in)  # S_in + A_0 + ... + A_{r-1}
    out = ops.prefill(q, k, v, prefix, out_dtype)
    final = ops.state_prefix(parts, world, state_in) if want_state else None
    return out, final
