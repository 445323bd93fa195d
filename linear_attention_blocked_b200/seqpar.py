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

Packed variable-length batches (lasp_prefill_varlen): the packed token axis
is cut into contiguous rank ranges at arbitrary points, so a sequence may
start on one rank and end several ranks later.  Each rank forms the local
prefix of the one sequence that is still open at the end of its range, the
local prefixes are all-gathered, and the sequence carried into the rank's
range starts from its carried-in state plus the local prefixes of the ranks
it spanned before; every other sequence of the range starts from its own
carried-in state.  The planning is plain host arithmetic on cu_seqlens
(plan_varlen_rank); the device steps are la_kv_aggregate, la_state_prefix
and la_prefill_varlen.

Gradients across ranks (lasp_prefill_backward): a rank's tokens see the
earlier ranks only through the state they hand on and the later ranks only
through that state's gradient, so each rank gathers two d x d sums per
(sequence, head) from every rank and runs la_prefill_backward on its own
tokens from the two.  For packed batches (lasp_prefill_backward_varlen)
only the sequence carried into a rank's range and the one still open at its
end cross rank boundaries, so each rank contributes the forward sum of its
open tail and the state-gradient sum of its carried-in head, and runs
la_prefill_backward_varlen on its own tokens.

The device steps run in the CUDA library (la_kv_aggregate, la_state_prefix,
la_prefill, la_prefill_varlen, la_prefill_backward); the collective is
torch.distributed's.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch
import torch.distributed as dist

from . import _binding


class DeviceOps:
    """The device steps of one rank, as this library's CUDA entry points."""

    @staticmethod
    def kv_aggregate(k, v):
        return _binding.kv_aggregate(k, v)

    @staticmethod
    def state_prefix(parts, count, state_in, out=None):
        return _binding.state_prefix(parts, count, state_in, out=out)

    @staticmethod
    def prefill(q, k, v, state_in, out_dtype):
        out, _ = _binding.prefill(q, k, v, state_in=state_in, out_dtype=out_dtype, want_state=False)
        return out

    @staticmethod
    def prefill_backward(q, k, v, dout, state_in, dstate_out, grad_dtype):
        return _binding.prefill_backward(q, k, v, dout, state_in=state_in, dstate_out=dstate_out,
                                         grad_dtype=grad_dtype, want_dstate_in=False)[:3]

    @staticmethod
    def prefill_varlen(q, k, v, cu_seqlens, max_seqlen, state_in, out_dtype):
        cu = torch.from_numpy(np.ascontiguousarray(cu_seqlens, dtype=np.int32)).to(q.device)
        return _binding.prefill_varlen(q, k, v, cu, max_seqlen, state_in=state_in, out_dtype=out_dtype)

    @staticmethod
    def prefill_backward_varlen(q, k, v, dout, cu_seqlens, max_seqlen, state_in, dstate_out, grad_dtype):
        cu = torch.from_numpy(np.ascontiguousarray(cu_seqlens, dtype=np.int32)).to(q.device)
        return _binding.prefill_backward_varlen(q, k, v, dout, cu, max_seqlen, state_in=state_in,
                                                dstate_out=dstate_out, grad_dtype=grad_dtype)


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


# --------------------------------------------------------------------------- gradients
def backward_local_sums(q, k, v, dout, ops=DeviceOps):
    """Step 1 of lasp_prefill_backward on one rank (step 2 gathers the
    results of every rank): the rank's sums
    A_r = sum k_t^T v_t (for the forward prefix of later ranks) and
    B_r = sum q_t^T g_t (for the state gradient of earlier ranks)."""
    return ops.kv_aggregate(k, v), ops.kv_aggregate(q, dout)


def backward_local_grads(rank, world, a_parts, b_parts, q, k, v, dout, state_in=None, dstate_out=None,
                         grad_dtype=torch.bfloat16, ops=DeviceOps):
    """Step 3 on one rank, given every rank's sums (a_parts, b_parts: [W, B,
    H, d, d], rank order).  The rank's tokens see the earlier ranks only
    through their state, S_in + A_0 + ... + A_{r-1}, and the later ranks only
    through the gradient of the state they hand on, G + B_{r+1} + ... +
    B_{W-1}; so its gradients are la_prefill_backward of its own tokens with
    those two.  Returns (dq, dk, dv, dS_in of the whole sequences)."""
    prefix = ops.state_prefix(a_parts[:rank], rank, state_in)
    later = b_parts[rank + 1:]
    suffix = ops.state_prefix(later, world - rank - 1, dstate_out)
    dq, dk, dv = ops.prefill_backward(q, k, v, dout, prefix, suffix, grad_dtype)
    dstate_in = ops.state_prefix(b_parts, world, dstate_out)  # sum over all tokens of q^T g, + G
    return dq, dk, dv, dstate_in


def lasp_prefill_backward(q, k, v, dout, group=None, state_in=None, dstate_out=None, grad_dtype=torch.bfloat16,
                          ops=DeviceOps):
    """Gradients of lasp_prefill on this rank's part [B, n_r, H, d] of every
    sequence, for dL/dout (this rank's rows) and dL/dS_out of the final
    state of the whole sequences (dstate_out, the same on every rank, or
    None).  Returns (dq, dk, dv for this rank's tokens, dS_in of the whole
    sequences, the same on every rank).  Two AllGathers, one for each of the
    rank's two d x d sums per (sequence, head); step 2 between
    backward_local_sums and backward_local_grads."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if q.dim() != 4:
        raise ValueError("q must be [B, n_r, H, d]")
    B, _, H, d = q.shape
    a, b = backward_local_sums(q, k, v, dout, ops)
    parts = []
    for local in (a, b):
        gathered = local.new_empty((world * B, H, d, d))  # rank-major
        dist.all_gather_into_tensor(gathered, local.contiguous(), group=group)
        parts.append(gathered.view(world, B, H, d, d))
    return backward_local_grads(rank, world, parts[0], parts[1], q, k, v, dout, state_in, dstate_out, grad_dtype,
                                ops)


# --------------------------------------------------------------------------- packed batches
def split_tokens(total_tokens: int, world: int) -> np.ndarray:
    """Rank boundaries [world + 1] cutting the packed token axis into ranges
    whose lengths differ by at most one token."""
    return (np.arange(world + 1, dtype=np.int64) * int(total_tokens)) // int(world)


@dataclass
class VarlenRankPlan:
    rank: int
    tok0: int                 # this rank holds packed tokens [tok0, tok1)
    tok1: int
    seq0: int                 # its local sequences are global sequences seq0 .. seq1-1
    seq1: int
    local_cu: np.ndarray      # int32 [seq1 - seq0 + 1], offsets into the rank's tokens
    max_seqlen: int
    carried_from: int         # rank where local sequence 0 began (== rank: not carried in)
    open_tail: tuple | None   # (a, b): the rank's tokens of the sequence continuing past tok1
    ends_here: np.ndarray     # bool [seq1 - seq0]: that sequence's final state is formed here

    @property
    def n_local(self) -> int:
        return self.seq1 - self.seq0

    @property
    def starts_here(self) -> np.ndarray:
        """bool [seq1 - seq0]: that sequence's first token is on this rank (so
        its state gradient dS_in is formed here)."""
        first = np.ones(self.n_local, bool)
        if self.n_local:
            first[0] = self.carried_from == self.rank
        return first


def plan_varlen_rank(cu_seqlens, bounds, rank: int) -> VarlenRankPlan:
    """Which sequences rank `rank` sees, and how they continue across ranks.

    cu_seqlens: int [nseq + 1] of the whole packed batch; bounds: int
    [world + 1], non-decreasing from 0 to the total token count.  A non-empty
    sequence belongs to every rank whose range it overlaps; an empty sequence
    at position p belongs to the first rank with p < tok1 (the last rank when
    p is the end of the batch), which also reports its final state (= its
    carried-in state).
    """
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    bd = np.asarray(bounds, dtype=np.int64)
    world = len(bd) - 1
    if cu.ndim != 1 or len(cu) < 1 or cu[0] != 0 or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must start at 0 and not decrease")
    if world < 1 or bd[0] != 0 or bd[-1] != cu[-1] or np.any(np.diff(bd) < 0):
        raise ValueError("bounds must run from 0 to the token count without decreasing")
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    tok0, tok1 = int(bd[rank]), int(bd[rank + 1])
    starts, ends = cu[:-1], cu[1:]
    nonempty = ends > starts
    overlap = np.maximum(starts, tok0) < np.minimum(ends, tok1)  # shares at least one token
    # owner rank of each empty sequence: first rank whose range ends after p
    owner = np.searchsorted(bd[1:], starts, side="right")
    owner = np.minimum(owner, world - 1)
    mine = overlap | (~nonempty & (owner == rank))
    idx = np.nonzero(mine)[0]
    if len(idx) == 0:
        seq0 = seq1 = int(np.searchsorted(starts, tok0, side="left"))
        return VarlenRankPlan(rank, tok0, tok1, seq0, seq1, np.zeros(1, np.int32), 0, rank, None,
                              np.zeros(0, bool))
    seq0, seq1 = int(idx[0]), int(idx[-1]) + 1
    if len(idx) != seq1 - seq0:
        raise AssertionError("local sequences are not contiguous")
    local_cu = (np.clip(cu[seq0:seq1 + 1], tok0, tok1) - tok0).astype(np.int32)
    lens = np.diff(local_cu)
    carried_from = rank
    if cu[seq0] < tok0:  # the first sequence began on an earlier rank
        carried_from = int(np.searchsorted(bd[1:], cu[seq0], side="right"))
    open_tail = None
    if cu[seq1] > tok1:  # the last sequence continues on a later rank
        open_tail = (int(local_cu[-2]), int(local_cu[-1]))
    ends_here = cu[seq0 + 1:seq1 + 1] <= tok1
    if open_tail is not None:
        ends_here[-1] = False
    return VarlenRankPlan(rank, tok0, tok1, seq0, seq1, local_cu, int(lens.max()) if len(lens) else 0,
                          carried_from, open_tail, ends_here.astype(bool))


def varlen_local_prefix(plan: VarlenRankPlan, k, v, ops=DeviceOps):
    """Step 1 on one rank: the local prefix [H, d, d] of the sequence still
    open at the end of its range (zero when every sequence ends there)."""
    _, H, d = k.shape
    a, b = plan.open_tail if plan.open_tail is not None else (0, 0)
    return ops.kv_aggregate(k[a:b].reshape(1, b - a, H, d), v[a:b].reshape(1, b - a, H, d))[0]


def varlen_local_scan(plan: VarlenRankPlan, q, k, v, parts, state_in=None, out_dtype=torch.bfloat16,
                      ops=DeviceOps):
    """Step 3 on one rank, given every rank's local prefix (parts [W, H, d,
    d], rank order): the carried-in states of the rank's sequences, then its
    local scan.  Returns (out [tokens, H, d], local final states)."""
    _, H, d = q.shape
    if plan.n_local == 0:
        return q.new_empty((0, H, d), dtype=out_dtype), parts.new_empty((0, H, d, d))
    sin = parts.new_empty((plan.n_local, H, d, d))
    s0 = None if state_in is None else state_in[plan.seq0]
    cf, r = plan.carried_from, plan.rank
    if cf < r:  # global prefix of the sequence carried into this range
        ops.state_prefix(parts[cf:r], r - cf, s0, sin[0])
    else:
        ops.state_prefix(None, 0, s0, sin[0])
    if plan.n_local > 1:
        rest = None if state_in is None else state_in[plan.seq0 + 1:plan.seq1]
        ops.state_prefix(None, 0, rest, sin[1:])
    return ops.prefill_varlen(q, k, v, plan.local_cu, plan.max_seqlen, sin, out_dtype)


def lasp_prefill_varlen(q, k, v, cu_seqlens, bounds, group=None, state_in=None, out_dtype=torch.bfloat16,
                        ops=DeviceOps):
    """Prefill of this rank's range [bounds[r], bounds[r+1]) of a packed batch.

    q, k, v: [bounds[r+1] - bounds[r], H, d] bf16 (this rank's tokens);
    cu_seqlens, bounds: host int arrays of the whole batch (the same on every
    rank); state_in: fp32 [nseq, H, d, d] carried-in states of all sequences
    (the same on every rank), or None for zero.  Returns (out [tokens, H, d],
    local final states [seq1 - seq0, H, d, d], plan): row i of the states is
    the final state of global sequence plan.seq0 + i where plan.ends_here[i]
    (the other rows, at most the last one, are only this rank's part).
    """
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if len(bounds) != world + 1:
        raise ValueError("bounds must hold world + 1 entries")
    plan = plan_varlen_rank(cu_seqlens, bounds, rank)
    if q.dim() != 3 or q.shape[0] != plan.tok1 - plan.tok0:
        raise ValueError("q must be [this rank's tokens, H, d]")
    _, H, d = q.shape
    local = varlen_local_prefix(plan, k, v, ops)
    gathered = local.new_empty((world * H, d, d))  # rank-major
    dist.all_gather_into_tensor(gathered, local.contiguous(), group=group)
    out, st = varlen_local_scan(plan, q, k, v, gathered.view(world, H, d, d), state_in, out_dtype, ops)
    return out, st, plan


def varlen_backward_local_sums(plan: VarlenRankPlan, q, k, v, dout, ops=DeviceOps):
    """Step 1 of lasp_prefill_backward_varlen on one rank: A_r = sum of
    k_t^T v_t over the sequence still open at the end of its range (the
    forward prefix later ranks need) and B_r = sum of q_t^T g_t over the
    sequence carried into its range (the state gradient earlier ranks need);
    zero where there is no such sequence.  Both [H, d, d]."""
    _, H, d = q.shape
    if plan.open_tail is not None:
        a, b = plan.open_tail
        A = ops.kv_aggregate(k[a:b].reshape(1, b - a, H, d), v[a:b].reshape(1, b - a, H, d))[0]
    else:
        A = ops.kv_aggregate(k[0:0].reshape(1, 0, H, d), v[0:0].reshape(1, 0, H, d))[0]
    n0 = int(plan.local_cu[1]) if plan.n_local and plan.carried_from < plan.rank else 0
    B = ops.kv_aggregate(q[0:n0].reshape(1, n0, H, d), dout[0:n0].reshape(1, n0, H, d))[0]
    return A, B


def varlen_backward_local_grads(plan: VarlenRankPlan, cu_seqlens, bounds, q, k, v, dout, a_parts, b_parts,
                                state_in=None, dstate_out=None, grad_dtype=torch.bfloat16, ops=DeviceOps):
    """Step 3 on one rank, given every rank's two sums (a_parts, b_parts:
    [W, H, d, d], rank order).  The sequence carried into the range starts
    from its carried-in state plus the A of the ranks it spanned before; the
    sequence still open at the end of the range ends with its state gradient
    plus the B of the ranks it spans after; every other sequence is local.
    Returns (dq, dk, dv for the rank's tokens, dS_in [seq1 - seq0, H, d, d]):
    row i is the whole dS_in of global sequence plan.seq0 + i where
    plan.starts_here[i]."""
    _, H, d = q.shape
    if plan.n_local == 0:
        e = q.new_empty((q.shape[0], H, d), dtype=grad_dtype)
        return e, e.clone(), e.clone(), a_parts.new_empty((0, H, d, d))
    r, cf = plan.rank, plan.carried_from
    sin = a_parts.new_empty((plan.n_local, H, d, d))
    s0 = None if state_in is None else state_in[plan.seq0]
    ops.state_prefix(a_parts[cf:r] if cf < r else None, r - cf, s0, sin[0])
    if plan.n_local > 1:
        rest = None if state_in is None else state_in[plan.seq0 + 1:plan.seq1]
        ops.state_prefix(None, 0, rest, sin[1:])
    gout = a_parts.new_empty((plan.n_local, H, d, d))
    last = plan.seq1 - 1
    head = None if dstate_out is None else dstate_out[plan.seq0:last]
    if plan.n_local > 1:
        ops.state_prefix(None, 0, head, gout[:-1])
    g_last = None if dstate_out is None else dstate_out[last]
    if plan.open_tail is not None:
        # the ranks after this one up to the one holding the sequence's last token
        bd = np.asarray(bounds, dtype=np.int64)
        end = int(np.searchsorted(bd[1:], int(np.asarray(cu_seqlens)[last + 1]), side="left"))
        ops.state_prefix(b_parts[r + 1:end + 1], end - r, g_last, gout[-1])
    else:
        ops.state_prefix(None, 0, g_last, gout[-1])
    return ops.prefill_backward_varlen(q, k, v, dout, plan.local_cu, plan.max_seqlen, sin, gout, grad_dtype)


def lasp_prefill_backward_varlen(q, k, v, dout, cu_seqlens, bounds, group=None, state_in=None, dstate_out=None,
                                 grad_dtype=torch.bfloat16, ops=DeviceOps):
    """Gradients of lasp_prefill_varlen on this rank's range [bounds[r],
    bounds[r+1]) of a packed batch, for dL/dout (this rank's rows) and
    dL/dS_out of every sequence's final state (dstate_out, fp32 [nseq, H, d,
    d], the same on every rank, or None).  Returns (dq, dk, dv [tokens, H,
    d], dS_in [seq1 - seq0, H, d, d], plan): row i of dS_in is the whole
    dS_in of global sequence plan.seq0 + i where plan.starts_here[i].  Two
    AllGathers of one d x d matrix per head."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    if len(bounds) != world + 1:
        raise ValueError("bounds must hold world + 1 entries")
    plan = plan_varlen_rank(cu_seqlens, bounds, rank)
    if q.dim() != 3 or q.shape[0] != plan.tok1 - plan.tok0:
        raise ValueError("q must be [this rank's tokens, H, d]")
    _, H, d = q.shape
    a, b = varlen_backward_local_sums(plan, q, k, v, dout, ops)
    parts = []
    for local in (a, b):
        gathered = local.new_empty((world * H, d, d))  # rank-major
        dist.all_gather_into_tensor(gathered, local.contiguous(), group=group)
        parts.append(gathered.view(world, H, d, d))
    dq, dk, dv, dsin = varlen_backward_local_grads(plan, cu_seqlens, bounds, q, k, v, dout, parts[0], parts[1],
                                                   state_in, dstate_out, grad_dtype, ops)
    return dq, dk, dv, dsin, plan

