"""Host-side helpers for running the hot path on several GPUs of one node.

The operation splits into independent (sequence, head) problems, so N GPUs
run N independent shares of a batch with no collective on the data path
(data parallelism; one process per GPU).  What needs coordinating is only on
the host:

  * shard_packed:   split a packed batch (cu_seqlens) into contiguous groups of
                    whole sequences with balanced token counts, one per rank;
  * local_problem:  the token range and rebased cu_seqlens of one rank's share;
  * max_over_ranks: the max of a per-rank timing (the job is as slow as its
                    slowest rank), over whatever process group is initialised
                    (nccl on GPUs, gloo on CPUs).
"""
from __future__ import annotations

import numpy as np


def shard_packed(lengths, world: int):
    """Split sequences 0..n-1 (in order) into `world` contiguous groups whose
    token totals are as even as a greedy prefix split makes them.  Returns a
    list of (first_seq, end_seq) half-open ranges, one per rank; a rank may
    get an empty range when there are fewer sequences than ranks."""
    lengths = np.asarray(lengths, dtype=np.int64)
    if world <= 0:
        raise ValueError("world must be positive")
    n = lengths.size
    total = int(lengths.sum())
    bounds = [0]
    csum = np.concatenate([[0], np.cumsum(lengths)])
    for r in range(1, world):
        target = total * r / world
        # first sequence boundary at or past the target, never going backwards
        i = int(np.searchsorted(csum, target, side="left"))
        i = min(max(i, bounds[-1]), n)
        # take the nearer of the two boundaries around the target
        if i > bounds[-1] and abs(csum[i - 1] - target) < abs(csum[i] - target):
            i -= 1
        bounds.append(i)
    bounds.append(n)
    return [(bounds[r], bounds[r + 1]) for r in range(world)]


def local_problem(cu_seqlens, group):
    """(token_start, token_end, local cu_seqlens) of the sequences in `group`."""
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    a, b = group
    t0, t1 = int(cu[a]), int(cu[b])
    return t0, t1, (cu[a:b + 1] - t0).astype(np.int32)


def max_over_ranks(value: float, device=None) -> float:
    """Max of `value` over the default process group (identity when there is
    no initialised group or it has one rank)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    if device is None:
        device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
