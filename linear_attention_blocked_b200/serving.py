"""Host-side planning of a mixed prefill/decode batch.

A serving step gathers new tokens from many requests; each request owns one
running state in a pool (its slot).  Requests with exactly one new token are
routed to the decode kernel, the others are packed as variable-length prefill
chunks ("MiniMax-01技术报告解读", §3.3 item 2: prefill and decode on separate
streams, length-1 tokens through the decode kernel).  `plan_batch` decides the
row order of the packed batch that `mixed_step` expects -- prefill chunks
first, then one row per decode token -- and builds the index arrays.  It does
no GPU work; placing each request's q, k, v rows at `row_offset` is the
caller's part.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass
class BatchPlan:
    prefill_ids: np.ndarray    # request indices packed as prefill chunks, in row order
    decode_ids: np.ndarray     # request indices served by the decode kernel, in row order
    row_offset: np.ndarray     # [n_requests] first row of each request (-1: no new tokens)
    cu_seqlens: np.ndarray     # int32 [n_prefill + 1] over the prefill rows
    prefill_slots: np.ndarray  # int32 [n_prefill]
    decode_slots: np.ndarray   # int32 [n_decode]
    prefill_tokens: int
    max_seqlen: int

    @property
    def total_rows(self) -> int:
        return self.prefill_tokens + len(self.decode_ids)


def plan_batch(lengths, slots) -> BatchPlan:
    """lengths[i]: new tokens of request i (>= 0); slots[i]: its state slot.
    Requests with no new tokens take no rows; one slot may serve one request."""
    lengths = np.asarray(lengths, dtype=np.int64)
    slots = np.asarray(slots, dtype=np.int64)
    if lengths.shape != slots.shape or lengths.ndim != 1:
        raise ValueError("lengths and slots must be 1-D and of equal length")
    if (lengths < 0).any():
        raise ValueError("negative length")
    active = lengths > 0
    if len(np.unique(slots[active])) != int(active.sum()):
        raise ValueError("two requests of one batch share a state slot")
    prefill_ids = np.nonzero(lengths > 1)[0]
    decode_ids = np.nonzero(lengths == 1)[0]
    cu = np.zeros(len(prefill_ids) + 1, dtype=np.int64)
    np.cumsum(lengths[prefill_ids], out=cu[1:])
    prefill_tokens = int(cu[-1])
    if prefill_tokens + len(decode_ids) > 0x7FFFFFFF:
        raise ValueError("batch too large")
    row_offset = np.full(len(lengths), -1, dtype=np.int64)
    row_offset[prefill_ids] = cu[:-1]
    row_offset[decode_ids] = prefill_tokens + np.arange(len(decode_ids))
    return BatchPlan(prefill_ids=prefill_ids, decode_ids=decode_ids, row_offset=row_offset,
                     cu_seqlens=cu.astype(np.int32), prefill_slots=slots[prefill_ids].astype(np.int32),
                     decode_slots=slots[decode_ids].astype(np.int32), prefill_tokens=prefill_tokens,
                     max_seqlen=int(lengths[prefill_ids].max()) if len(prefill_ids) else 0)
