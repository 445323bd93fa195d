"""Host planning of a mixed prefill/decode batch (no GPU)."""
import numpy as np
import pytest

from linear_attention_blocked_b200.serving import plan_batch


def test_routing_order_and_offsets():
    lengths = [300, 1, 0, 777, 1, 1, 64, 2]
    slots = [5, 2, 9, 0, 7, 3, 1, 6]
    p = plan_batch(lengths, slots)
    # length-1 requests go to the decode kernel, longer ones are packed as prefill chunks
    assert list(p.decode_ids) == [1, 4, 5]
    assert list(p.prefill_ids) == [0, 3, 6, 7]
    assert list(p.cu_seqlens) == [0, 300, 1077, 1141, 1143]
    assert p.prefill_tokens == 1143 and p.total_rows == 1146 and p.max_seqlen == 777
    assert list(p.prefill_slots) == [5, 0, 1, 6] and list(p.decode_slots) == [2, 7, 3]
    # every active request's rows are where the plan says; inactive ones take none
    assert p.row_offset[2] == -1
    rows = np.zeros(p.total_rows, dtype=int)
    for i, n in enumerate(lengths):
        if n:
            rows[p.row_offset[i]:p.row_offset[i] + n] += 1
    assert (rows == 1).all()
    assert p.cu_seqlens.dtype == np.int32 and p.decode_slots.dtype == np.int32


def test_degenerate_batches():
    p = plan_batch([1, 1], [0, 1])
    assert p.prefill_tokens == 0 and list(p.cu_seqlens) == [0] and p.max_seqlen == 0
    p = plan_batch([5], [3])
    assert len(p.decode_ids) == 0 and p.total_rows == 5
    p = plan_batch([], [])
    assert p.total_rows == 0


def test_rejects_shared_slots_and_bad_lengths():
    with pytest.raises(ValueError):
        plan_batch([3, 1], [2, 2])
    plan_batch([3, 0], [2, 2])  # an idle request may share a slot
    with pytest.raises(ValueError):
        plan_batch([-1], [0])
    with pytest.raises(ValueError):
        plan_batch([1, 2], [0])
