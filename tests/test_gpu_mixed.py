"""GPU parity of the state-pool entry points and the mixed prefill/decode step
against the fp64 oracle: every request continues from its own slot of a pool
of running states; prefill chunks and decode tokens of one batch run on two
streams."""
import numpy as np
import pytest
import torch

import la_inputs
import linear_attention_blocked_b200 as la
from parity_util import check_out, check_state, to_np

pytestmark = pytest.mark.gpu

D = 128
H = 4
N_SLOTS = 10


def _pool(seed):
    gen = torch.Generator(device="cuda").manual_seed(seed)
    return torch.randn((N_SLOTS, H, D, D), generator=gen, device="cuda") * 0.2


def _reference(oracle_mod, q, k, v, plan, pool0):
    """The whole packed batch as a varlen batch in row order (each decode token a
    length-1 sequence), each sequence starting from its slot's state."""
    nd = len(plan.decode_ids)
    cu = np.concatenate([plan.cu_seqlens, plan.prefill_tokens + 1 + np.arange(nd)]).astype(np.int32)
    slots = np.concatenate([plan.prefill_slots, plan.decode_slots]).astype(np.int64)
    sin = to_np(pool0)[slots]
    out, st = oracle_mod.recurrent(la_inputs.bits(q), la_inputs.bits(k), la_inputs.bits(v), cu, state_in=sin)
    return out, st, slots


@pytest.mark.parametrize("two_streams", [False, True])
def test_mixed_step_matches_oracle(oracle_mod, two_streams):
    lengths = [300, 1, 0, 777, 1, 1, 64, 2, 129]
    slots = [5, 2, 9, 0, 7, 3, 1, 6, 8]
    plan = la.plan_batch(lengths, slots)
    q, k, v = la_inputs.qkv((plan.total_rows, H, D), seed=71, device="cuda")
    pool0 = _pool(72)
    pool = pool0.clone()
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    s_pre = torch.cuda.current_stream()
    s_dec = torch.cuda.Stream() if two_streams else s_pre
    out = la.mixed_step(q, k, v, dev(plan.cu_seqlens), dev(plan.prefill_slots), plan.max_seqlen,
                        dev(plan.decode_slots), pool, out_dtype=torch.float32,
                        prefill_stream=s_pre, decode_stream=s_dec)
    assert la.get_device_status(s_pre) == la.LA_OK
    ref, rst, used = _reference(oracle_mod, q, k, v, plan, pool0)
    check_out(to_np(out), ref, bf16_out=False, what="mixed batch outputs")
    check_state(to_np(pool)[used], rst, what="slot states after the step")
    untouched = sorted(set(range(N_SLOTS)) - set(used.tolist()))
    assert torch.equal(pool[untouched], pool0[untouched])  # slot 4 (idle request) and unnamed slots


def test_decode_then_prefill_on_slots_equals_one_sequence(oracle_mod):
    """prefill chunk -> decode token -> prefill chunk on one slot equals the
    recurrent scan over the concatenated tokens."""
    q, k, v = la_inputs.qkv((400, H, D), seed=73, device="cuda")
    pool0 = _pool(74)
    pool = pool0.clone()
    slot = torch.tensor([3], dtype=torch.int32, device="cuda")
    parts = [(0, 250), (250, 251), (251, 400)]
    outs = []
    for a, b in parts:
        if b - a == 1:
            outs.append(la.decode_step_slots(q[a:b], k[a:b], v[a:b], pool, slot, out_dtype=torch.float32))
        else:
            cu = torch.tensor([0, b - a], dtype=torch.int32, device="cuda")
            outs.append(la.prefill_varlen_slots(q[a:b].contiguous(), k[a:b].contiguous(), v[a:b].contiguous(),
                                                cu, slot, b - a, pool, out_dtype=torch.float32))
    assert la.get_device_status() == la.LA_OK
    ref, rst = oracle_mod.recurrent(la_inputs.bits(q), la_inputs.bits(k), la_inputs.bits(v),
                                    np.array([0, 400], np.int32), state_in=to_np(pool0)[[3]])
    check_out(to_np(torch.cat(outs, 0)), ref, bf16_out=False, what="chunked through one slot")
    check_state(to_np(pool[[3]]), rst, what="slot 3")
    others = [i for i in range(N_SLOTS) if i != 3]
    assert torch.equal(pool[others], pool0[others])


def test_slot_out_of_range_is_reported_and_skipped():
    q, k, v = la_inputs.qkv((2, H, D), seed=75, device="cuda")
    pool0 = _pool(76)
    pool = pool0.clone()
    slots = torch.tensor([1, N_SLOTS], dtype=torch.int32, device="cuda")   # the second is out of range
    la.decode_step_slots(q, k, v, pool, slots)
    assert la.get_device_status() == la.LA_ERR_INVALID_ARGUMENT
    assert not torch.equal(pool[1], pool0[1])                               # row 0 ran
    assert torch.equal(pool[2:], pool0[2:])
    cu = torch.tensor([0, 2], dtype=torch.int32, device="cuda")
    la.prefill_varlen_slots(q, k, v, cu, torch.tensor([-1], dtype=torch.int32, device="cuda"), 2, pool)
    assert la.get_device_status() == la.LA_ERR_INVALID_ARGUMENT
    assert la.get_device_status() == la.LA_OK                                # the word is cleared
