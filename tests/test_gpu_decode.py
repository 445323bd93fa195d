"""GPU parity of la_decode_step (through the C ABI) against the fp64 oracle,
and the decode-after-prefill invariant."""
import numpy as np
import pytest
import torch

import la_inputs
import linear_attention_blocked_b200 as la
from parity_util import check_out, check_state, to_np

pytestmark = pytest.mark.gpu

D = 128


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_decode_steps_match_oracle(oracle_mod, out_dtype):
    B, H, steps = 5, 3, 8
    gen = torch.Generator(device="cuda").manual_seed(21)
    state = torch.randn((B, H, D, D), generator=gen, device="cuda") * 0.5
    ref_state = to_np(state)
    for s in range(steps):
        q, k, v = la_inputs.qkv((B, H, D), seed=la_inputs.decode_seed(21, s), device="cuda")
        o = la.decode_step(q, k, v, state, out_dtype=out_dtype)
        ref_o, ref_state = oracle_mod.decode_step(la_inputs.bits(q), la_inputs.bits(k),
                                                  la_inputs.bits(v), ref_state)
        check_out(to_np(o), ref_o, bf16_out=out_dtype == torch.bfloat16, what=f"step {s}")
    assert la.get_device_status() == la.LA_OK
    check_state(to_np(state), ref_state)


def test_decode_after_prefill_equals_longer_prefill(oracle_mod):
    """prefill(N) followed by m decode steps == prefill(N + m)."""
    B, N, m, H = 2, 500, 6, 2
    q, k, v = la_inputs.qkv((B, N + m, H, D), seed=22, device="cuda")
    out_full, st_full = la.prefill(q, k, v, out_dtype=torch.float32)
    _, state = la.prefill(q[:, :N].contiguous(), k[:, :N].contiguous(), v[:, :N].contiguous(),
                          out_dtype=torch.float32)
    for t in range(N, N + m):
        o = la.decode_step(q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(), state,
                           out_dtype=torch.float32)
        check_out(to_np(o), to_np(out_full[:, t]), bf16_out=False, what=f"token {t}")
    check_state(to_np(state), to_np(st_full))
    cu = la_inputs.cu_seqlens_from_lengths([N + m] * B)
    _, rst = oracle_mod.recurrent(la_inputs.bits(q.reshape(-1, H, D)), la_inputs.bits(k.reshape(-1, H, D)),
                                  la_inputs.bits(v.reshape(-1, H, D)), cu)
    check_state(to_np(state), rst)
    assert la.get_device_status() == la.LA_OK
