"""la_prefill_noalloc: the prefill entry point for callers that cannot allocate
device memory when they call (a plugin whose host framework owns the
allocator, a server that reserved all GPU memory up front and forbids
cudaMalloc on its request path).  It uses a fixed scratch array inside the
library instead of a caller-provided workspace.

Called here through the C ABI (ctypes), two calls in a row on different
inputs (the calls share the scratch), and compared element by element with
the fp64 oracle under the tolerances of the other parity tests, for both
output dtypes, with and without a carried-in state; the shapes include one
just under the scratch limit and one where the segments are lengthened past
32768 tokens (the state then reaches the inter-block product as bf16 hi + lo).
A second comparison against la_prefill on the same inputs, run with the
segment length the scratch-bound call chose, checks that the two entry points
compute the same thing.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import la_inputs
import linear_attention_blocked_b200 as la
from parity_util import check_out, check_state, to_np

pytestmark = pytest.mark.gpu

D = 128


def _noalloc(q, k, v, out, state_out, state_in=None):
    B, N, H, d = q.shape
    code = la.LA_FP32 if out.dtype == torch.float32 else la.LA_BF16
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return la.lib().la_prefill_noalloc(p(q), p(k), p(v), B, N, H, d, 0, p(state_in), p(out), code,
                                       p(state_out), stream)


def _oracle(oracle_mod, q, k, v, state_in, heads):
    """fp64 recurrent form of the B sequences of [B, N, H, d] q, k, v on `heads`."""
    B, N, H, _ = q.shape
    hsel = torch.as_tensor(heads, device=q.device, dtype=torch.long)
    Q = la_inputs.bits(q[:, :, hsel].reshape(B * N, len(heads), D))
    K = la_inputs.bits(k[:, :, hsel].reshape(B * N, len(heads), D))
    V = la_inputs.bits(v[:, :, hsel].reshape(B * N, len(heads), D))
    sin = None if state_in is None else to_np(state_in[:, hsel])
    cu = la_inputs.cu_seqlens_from_lengths([N] * B)
    out, st = oracle_mod.recurrent(Q, K, V, cu, state_in=sin)
    return out.reshape(B, N, len(heads), D), st


CASES = [
    # (B, N, H, heads checked against the oracle, segment length expected or None)
    ((2, 1500, 4), None, None),
    ((1, 32768, 64), 8, None),
    ((4, 4096, 64), 8, 4096),        # 256 (sequence, head) pairs: one segment each, under the limit
    ((1, 131072, 64), 4, 32768),     # segments of 32768 tokens; the last three end past 32768
]


@pytest.mark.parametrize("with_state", [True, False])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c[0])))
def test_noalloc_matches_oracle_twice(oracle_mod, case, out_dtype, with_state):
    (B, N, H), nheads, seg_expect = case
    la.set_segment_len(0)
    heads = list(range(H)) if nheads is None else \
        sorted(np.random.default_rng(B * N + H).choice(H, nheads, replace=False).tolist())
    bf16 = out_dtype == torch.bfloat16
    for call in range(2):                     # two calls in a row share the scratch
        q, k, v = la_inputs.qkv((B, N, H, D), seed=700 + call, device="cuda")
        s_in = None
        if with_state:
            gen = torch.Generator(device="cuda").manual_seed(800 + call)
            s_in = torch.randn((B, H, D, D), generator=gen, device="cuda") * 0.1
        out = torch.empty((B, N, H, D), dtype=out_dtype, device="cuda")
        st = torch.full((B, H, D, D), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(q, k, v, out, st, s_in) == la.LA_OK
        assert la.get_device_status() == la.LA_OK
        if seg_expect is not None:
            assert la.last_segment_len() == seg_expect
        ref, rst = _oracle(oracle_mod, q, k, v, s_in, heads)
        hsel = torch.as_tensor(heads, device="cuda", dtype=torch.long)
        what = f"{B}x{N}x{H} {out_dtype} state={with_state} call {call}"
        check_out(to_np(out[:, :, hsel]), ref, bf16_out=bf16, what=what)
        check_state(to_np(st[:, hsel]), rst, what=what)
        # the workspace entry point on the same inputs, with the segment length
        # the scratch-bound call chose, computes the same outputs and states
        la.set_segment_len(la.last_segment_len())
        try:
            ref_out, ref_st = la.prefill(q, k, v, state_in=s_in, out_dtype=out_dtype)
        finally:
            la.set_segment_len(0)
        assert la.get_device_status() == la.LA_OK
        check_out(to_np(out[:, :, hsel]), to_np(ref_out[:, :, hsel]), bf16_out=bf16, what=what + " vs la_prefill")
        check_state(to_np(st), to_np(ref_st), what=what + " vs la_prefill")
        del q, k, v, out, st, ref_out, ref_st


def test_noalloc_empty_sequences(oracle_mod):
    B, N, H = 3, 0, 4
    q = torch.empty((B, N, H, D), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((B, N, H, D), dtype=torch.float32, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(5)
    s_in = torch.randn((B, H, D, D), generator=gen, device="cuda")
    st = torch.zeros((B, H, D, D), dtype=torch.float32, device="cuda")
    for _ in range(2):
        st.zero_()
        assert _noalloc(q, q, q, out, st, s_in) == la.LA_OK
        assert la.get_device_status() == la.LA_OK
        assert torch.equal(st, s_in)          # the final state of an empty sequence is its start state


def test_noalloc_rejects_problems_beyond_its_scratch():
    B, N, H = 8, 128, 64                      # 512 (sequence, head) pairs: needs more than 32 MiB
    q, k, v = la_inputs.qkv((B, N, H, D), seed=9, device="cuda")
    out = torch.full((B, N, H, D), 3.0, dtype=torch.float32, device="cuda")
    st = torch.zeros((B, H, D, D), dtype=torch.float32, device="cuda")
    assert _noalloc(q, k, v, out, st) == la.LA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(out == 3.0)              # nothing was launched
    assert la.get_device_status() == la.LA_OK
