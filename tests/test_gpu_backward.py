"""GPU parity of la_prefill_backward (the gradients of la_prefill) against
the fp64 oracle's gradients, element by element, on seeded inputs: ragged
tails, several cross-SM segments, carried-in states and state gradients, bf16
and fp32 gradients, sampled heads at 4096 tokens, and at the single-sequence
prefill workload (B=1, H=64, N=32768) and at 131072 tokens windows of rows
of sampled heads (the first, the last, and one across the point where the
reversed sweep switches its state to bf16 hi + lo), with the rest of the
sequence summarised by the oracle's forward."""
import numpy as np
import pytest
import torch

import la_inputs
import linear_attention_blocked_b200 as la
from parity_util import check_out, check_state, to_np

pytestmark = pytest.mark.gpu

D = 128


@pytest.fixture(autouse=True)
def _clean_controls():
    la.set_segment_len(0)
    yield
    la.set_segment_len(0)
    assert la.get_device_status() == la.LA_OK


def _inputs(B, N, H, seed):
    q, k, v = la_inputs.qkv((B, N, H, D), seed=seed, device="cuda")
    g, _, _ = la_inputs.qkv((B, N, H, D), seed=seed + 1, device="cuda")
    return q, k, v, g


def _oracle(oracle_mod, q, k, v, g, sin=None, gs=None, heads=None):
    B, N, H, _ = q.shape
    flat = lambda t: la_inputs.bits(t.reshape(B * N, H, D))  # noqa: E731
    cu = (np.arange(B + 1) * N).astype(np.int32)
    sel = lambda s: None if s is None else (to_np(s) if heads is None else to_np(s)[:, heads])  # noqa: E731
    return oracle_mod.backward(flat(q), flat(k), flat(v), flat(g), cu, heads=heads, state_in=sel(sin),
                               dstate_out=sel(gs))


def _check_all(got, ref, B, N, nh, bf16, what):
    for name, x, y in zip(("dq", "dk", "dv"), got[:3], ref[:3]):
        check_out(to_np(x).reshape(B * N, nh, D), y, bf16_out=bf16, what=f"{what} {name}")
    if got[3] is not None:
        check_state(to_np(got[3]), ref[3], what=f"{what} dS_in")


@pytest.mark.parametrize("B,N,H,seg", [(1, 300, 2, 0), (2, 129, 3, 0), (1, 1000, 2, 256), (2, 1, 2, 0),
                                       (1, 2500, 3, 0), (3, 777, 2, 128)])
@pytest.mark.parametrize("with_states", [False, True])
def test_backward_matches_oracle(oracle_mod, B, N, H, seg, with_states):
    q, k, v, g = _inputs(B, N, H, seed=900 + N + H)
    gen = torch.Generator(device="cuda").manual_seed(901)
    sin = torch.randn((B, H, D, D), generator=gen, device="cuda") * 0.2 if with_states else None
    gs = torch.randn((B, H, D, D), generator=gen, device="cuda") * 0.05 if with_states else None
    if seg:
        la.set_segment_len(seg)
    got = la.prefill_backward(q, k, v, g, state_in=sin, dstate_out=gs, grad_dtype=torch.float32)
    assert la.get_device_status() == la.LA_OK
    _check_all(got, _oracle(oracle_mod, q, k, v, g, sin, gs), B, N, H, False, f"B={B} N={N} H={H} seg={seg}")


def test_backward_bf16_sampled_heads(oracle_mod):
    B, N, H = 1, 4096, 8
    heads = [1, 6]
    q, k, v, g = _inputs(B, N, H, seed=950)
    gs = torch.randn((B, H, D, D), device="cuda") * 0.05
    dq, dk, dv, dsin = la.prefill_backward(q, k, v, g, dstate_out=gs)
    assert la.get_device_status() == la.LA_OK
    ref = _oracle(oracle_mod, q, k, v, g, None, gs, heads=heads)
    got = (dq[:, :, heads], dk[:, :, heads], dv[:, :, heads], dsin[:, heads])
    _check_all(got, ref, B, N, len(heads), True, "bf16 sampled heads")


@pytest.mark.parametrize("N,H,heads,R,mid", [(32768, 64, [0, 37], 4096, None), (131072, 2, [0, 1], 2048, 98304)])
def test_backward_long_sequence_sampled_rows(oracle_mod, N, H, heads, R, mid):
    """B=1 and N=32768, H=64 (the single-sequence prefill workload) or
    N=131072, H=2 (long enough for the reversed sweep to switch its state to
    bf16 hi + lo, at token 98304 with 4096-token segments): bf16 gradients of
    the sampled heads on windows of R rows -- the first, the last and, at
    131072 tokens, one straddling that switch -- against the oracle.  A
    window [a, b) sees the rest of the sequence only through d x d sums,
    which the oracle's forward supplies: S_in = sum_{t < a} k_t^T v_t (its
    final state over the earlier tokens) for dq, and dS_out = sum_{t >= b}
    q_t^T g_t (its final state with (k, v) = (q, g) over the later tokens)
    for dk and dv.  dS_in = sum_t q_t^T g_t, the reversed sweep's final
    state: against the oracle on the sampled heads and against
    la_kv_aggregate(q, dout) on all."""
    B = 1
    q, k, v, g = _inputs(B, N, H, seed=960 + H)
    dq, dk, dv, dsin = la.prefill_backward(q, k, v, g)
    assert la.get_device_status() == la.LA_OK
    check_state(to_np(dsin), to_np(la.kv_aggregate(q, g)), what=f"N={N} dS_in vs la_kv_aggregate")
    bits = lambda t, a, b: la_inputs.bits(t[0, a:b])  # noqa: E731
    cu = lambda n: np.array([0, n], np.int32)  # noqa: E731
    _, W = oracle_mod.recurrent(bits(q, 0, N), bits(q, 0, N), bits(g, 0, N), cu(N), heads=heads)
    check_state(to_np(dsin[0, heads]), W[0], what=f"N={N} dS_in vs oracle")
    windows = [(0, R), (N - R, N)] + ([(mid - R // 2, mid + R // 2)] if mid else [])
    for a, b in windows:
        S = None
        if a > 0:
            _, S = oracle_mod.recurrent(bits(q, 0, a), bits(k, 0, a), bits(v, 0, a), cu(a), heads=heads)
        G = None
        if b < N:
            _, G = oracle_mod.recurrent(bits(q, b, N), bits(q, b, N), bits(g, b, N), cu(N - b), heads=heads)
        ref = oracle_mod.backward(bits(q, a, b), bits(k, a, b), bits(v, a, b), bits(g, a, b), cu(b - a),
                                  heads=heads, state_in=S, dstate_out=G)
        for name, x, y in zip(("dq", "dk", "dv"), (dq, dk, dv), ref[:3]):
            check_out(to_np(x[0, a:b, heads]), y, bf16_out=True, what=f"N={N} rows {a}-{b} {name}")
