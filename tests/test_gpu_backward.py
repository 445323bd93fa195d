"""GPU parity of la_prefill_backward (the gradients of la_prefill) against
the fp64 oracle's gradients, element by element, on seeded inputs: ragged
tails, several cross-SM segments, carried-in states and state gradients, bf16
and fp32 gradients, sampled heads at 4096 tokens, and at the single-sequence
prefill workload (B=1, H=64, N=32768) and at 131072 tokens windows of rows
of sampled heads (the first, the last, and one across the point where the
reversed sweep switches its state to bf16 hi + lo), with the rest of the
sequence summarised by the oracle's forward; and the packed-batch form
(la_prefill_backward_varlen) on packed sequences with empty and ragged
members, against the oracle and bit for bit against the fixed-length form
at equal lengths."""
import ctypes

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


def _oracle_packed(oracle_mod, q, k, v, g, cu, sin=None, gs=None):
    return oracle_mod.backward(la_inputs.bits(q), la_inputs.bits(k), la_inputs.bits(v), la_inputs.bits(g), cu,
                               state_in=None if sin is None else to_np(sin),
                               dstate_out=None if gs is None else to_np(gs))


@pytest.mark.parametrize("lens,H,seg", [([300, 0, 1, 2500, 129, 0, 777], 3, 256), ([128, 256, 1000], 2, 0),
                                        ([5000, 37, 3100], 2, 1024)])
@pytest.mark.parametrize("with_states", [False, True])
def test_backward_varlen_matches_oracle(oracle_mod, lens, H, seg, with_states):
    """la_prefill_backward_varlen on packed batches with empty, one-token and
    ragged sequences, several segments per sequence (the reversed sweep
    starts at each sequence's last, partial segment), with and without
    carried-in states and state gradients: fp32 gradients and dS_in of every
    sequence against the oracle's gradients of the packed forward."""
    cu = la_inputs.cu_seqlens_from_lengths(lens)
    T, nseq = int(cu[-1]), len(lens)
    q, k, v = la_inputs.qkv((T, H, D), seed=980 + T, device="cuda")
    g, _, _ = la_inputs.qkv((T, H, D), seed=981 + T, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(982)
    sin = torch.randn((nseq, H, D, D), generator=gen, device="cuda") * 0.2 if with_states else None
    gs = torch.randn((nseq, H, D, D), generator=gen, device="cuda") * 0.05 if with_states else None
    if seg:
        la.set_segment_len(seg)
    got = la.prefill_backward_varlen(q, k, v, g, torch.from_numpy(cu).cuda(), max(lens), state_in=sin,
                                     dstate_out=gs, grad_dtype=torch.float32)
    assert la.get_device_status() == la.LA_OK
    ref = _oracle_packed(oracle_mod, q, k, v, g, cu, sin, gs)
    what = f"lens={lens} seg={seg} states={with_states}"
    for name, x, y in zip(("dq", "dk", "dv"), got[:3], ref[:3]):
        check_out(to_np(x), y, bf16_out=False, what=f"{what} {name}")
    check_state(to_np(got[3]), ref[3], what=f"{what} dS_in")
    for i, n in enumerate(lens):  # an empty sequence passes its state gradient through
        if n == 0:
            assert torch.equal(got[3][i], gs[i] if gs is not None else torch.zeros_like(got[3][i]))


def test_backward_varlen_equal_lengths_match_fixed():
    """Equal lengths: the packed entry point builds the same segments as the
    fixed-length one, so its gradients are the same bits."""
    B, N, H = 3, 700, 2
    q, k, v, g = _inputs(B, N, H, seed=990)
    la.set_segment_len(256)
    fixed = la.prefill_backward(q, k, v, g)
    cu = torch.from_numpy(la_inputs.cu_seqlens_from_lengths([N] * B)).cuda()
    flat = lambda t: t.reshape(B * N, H, D)  # noqa: E731
    packed = la.prefill_backward_varlen(flat(q), flat(k), flat(v), flat(g), cu, N)
    assert la.get_device_status() == la.LA_OK
    for x, y in zip(fixed[:3], packed[:3]):
        assert torch.equal(flat(x), y)
    assert torch.equal(fixed[3], packed[3])


def test_backward_varlen_rejects_a_bad_table():
    """A cu_seqlens table that does not end at the token count is refused on
    the device: the status word says so and no gradient is written."""
    lens = [100, 200]
    T, H = 300, 2
    q, k, v = la_inputs.qkv((T, H, D), seed=995, device="cuda")
    bad = torch.tensor([0, 100, 250], dtype=torch.int32, device="cuda")
    grads = [torch.full((T, H, D), 7.0, dtype=torch.float32, device="cuda") for _ in range(3)]
    dsin = torch.full((2, H, D, D), 7.0, dtype=torch.float32, device="cuda")
    ws = torch.empty(la.backward_varlen_workspace_size(2, T, max(lens), H), dtype=torch.uint8, device="cuda")
    L = la.lib()
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = L.la_prefill_backward_varlen(P(q), P(k), P(v), P(q), P(bad), 2, T, 200, H, D, None, None, P(grads[0]),
                                      P(grads[1]), P(grads[2]), la.LA_FP32, P(dsin), P(ws), ws.numel(),
                                      ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == la.LA_OK                           # the table is checked on the device
    assert la.get_device_status() == la.LA_ERR_INVALID_ARGUMENT
    assert all(torch.all(x == 7.0) for x in grads) and torch.all(dsin == 7.0)
