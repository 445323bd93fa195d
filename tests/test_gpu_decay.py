"""GPU parity of the per-head decay entry points (la_prefill_decay,
la_prefill_varlen_decay, la_decode_step_decay, through the C ABI) against the
fp64 oracle's decayed forms, element by element on seeded inputs: ragged
tails, several segments per head, carried-in states, packed sequences with
empty members, the bf16 hi + lo state path of long sequences, decode after
prefill, lambda = 1, and rejected decay values.

Decays: the geometric per-head schedule lambda_h = exp(-2^(-8 (h+1) / H))
(values from about 0.37 to 0.996 at H = 8), plus exactly 1 and a small value
on some heads.  Tolerances are those of every other parity test (output
rel-L2 <= 5e-3, max-abs <= 2e-2; fp32 state rel-L2 <= 1e-4)."""
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


def geometric_decays(H):
    return np.exp(-(2.0 ** (-8.0 * (np.arange(H) + 1) / H)))


def _dev(lam):
    return torch.tensor(np.asarray(lam, np.float32), device="cuda")


def _oracle(oracle_mod, q, k, v, cu, lam, state_in=None, heads=None):
    """Decayed recurrent form on packed [T, H, d] bf16 tensors (fp32 decays as the GPU sees them)."""
    sin = None if state_in is None else to_np(state_in)
    if sin is not None and heads is not None:
        sin = sin[:, heads]
    lam64 = np.asarray(lam, np.float32).astype(np.float64)
    return oracle_mod.recurrent_decay(la_inputs.bits(q), la_inputs.bits(k), la_inputs.bits(v), cu, lam64,
                                      heads=heads, state_in=sin)


@pytest.mark.parametrize("N", [1, 127, 129, 300, 1000])
@pytest.mark.parametrize("seg", [0, 128, 256])
def test_decay_ragged_and_segmented(oracle_mod, N, seg):
    B, H = 2, 3
    lam = [1.0, 0.97, 0.5]
    q, k, v = la_inputs.qkv((B, N, H, D), seed=900 + N, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(9)
    state_in = torch.randn((B, H, D, D), generator=gen, device="cuda") * 0.3
    la.set_segment_len(seg)
    out, st = la.prefill(q, k, v, state_in=state_in, out_dtype=torch.float32, decay=_dev(lam))
    assert la.get_device_status() == la.LA_OK
    cu = la_inputs.cu_seqlens_from_lengths([N] * B)
    ref, rst = _oracle(oracle_mod, q.reshape(B * N, H, D), k.reshape(B * N, H, D), v.reshape(B * N, H, D),
                       cu, lam, state_in)
    check_out(to_np(out.reshape(B * N, H, D)), ref, bf16_out=False, what=f"N={N} seg={seg}")
    check_state(to_np(st), rst, what=f"N={N} seg={seg}")


def test_decay_32k_bf16_geometric(oracle_mod):
    B, N, H = 1, 32768, 8
    lam = geometric_decays(H)
    q, k, v = la_inputs.qkv((B, N, H, D), seed=901, device="cuda")
    out, st = la.prefill(q, k, v, out_dtype=torch.bfloat16, decay=_dev(lam))
    assert la.get_device_status() == la.LA_OK
    ref, rst = _oracle(oracle_mod, q[0], k[0], v[0], np.array([0, N], np.int32), lam)
    check_out(to_np(out[0]), ref, bf16_out=True, what="32K bf16")
    check_state(to_np(st[0]), rst[0], what="32K state")


def test_decay_varlen_packed_with_empty(oracle_mod):
    lens = [300, 0, 1, 2500, 129, 0, 777]
    H = 4
    lam = [0.999, 1.0, 0.8, 0.25]
    cu = la_inputs.cu_seqlens_from_lengths(lens)
    T = int(cu[-1])
    q, k, v = la_inputs.qkv((T, H, D), seed=902, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(10)
    state_in = torch.randn((len(lens), H, D, D), generator=gen, device="cuda") * 0.2
    la.set_segment_len(256)
    out, st = la.prefill_varlen(q, k, v, torch.from_numpy(cu).cuda(), max(lens), state_in=state_in,
                                out_dtype=torch.float32, decay=_dev(lam))
    assert la.get_device_status() == la.LA_OK
    ref, rst = _oracle(oracle_mod, q, k, v, cu, lam, state_in)
    check_out(to_np(out), ref, bf16_out=False, what="varlen decay")
    check_state(to_np(st), rst, what="varlen decay states")
    assert torch.equal(st[1], state_in[1]) and torch.equal(st[5], state_in[5])  # empty: unchanged


def test_decay_long_sequence_hi_lo_path(oracle_mod):
    """131072 tokens: segments past 32768 hand S to the inter-block product as
    bf16 hi + lo; heads with lambda = 1 and lambda close to 1 keep S growing."""
    B, N, H = 1, 131072, 4
    lam = [1.0, 1.0 - 1e-5, 0.9995, 0.6]
    q, k, v = la_inputs.qkv((B, N, H, D), seed=903, device="cuda")
    for dtype in (torch.float32, torch.bfloat16):
        out, st = la.prefill(q, k, v, out_dtype=dtype, decay=_dev(lam))
        assert la.get_device_status() == la.LA_OK
        if dtype == torch.float32:
            ref, rst = _oracle(oracle_mod, q[0], k[0], v[0], np.array([0, N], np.int32), lam)
        check_out(to_np(out[0]), ref, bf16_out=dtype == torch.bfloat16, what=f"131072 {dtype}")
        check_state(to_np(st[0]), rst[0], what="131072 state")
        del out, st


def test_decay_one_matches_undecayed(oracle_mod):
    B, N, H = 2, 2000, 3
    q, k, v = la_inputs.qkv((B, N, H, D), seed=904, device="cuda")
    la.set_segment_len(512)
    out_d, st_d = la.prefill(q, k, v, out_dtype=torch.float32, decay=_dev([1.0] * H))
    out_u, st_u = la.prefill(q, k, v, out_dtype=torch.float32)
    assert la.get_device_status() == la.LA_OK
    check_out(to_np(out_d), to_np(out_u), bf16_out=False, what="lambda=1 vs undecayed kernel")
    check_state(to_np(st_d), to_np(st_u), what="lambda=1 states")
    cu = la_inputs.cu_seqlens_from_lengths([N] * B)
    ref, rst = oracle_mod.recurrent(la_inputs.bits(q.reshape(-1, H, D)), la_inputs.bits(k.reshape(-1, H, D)),
                                    la_inputs.bits(v.reshape(-1, H, D)), cu)
    check_out(to_np(out_d.reshape(-1, H, D)), ref, bf16_out=False, what="lambda=1 vs undecayed oracle")
    check_state(to_np(st_d), rst, what="lambda=1 vs undecayed oracle states")


def test_decay_decode_after_prefill(oracle_mod):
    """Decayed decode steps continue a decayed prefill exactly like the
    prefill of the longer sequences (oracle), step by step."""
    B, N, H, STEPS = 3, 700, 4, 12
    lam = [0.95, 1.0, 0.7, 0.999]
    q, k, v = la_inputs.qkv((B, N + STEPS, H, D), seed=905, device="cuda")
    _, st = la.prefill(q[:, :N].contiguous(), k[:, :N].contiguous(), v[:, :N].contiguous(),
                       out_dtype=torch.float32, decay=_dev(lam))
    cu = la_inputs.cu_seqlens_from_lengths([N + STEPS] * B)
    ref, rst = _oracle(oracle_mod, q.reshape(-1, H, D), k.reshape(-1, H, D), v.reshape(-1, H, D), cu, lam)
    ref = ref.reshape(B, N + STEPS, H, D)
    dec = _dev(lam)
    for s in range(STEPS):
        o = la.decode_step(q[:, N + s].contiguous(), k[:, N + s].contiguous(), v[:, N + s].contiguous(), st,
                           out_dtype=torch.float32, decay=dec)
        check_out(to_np(o), ref[:, N + s], bf16_out=False, what=f"decode step {s}")
    assert la.get_device_status() == la.LA_OK
    check_state(to_np(st), rst, what="state after decayed decode")


def test_decay_decode_vs_oracle_step(oracle_mod):
    B, H = 64, 8
    lam = geometric_decays(H)
    gen = torch.Generator(device="cuda").manual_seed(11)
    state = torch.randn((B, H, D, D), generator=gen, device="cuda") * 0.1
    ref_state = to_np(state)
    for s in range(4):
        q, k, v = la_inputs.qkv((B, H, D), seed=la_inputs.decode_seed(906, s), device="cuda")
        o = la.decode_step(q, k, v, state, out_dtype=torch.bfloat16, decay=_dev(lam))
        ro, ref_state = oracle_mod.decode_step_decay(la_inputs.bits(q), la_inputs.bits(k), la_inputs.bits(v),
                                                     ref_state, np.asarray(lam, np.float32).astype(np.float64))
        check_out(to_np(o), ro, bf16_out=True, what=f"decode {s}")
    assert la.get_device_status() == la.LA_OK
    check_state(to_np(state), ref_state, what="decode states")


@pytest.mark.parametrize("bad", [0.0, 1.5, float("nan"), -0.5])
def test_decay_rejects_values_outside_unit_interval(bad):
    B, N, H = 1, 256, 2
    q, k, v = la_inputs.qkv((B, N, H, D), seed=907, device="cuda")
    out = torch.full((B, N, H, D), 7.0, dtype=torch.float32, device="cuda")
    st = torch.full((B, H, D, D), 7.0, dtype=torch.float32, device="cuda")
    la.prefill(q, k, v, out=out, state_out=st, decay=_dev([0.9, bad]))
    assert la.get_device_status() == la.LA_ERR_INVALID_ARGUMENT
    assert torch.all(out == 7.0) and torch.all(st == 7.0)      # nothing computed
    qd, kd, vd = la_inputs.qkv((2, H, D), seed=908, device="cuda")
    sd = torch.zeros((2, H, D, D), dtype=torch.float32, device="cuda")
    od = torch.full((2, H, D), 7.0, dtype=torch.float32, device="cuda")
    la.decode_step(qd, kd, vd, sd, out=od, decay=_dev([0.9, bad]))
    assert la.get_device_status() == la.LA_ERR_INVALID_ARGUMENT
    assert torch.all(od[:, 1] == 7.0) and torch.all(sd[:, 1] == 0.0)  # the bad head's rows skipped
    assert not torch.all(od[:, 0] == 7.0)                              # the good head ran
