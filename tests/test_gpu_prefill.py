"""GPU parity of la_prefill / la_prefill_varlen (through the C ABI) against the
fp64 oracle, element by element, on seeded inputs: several row blocks, ragged
tails, multi-segment cross-SM hand-off, carried-in states, packed sequences
with empty members, and the invariants of the method."""
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
    la.debug_inject(0)
    la.set_wait_limit_ns(0)
    yield
    la.set_segment_len(0)
    la.debug_inject(0)
    la.set_wait_limit_ns(0)
    assert la.get_device_status() == la.LA_OK


def _oracle_prefill(oracle_mod, q, k, v, cu, state_in=None, heads=None, form="recurrent", block=None):
    Q, K, V = la_inputs.bits(q), la_inputs.bits(k), la_inputs.bits(v)
    sin = None if state_in is None else to_np(state_in)
    if sin is not None and heads is not None:
        sin = sin[:, heads]
    if form == "blocked":
        return oracle_mod.blocked(Q, K, V, cu, block, heads=heads, state_in=sin)
    return getattr(oracle_mod, form)(Q, K, V, cu, heads=heads, state_in=sin)


def test_config1_small_prefill_fp32(oracle_mod):
    """B=1, H=2, N=1024, fp32 out, row blocks of 64 (the block of this
    configuration); the oracle's blocked form at block 64 and its quadratic
    form both serve as reference."""
    B, N, H = 1, 1024, 2
    q, k, v = la_inputs.qkv((B, N, H, D), seed=1, device="cuda")
    out, st = la.prefill(q, k, v, block=64, out_dtype=torch.float32)
    assert la.get_device_status() == la.LA_OK
    cu = np.array([0, N], np.int32)
    ref_b, st_b = _oracle_prefill(oracle_mod, q[0], k[0], v[0], cu, form="blocked", block=64)
    ref_q, _ = _oracle_prefill(oracle_mod, q[0], k[0], v[0], cu, form="quadratic")
    check_out(to_np(out[0]), ref_b, bf16_out=False, what="vs blocked-64")
    check_out(to_np(out[0]), ref_q, bf16_out=False, what="vs quadratic")
    check_state(to_np(st[0]), st_b[0], what="final state")


@pytest.mark.parametrize("N", [1, 5, 127, 128, 129, 300, 1000])
@pytest.mark.parametrize("seg", [0, 128, 256])
def test_prefill_ragged_and_segmented(oracle_mod, N, seg):
    B, H = 2, 3
    q, k, v = la_inputs.qkv((B, N, H, D), seed=100 + N, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(7)
    state_in = torch.randn((B, H, D, D), generator=gen, device="cuda") * 0.3
    la.set_segment_len(seg)
    out, st = la.prefill(q, k, v, state_in=state_in, out_dtype=torch.float32)
    assert la.get_device_status() == la.LA_OK
    cu = la_inputs.cu_seqlens_from_lengths([N] * B)
    ref, rst = _oracle_prefill(oracle_mod, q.reshape(B * N, H, D), k.reshape(B * N, H, D),
                               v.reshape(B * N, H, D), cu, state_in=state_in)
    check_out(to_np(out.reshape(B * N, H, D)), ref, bf16_out=False, what=f"N={N} seg={seg}")
    check_state(to_np(st), rst, what=f"N={N} seg={seg}")


def test_prefill_bf16_out_many_segments(oracle_mod):
    B, N, H = 1, 4096, 4
    q, k, v = la_inputs.qkv((B, N, H, D), seed=3, device="cuda")
    la.set_segment_len(128)   # 32 segments per head: long hand-off chains
    out, st = la.prefill(q, k, v, out_dtype=torch.bfloat16)
    assert la.get_device_status() == la.LA_OK
    assert la.last_segment_len() == 128
    cu = np.array([0, N], np.int32)
    ref, rst = _oracle_prefill(oracle_mod, q[0], k[0], v[0], cu)
    check_out(to_np(out[0]), ref, bf16_out=True, what="bf16 out")
    check_state(to_np(st[0]), rst[0], what="state")


def test_prefill_in_place_state(oracle_mod):
    B, N, H = 2, 700, 2
    q, k, v = la_inputs.qkv((B, N, H, D), seed=4, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(9)
    s = torch.randn((B, H, D, D), generator=gen, device="cuda")
    s0 = s.clone()
    la.set_segment_len(256)
    out, st = la.prefill(q, k, v, state_in=s, state_out=s, out_dtype=torch.float32)
    assert st.data_ptr() == s.data_ptr()
    cu = la_inputs.cu_seqlens_from_lengths([N] * B)
    ref, rst = _oracle_prefill(oracle_mod, q.reshape(-1, H, D), k.reshape(-1, H, D), v.reshape(-1, H, D),
                               cu, state_in=s0)
    check_out(to_np(out.reshape(-1, H, D)), ref, bf16_out=False)
    check_state(to_np(s), rst)


def test_varlen_packed_with_empty_and_ragged(oracle_mod):
    lens = [0, 1, 127, 128, 129, 1000, 0, 2500, 64]
    H = 3
    T = sum(lens)
    q, k, v = la_inputs.qkv((T, H, D), seed=5, device="cuda")
    cu = la_inputs.cu_seqlens_from_lengths(lens)
    cu_d = torch.from_numpy(cu).cuda()
    gen = torch.Generator(device="cuda").manual_seed(11)
    state_in = torch.randn((len(lens), H, D, D), generator=gen, device="cuda") * 0.2
    for seg in (0, 256):
        la.set_segment_len(seg)
        out, st = la.prefill_varlen(q, k, v, cu_d, max(lens), state_in=state_in, out_dtype=torch.float32)
        assert la.get_device_status() == la.LA_OK
        ref, rst = _oracle_prefill(oracle_mod, q, k, v, cu, state_in=state_in)
        check_out(to_np(out), ref, bf16_out=False, what=f"varlen seg={seg}")
        check_state(to_np(st), rst, what=f"varlen seg={seg}")
        # empty sequences return their carried-in state unchanged
        for i in (0, 6):
            assert torch.equal(st[i], state_in[i])


def test_varlen_sequences_are_isolated():
    """Changing one packed sequence changes none of the others (bitwise)."""
    lens = [300, 129, 515, 128]
    H, T = 2, sum(lens)
    q, k, v = la_inputs.qkv((T, H, D), seed=6, device="cuda")
    cu = la_inputs.cu_seqlens_from_lengths(lens)
    cu_d = torch.from_numpy(cu).cuda()
    la.set_segment_len(128)
    out1, st1 = la.prefill_varlen(q, k, v, cu_d, max(lens), out_dtype=torch.float32)
    a, b = int(cu[1]), int(cu[2])
    q2, k2, v2 = q.clone(), k.clone(), v.clone()
    q2[a:b], k2[a:b], v2[a:b] = la_inputs.qkv((b - a, H, D), seed=66, device="cuda")
    out2, st2 = la.prefill_varlen(q2, k2, v2, cu_d, max(lens), out_dtype=torch.float32)
    assert torch.equal(out1[:a], out2[:a]) and torch.equal(out1[b:], out2[b:])
    assert torch.equal(st1[0], st2[0]) and torch.equal(st1[2:], st2[2:])
    assert not torch.equal(out1[a:b], out2[a:b])
    # NaN in one sequence stays in that sequence (the neighbour's ragged last
    # block reads these rows through TMA and must not pick them up)
    q2[a:b], k2[a:b], v2[a:b] = float("nan"), float("nan"), float("nan")
    out3, st3 = la.prefill_varlen(q2, k2, v2, cu_d, max(lens), out_dtype=torch.float32)
    assert torch.equal(out1[:a], out3[:a]) and torch.equal(out1[b:], out3[b:])
    assert torch.equal(st1[0], st3[0]) and torch.equal(st1[2:], st3[2:])


def test_state_carry_equals_longer_prefill():
    """prefill(A) then prefill(B, state_in = S_A) == prefill(A ++ B)."""
    H, NA, NB = 2, 640, 333
    q, k, v = la_inputs.qkv((1, NA + NB, H, D), seed=8, device="cuda")
    out_full, st_full = la.prefill(q, k, v, out_dtype=torch.float32)
    _, sA = la.prefill(q[:, :NA].contiguous(), k[:, :NA].contiguous(), v[:, :NA].contiguous(),
                       out_dtype=torch.float32)
    outB, sB = la.prefill(q[:, NA:].contiguous(), k[:, NA:].contiguous(), v[:, NA:].contiguous(),
                          state_in=sA, out_dtype=torch.float32)
    check_out(to_np(outB), to_np(out_full[:, NA:]), bf16_out=False)
    check_state(to_np(sB), to_np(st_full))


def test_invalid_cu_seqlens_is_reported_on_device():
    H, T = 1, 256
    q, k, v = la_inputs.qkv((T, H, D), seed=9, device="cuda")
    cu_bad = torch.tensor([0, 200, 100, 256], dtype=torch.int32, device="cuda")   # decreasing
    out = torch.full((T, H, D), 7.0, device="cuda")
    la.prefill_varlen(q, k, v, cu_bad, 256, out=out, out_dtype=torch.float32)
    assert la.get_device_status() == la.LA_ERR_INVALID_ARGUMENT
    assert torch.all(out == 7.0)                     # nothing was computed
    cu_big = torch.tensor([0, 100, 256], dtype=torch.int32, device="cuda")      # exceeds max_seqlen
    la.prefill_varlen(q, k, v, cu_big, 120, out=out, out_dtype=torch.float32)
    assert la.get_device_status() == la.LA_ERR_INVALID_ARGUMENT
    assert la.get_device_status() == la.LA_OK        # the word was cleared


def test_bounded_wait_reports_timeout_and_recovers(oracle_mod):
    """Host-side fault injection: segments never publish their prefix, so every
    successor's bounded wait runs out; the kernel still finishes, the status
    word says LA_ERR_TIMEOUT, and the next normal call is correct."""
    B, N, H = 1, 2048, 2
    q, k, v = la_inputs.qkv((B, N, H, D), seed=10, device="cuda")
    la.set_segment_len(256)
    la.set_wait_limit_ns(20_000_000)   # 20 ms
    la.debug_inject(la.LA_INJECT_SKIP_PUBLISH)
    la.prefill(q, k, v, out_dtype=torch.float32)
    assert la.get_device_status() == la.LA_ERR_TIMEOUT
    la.debug_inject(la.LA_INJECT_NONE)
    la.set_wait_limit_ns(0)
    out, st = la.prefill(q, k, v, out_dtype=torch.float32)
    assert la.get_device_status() == la.LA_OK
    ref, rst = _oracle_prefill(oracle_mod, q[0], k[0], v[0], np.array([0, N], np.int32))
    check_out(to_np(out[0]), ref, bf16_out=False)
    check_state(to_np(st[0]), rst[0])


def test_kernel_launch_count_increases():
    before = la.kernel_launches()
    q, k, v = la_inputs.qkv((1, 256, 1, D), seed=12, device="cuda")
    la.prefill(q, k, v)
    torch.cuda.synchronize()
    assert la.kernel_launches() == before + 2    # scheduler + prefill


def test_long_sequence_uses_split_state_and_stays_accurate(oracle_mod):
    """128K tokens: segments past token 65536 switch the inter-block product to
    the two-term (bf16 hi + lo) state; fp32 outputs stay within 2e-2 max abs
    everywhere along the sequence."""
    B, N, H = 1, 131072, 2
    q, k, v = la_inputs.qkv((B, N, H, D), seed=13, device="cuda")
    out, st = la.prefill(q, k, v, out_dtype=torch.float32)
    assert la.get_device_status() == la.LA_OK
    ref, rst = _oracle_prefill(oracle_mod, q[0], k[0], v[0], np.array([0, N], np.int32))
    got = to_np(out[0])
    for lo, hi in ((0, 65536), (65536, N)):   # both precision regimes
        check_out(got[lo:hi], ref[lo:hi], bf16_out=False, what=f"tokens [{lo}, {hi})")
    check_state(to_np(st[0]), rst[0])


def test_empty_problems():
    """B = 0 and N = 0 launch nothing or only carry the state; an all-empty
    packed batch returns every carried-in state unchanged."""
    z = torch.empty((0, 16, 2, D), dtype=torch.bfloat16, device="cuda")
    out, st = la.prefill(z, z, z, want_state=False)
    assert out.shape == (0, 16, 2, D)
    z2 = torch.empty((3, 0, 2, D), dtype=torch.bfloat16, device="cuda")
    sin = torch.randn((3, 2, D, D), device="cuda")
    out, st = la.prefill(z2, z2, z2, state_in=sin)
    assert torch.equal(st, sin)
    zt = torch.empty((0, 2, D), dtype=torch.bfloat16, device="cuda")
    cu = torch.zeros(4, dtype=torch.int32, device="cuda")
    sin3 = torch.randn((3, 2, D, D), device="cuda")
    out, st = la.prefill_varlen(zt, zt, zt, cu, 0, state_in=sin3)
    assert torch.equal(st, sin3)
    assert la.get_device_status() == la.LA_OK


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_output_only_16_byte_aligned(oracle_mod, dtype):
    """An output buffer that is 16- but not 32-byte aligned (the minimum the C
    ABI accepts) takes the 16-byte store path and gives the same result."""
    B, N, H = 1, 640, 2
    q, k, v = la_inputs.qkv((B, N, H, D), seed=61, device="cuda")
    esz = torch.finfo(dtype).bits // 8
    flat = torch.empty(B * N * H * D + 64, dtype=dtype, device="cuda")
    shift = (16 - flat.data_ptr() % 32) % 32 // esz  # first element 16 bytes past a 32-byte boundary
    out = flat[shift:shift + B * N * H * D].view(B, N, H, D)
    assert out.data_ptr() % 32 == 16
    la.set_segment_len(256)
    out2, _ = la.prefill(q, k, v, out=out, out_dtype=dtype)
    assert out2.data_ptr() == out.data_ptr()
    ref, _ = _oracle_prefill(oracle_mod, q[0], k[0], v[0], np.array([0, N], np.int32))
    check_out(to_np(out[0]), ref, bf16_out=dtype == torch.bfloat16, what="16-byte aligned out")


# ------------------------------------------------------------------ row blocks of 64
@pytest.mark.parametrize("N", [1, 63, 64, 65, 127, 129, 300, 1000])
@pytest.mark.parametrize("seg", [0, 128, 256])
def test_block64_ragged_and_segmented(oracle_mod, N, seg):
    """block = 64: two 64-row blocks per 128-row tile, each with its own state
    snapshot; against the oracle's blocked form at 64 and its recurrent form."""
    B, H = 2, 3
    q, k, v = la_inputs.qkv((B, N, H, D), seed=200 + N, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(17)
    state_in = torch.randn((B, H, D, D), generator=gen, device="cuda") * 0.3
    la.set_segment_len(seg)
    out, st = la.prefill(q, k, v, block=64, state_in=state_in, out_dtype=torch.float32)
    assert la.get_device_status() == la.LA_OK
    cu = la_inputs.cu_seqlens_from_lengths([N] * B)
    qf, kf, vf = (x.reshape(B * N, H, D) for x in (q, k, v))
    ref, rst = _oracle_prefill(oracle_mod, qf, kf, vf, cu, state_in=state_in, form="blocked", block=64)
    check_out(to_np(out.reshape(B * N, H, D)), ref, bf16_out=False, what=f"block64 N={N} seg={seg}")
    check_state(to_np(st), rst, what=f"block64 N={N} seg={seg}")
    ref2, _ = _oracle_prefill(oracle_mod, qf, kf, vf, cu, state_in=state_in)
    check_out(to_np(out.reshape(B * N, H, D)), ref2, bf16_out=False, what=f"block64 vs recurrent N={N}")


def test_block64_varlen_bf16(oracle_mod):
    lens = [0, 1, 64, 65, 1000, 0, 2500, 191]
    H = 4
    T = sum(lens)
    q, k, v = la_inputs.qkv((T, H, D), seed=210, device="cuda")
    cu = la_inputs.cu_seqlens_from_lengths(lens)
    la.set_segment_len(256)
    out, st = la.prefill_varlen(q, k, v, torch.from_numpy(cu).cuda(), max(lens), block=64,
                                out_dtype=torch.bfloat16)
    assert la.get_device_status() == la.LA_OK
    ref, rst = _oracle_prefill(oracle_mod, q, k, v, cu, form="blocked", block=64)
    check_out(to_np(out), ref, bf16_out=True, what="block64 varlen")
    check_state(to_np(st), rst, what="block64 varlen states")


def test_block64_long_sequence_hi_lo(oracle_mod):
    """131072 tokens at block 64: the state reaches the inter-block products as
    bf16 hi + lo past 65536 tokens, two row halves per tile."""
    B, N, H = 1, 131072, 2
    q, k, v = la_inputs.qkv((B, N, H, D), seed=211, device="cuda")
    out, st = la.prefill(q, k, v, block=64, out_dtype=torch.float32)
    assert la.get_device_status() == la.LA_OK
    ref, rst = _oracle_prefill(oracle_mod, q[0], k[0], v[0], np.array([0, N], np.int32))
    check_out(to_np(out[0]), ref, bf16_out=False, what="block64 131072")
    check_state(to_np(st[0]), rst[0], what="block64 131072 state")


@pytest.mark.parametrize("block", [64, 256])
def test_block_64_256_rejected_with_decay(block):
    q, k, v = la_inputs.qkv((1, 128, 2, D), seed=212, device="cuda")
    with pytest.raises(la.LAError) as e:
        la.prefill(q, k, v, block=block, decay=torch.ones(2, device="cuda"))
    assert e.value.status == la.LA_ERR_UNSUPPORTED


# ------------------------------------------------------------------ row blocks of 256
@pytest.mark.parametrize("N", [1, 127, 128, 129, 255, 256, 257, 383, 1000])
@pytest.mark.parametrize("seg", [0, 128, 256, 512])
def test_block256_ragged_and_segmented(oracle_mod, N, seg):
    """block = 256: pairs of 128-row tiles share one state snapshot, the second
    tile's queries meet the first tile's keys in the intra-block product;
    against the oracle's blocked form at 256 (a segment length of 128 is
    raised to 256 so that segments hold whole blocks)."""
    B, H = 2, 3
    q, k, v = la_inputs.qkv((B, N, H, D), seed=300 + N, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(19)
    state_in = torch.randn((B, H, D, D), generator=gen, device="cuda") * 0.3
    la.set_segment_len(seg)
    out, st = la.prefill(q, k, v, block=256, state_in=state_in, out_dtype=torch.float32)
    assert la.get_device_status() == la.LA_OK
    if seg:
        assert la.last_segment_len() % 256 == 0
    cu = la_inputs.cu_seqlens_from_lengths([N] * B)
    qf, kf, vf = (x.reshape(B * N, H, D) for x in (q, k, v))
    ref, rst = _oracle_prefill(oracle_mod, qf, kf, vf, cu, state_in=state_in, form="blocked", block=256)
    check_out(to_np(out.reshape(B * N, H, D)), ref, bf16_out=False, what=f"block256 N={N} seg={seg}")
    check_state(to_np(st), rst, what=f"block256 N={N} seg={seg}")


def test_block256_varlen_bf16(oracle_mod):
    lens = [0, 1, 256, 257, 1000, 0, 2500, 383]
    H = 4
    T = sum(lens)
    q, k, v = la_inputs.qkv((T, H, D), seed=310, device="cuda")
    cu = la_inputs.cu_seqlens_from_lengths(lens)
    la.set_segment_len(512)
    out, st = la.prefill_varlen(q, k, v, torch.from_numpy(cu).cuda(), max(lens), block=256,
                                out_dtype=torch.bfloat16)
    assert la.get_device_status() == la.LA_OK
    ref, rst = _oracle_prefill(oracle_mod, q, k, v, cu, form="blocked", block=256)
    check_out(to_np(out), ref, bf16_out=True, what="block256 varlen")
    check_state(to_np(st), rst, what="block256 varlen states")


def test_block256_32k_all_heads(oracle_mod):
    """The 32K-token, 64-head workload at block 256, bf16 output, every head."""
    B, N, H = 1, 32768, 64
    q, k, v = la_inputs.qkv((B, N, H, D), seed=20250101, device="cuda")
    out, st = la.prefill(q, k, v, block=256, out_dtype=torch.bfloat16)
    assert la.get_device_status() == la.LA_OK
    ref, rst = _oracle_prefill(oracle_mod, q[0], k[0], v[0], np.array([0, N], np.int32))
    check_out(to_np(out[0]), ref, bf16_out=True, what="block256 32K")
    check_state(to_np(st[0]), rst[0], what="block256 32K states")


def test_block256_long_sequence_hi_lo(oracle_mod):
    B, N, H = 1, 131072, 2
    q, k, v = la_inputs.qkv((B, N, H, D), seed=311, device="cuda")
    out, st = la.prefill(q, k, v, block=256, out_dtype=torch.float32)
    assert la.get_device_status() == la.LA_OK
    ref, rst = _oracle_prefill(oracle_mod, q[0], k[0], v[0], np.array([0, N], np.int32))
    check_out(to_np(out[0]), ref, bf16_out=False, what="block256 131072")
    check_state(to_np(st[0]), rst[0], what="block256 131072 state")


def test_blocks_agree():
    """The three block lengths compute the same operation: outputs agree to the
    output tolerance, final states to the state tolerance."""
    B, N, H = 2, 3000, 4
    q, k, v = la_inputs.qkv((B, N, H, D), seed=312, device="cuda")
    res = {blk: la.prefill(q, k, v, block=blk, out_dtype=torch.float32) for blk in (64, 128, 256)}
    assert la.get_device_status() == la.LA_OK
    for blk in (64, 256):
        check_out(to_np(res[blk][0]), to_np(res[128][0]), bf16_out=False, what=f"block {blk} vs 128")
        check_state(to_np(res[blk][1]), to_np(res[128][1]), what=f"block {blk} vs 128 states")
