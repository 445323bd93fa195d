"""GPU parity of the sequence-parallel steps (LASP+ across ranks) against the
fp64 oracle: the local prefix la_kv_aggregate equals the oracle's final state
from a zero state; the global prefix la_state_prefix is the ordered fp32 sum
it is defined as; and ranks emulated one after another on one GPU (local
prefix, gather, global prefix, local scan) reproduce the oracle's result for
the whole sequences.  One more test runs lasp_prefill itself under a one-rank
NCCL process group."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import la_inputs
import linear_attention_blocked_b200 as la
from parity_util import check_out, check_state, to_np

pytestmark = pytest.mark.gpu

D = 128
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cu(B, N):
    return (np.arange(B + 1) * N).astype(np.int32)


def _oracle_state(oracle_mod, k, v, heads=None):
    """Final state from a zero state over each sequence of [B, N, H, D] k, v."""
    B, N, H, _ = k.shape
    K = la_inputs.bits(k.reshape(B * N, H, D))
    V = la_inputs.bits(v.reshape(B * N, H, D))
    _, st = oracle_mod.recurrent(K, K, V, _cu(B, N), heads=heads)
    return st


# (B, N, H): every pair cut into one-block pieces; pairs cut at ragged points;
# one whole pair per CTA; ragged tails inside and at the end of the batch;
# single tokens; more pairs than CTAs.
@pytest.mark.parametrize("B,N,H", [(1, 1000, 3), (2, 129, 5), (1, 384, 100), (1, 640, 64), (3, 1, 2),
                                   (2, 300, 7), (4, 2050, 40)])
def test_kv_aggregate_matches_oracle(oracle_mod, B, N, H):
    _, k, v = la_inputs.qkv((B, N, H, D), seed=500 + N + H, device="cuda")
    agg = la.kv_aggregate(k, v)
    assert la.get_device_status() == la.LA_OK
    check_state(to_np(agg), _oracle_state(oracle_mod, k, v), what=f"A for B={B} N={N} H={H}")


def test_kv_aggregate_full_size_sampled_heads(oracle_mod):
    """B=1, N=32768, H=64 (the single-sequence prefill workload), three heads
    checked against the oracle, every head against la_prefill's final state."""
    B, N, H = 1, 32768, 64
    q, k, v = la_inputs.qkv((B, N, H, D), seed=42, device="cuda")
    agg = la.kv_aggregate(k, v)
    _, st = la.prefill(q, k, v)
    assert la.get_device_status() == la.LA_OK
    heads = [0, 17, 63]
    check_state(to_np(agg[:, heads]), _oracle_state(oracle_mod, k, v, heads=heads), what="sampled heads")
    check_state(to_np(agg), to_np(st), what="A vs prefill final state (all heads)")


def test_kv_aggregate_empty_and_deterministic():
    B, H = 2, 3
    k = torch.empty((B, 0, H, D), dtype=torch.bfloat16, device="cuda")
    agg = la.kv_aggregate(k, k.clone())
    assert torch.count_nonzero(agg) == 0
    _, k, v = la_inputs.qkv((B, 777, H, D), seed=9, device="cuda")
    a1 = la.kv_aggregate(k, v)
    a2 = la.kv_aggregate(k, v)
    assert torch.equal(a1, a2)
    assert la.get_device_status() == la.LA_OK


@pytest.mark.parametrize("count", [0, 1, 3, 4])
@pytest.mark.parametrize("with_state", [False, True])
def test_state_prefix_is_the_ordered_fp32_sum(count, with_state):
    W, B, H = 4, 2, 3
    gen = torch.Generator(device="cuda").manual_seed(11 + count)
    parts = torch.randn((W, B, H, D, D), generator=gen, device="cuda")
    sin = torch.randn((B, H, D, D), generator=gen, device="cuda") if with_state else None
    out = la.state_prefix(parts, count, sin)
    # the same additions in the same order in fp32 on the host: bit-exact
    ref = to_np(sin).astype(np.float32) if with_state else np.zeros((B, H, D, D), np.float32)
    p = parts.cpu().numpy()
    for i in range(count):
        ref = (ref + p[i]).astype(np.float32)
    assert np.array_equal(out.cpu().numpy(), ref)
    if with_state:  # in place
        la.state_prefix(parts, count, sin, out=sin)
        assert np.array_equal(sin.cpu().numpy(), ref)


def test_emulated_ranks_reproduce_the_whole_sequence(oracle_mod):
    """Three ranks with parts of 700, 1500 and 829 tokens, run one after the
    other on this GPU: local prefixes, their stack standing in for the
    AllGather, global prefixes, local scans seeded with them."""
    B, H = 2, 4
    lens = [700, 1500, 829]
    N = sum(lens)
    q, k, v = la_inputs.qkv((B, N, H, D), seed=321, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(322)
    sin = torch.randn((B, H, D, D), generator=gen, device="cuda") * 0.1
    bounds = np.concatenate([[0], np.cumsum(lens)])
    shard = lambda t, r: t[:, bounds[r]:bounds[r + 1]].contiguous()
    parts = torch.stack([la.kv_aggregate(shard(k, r), shard(v, r)) for r in range(len(lens))])
    outs = []
    for r in range(len(lens)):
        prefix = la.state_prefix(parts, r, sin)
        o, _ = la.prefill(shard(q, r), shard(k, r), shard(v, r), state_in=prefix, out_dtype=torch.float32,
                          want_state=False)
        outs.append(o)
    final = la.state_prefix(parts, len(lens), sin)
    assert la.get_device_status() == la.LA_OK
    Q, K, V = (la_inputs.bits(t.reshape(B * N, H, D)) for t in (q, k, v))
    ref, rst = oracle_mod.recurrent(Q, K, V, _cu(B, N), state_in=to_np(sin))
    got = torch.cat(outs, dim=1).reshape(B * N, H, D)
    check_out(to_np(got), ref, bf16_out=False, what="rank outputs")
    check_state(to_np(final), rst, what="final state")


@pytest.mark.parametrize("lens,world", [([300, 0, 1290, 77, 0, 2100, 1, 129], 3),
                                        ([40, 5000, 60], 4)])
def test_emulated_ranks_on_a_packed_batch(oracle_mod, lens, world):
    """A packed batch cut evenly into ranges at arbitrary tokens (sequences
    spanning several ranks, empty sequences), run through the same two steps
    lasp_prefill_varlen runs on each rank, with a stack of the local prefixes
    standing in for the AllGather."""
    from linear_attention_blocked_b200 import seqpar
    H = 4
    cu = la_inputs.cu_seqlens_from_lengths(lens)
    T = int(cu[-1])
    q, k, v = la_inputs.qkv((T, H, D), seed=410 + world, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(411)
    sin = torch.randn((len(lens), H, D, D), generator=gen, device="cuda") * 0.1
    bounds = seqpar.split_tokens(T, world)
    plans = [seqpar.plan_varlen_rank(cu, bounds, r) for r in range(world)]
    rng = lambda t, p: t[p.tok0:p.tok1].contiguous()
    parts = torch.stack([seqpar.varlen_local_prefix(p, rng(k, p), rng(v, p)) for p in plans])
    outs, final = [], torch.full((len(lens), H, D, D), float("nan"), device="cuda")
    for p in plans:
        o, st = seqpar.varlen_local_scan(p, rng(q, p), rng(k, p), rng(v, p), parts, sin, torch.float32)
        outs.append(o)
        for i in np.nonzero(p.ends_here)[0]:
            final[p.seq0 + i] = st[i]
    assert la.get_device_status() == la.LA_OK
    ref, rst = oracle_mod.recurrent(la_inputs.bits(q), la_inputs.bits(k), la_inputs.bits(v), cu,
                                    state_in=to_np(sin))
    check_out(to_np(torch.cat(outs, 0)), ref, bf16_out=False, what="packed outputs")
    check_state(to_np(final), rst, what="final states")


@pytest.mark.parametrize("lens,world", [([300, 0, 1290, 77, 0, 2100, 1, 129], 3), ([40, 3000, 60], 4)])
def test_emulated_ranks_gradients_on_a_packed_batch(oracle_mod, lens, world):
    """The gradients of a packed batch cut evenly into ranges at arbitrary
    tokens, through the two steps lasp_prefill_backward_varlen runs on each
    rank (a stack of the local sums standing in for the AllGathers), against
    the oracle's gradients of the whole batch; each sequence's dS_in is taken
    from the rank where it starts."""
    from linear_attention_blocked_b200 import seqpar
    H = 2
    cu = la_inputs.cu_seqlens_from_lengths(lens)
    T = int(cu[-1])
    q, k, v = la_inputs.qkv((T, H, D), seed=430 + world, device="cuda")
    g, _, _ = la_inputs.qkv((T, H, D), seed=431 + world, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(432)
    sin = torch.randn((len(lens), H, D, D), generator=gen, device="cuda") * 0.1
    gs = torch.randn((len(lens), H, D, D), generator=gen, device="cuda") * 0.05
    bounds = seqpar.split_tokens(T, world)
    plans = [seqpar.plan_varlen_rank(cu, bounds, r) for r in range(world)]
    rng = lambda t, p: t[p.tok0:p.tok1].contiguous()  # noqa: E731
    sums = [seqpar.varlen_backward_local_sums(p, rng(q, p), rng(k, p), rng(v, p), rng(g, p)) for p in plans]
    a_parts = torch.stack([a for a, _ in sums])
    b_parts = torch.stack([b for _, b in sums])
    grads = [[], [], []]
    dsin = torch.full((len(lens), H, D, D), float("nan"), device="cuda")
    for p in plans:
        dq, dk, dv, ds = seqpar.varlen_backward_local_grads(p, cu, bounds, rng(q, p), rng(k, p), rng(v, p),
                                                            rng(g, p), a_parts, b_parts, sin, gs, torch.float32)
        for lst, x in zip(grads, (dq, dk, dv)):
            lst.append(x)
        for i in np.nonzero(p.starts_here)[0]:
            dsin[p.seq0 + i] = ds[i]
    assert la.get_device_status() == la.LA_OK
    ref = oracle_mod.backward(*(la_inputs.bits(t) for t in (q, k, v, g)), cu, state_in=to_np(sin),
                              dstate_out=to_np(gs))
    for name, lst, y in zip(("dq", "dk", "dv"), grads, ref[:3]):
        check_out(to_np(torch.cat(lst, 0)), y, bf16_out=False, what=f"packed {name}")
    check_state(to_np(dsin), ref[3], what="packed dS_in")


def test_emulated_ranks_gradients(oracle_mod):
    """Gradients across three ranks (parts of 700, 1500 and 829 tokens), run
    one after the other on this GPU through the same two steps
    lasp_prefill_backward runs on each rank, with stacks of the ranks' sums
    standing in for the AllGathers; fp32 gradients against the oracle's
    gradients of the whole sequences, with a carried-in state and a state
    gradient."""
    from linear_attention_blocked_b200 import seqpar
    B, H = 2, 3
    lens = [700, 1500, 829]
    N = sum(lens)
    q, k, v = la_inputs.qkv((B, N, H, D), seed=331, device="cuda")
    g, _, _ = la_inputs.qkv((B, N, H, D), seed=332, device="cuda")
    gen = torch.Generator(device="cuda").manual_seed(333)
    sin = torch.randn((B, H, D, D), generator=gen, device="cuda") * 0.1
    gs = torch.randn((B, H, D, D), generator=gen, device="cuda") * 0.05
    bounds = np.concatenate([[0], np.cumsum(lens)])
    shard = lambda t, r: t[:, bounds[r]:bounds[r + 1]].contiguous()  # noqa: E731
    W = len(lens)
    sums = [seqpar.backward_local_sums(shard(q, r), shard(k, r), shard(v, r), shard(g, r)) for r in range(W)]
    a_parts = torch.stack([a for a, _ in sums])
    b_parts = torch.stack([b for _, b in sums])
    grads = [seqpar.backward_local_grads(r, W, a_parts, b_parts, shard(q, r), shard(k, r), shard(v, r), shard(g, r),
                                         sin, gs, torch.float32) for r in range(W)]
    assert la.get_device_status() == la.LA_OK
    flat = lambda t: la_inputs.bits(t.reshape(B * N, H, D))  # noqa: E731
    ref = oracle_mod.backward(flat(q), flat(k), flat(v), flat(g), _cu(B, N), state_in=to_np(sin),
                              dstate_out=to_np(gs))
    for i, name in enumerate(("dq", "dk", "dv")):
        got = torch.cat([gr[i] for gr in grads], dim=1).reshape(B * N, H, D)
        check_out(to_np(got), ref[i], bf16_out=False, what=f"ranks {name}")
    for gr in grads:
        check_state(to_np(gr[3]), ref[3], what="dS_in")


_ONE_RANK = r"""
import os, sys
sys.path.insert(0, os.environ["LA_ROOT"])
import torch, torch.distributed as dist
import la_inputs
import linear_attention_blocked_b200 as la
torch.cuda.set_device(0)
dist.init_process_group("nccl", init_method="tcp://127.0.0.1:" + os.environ["LA_PORT"], rank=0, world_size=1)
B, N, H, D = 2, 1000, 8, 128
q, k, v = la_inputs.qkv((B, N, H, D), seed=77, device="cuda")
sin = torch.randn((B, H, D, D), device="cuda") * 0.1
out, final = la.lasp_prefill(q, k, v, state_in=sin)
ref, st = la.prefill(q, k, v, state_in=sin)
torch.cuda.synchronize()
same = torch.equal(out, ref)
rel = float((final - st).norm() / st.norm())
import numpy as np
cu = la_inputs.cu_seqlens_from_lengths([700, 0, 1300])
qp, kp, vp = (t.reshape(-1, H, D)[:2000].contiguous() for t in (q, k, v))
sinp = torch.randn((3, H, D, D), device="cuda") * 0.1
outp, stp, plan = la.seqpar.lasp_prefill_varlen(qp, kp, vp, cu, np.array([0, 2000]), state_in=sinp)
refp, rstp = la.prefill_varlen(qp, kp, vp, torch.from_numpy(cu).cuda(), 1300, state_in=sinp)
same = same and torch.equal(outp, refp) and torch.equal(stp, rstp) and bool(plan.ends_here.all())
g = torch.randn_like(q.float()).mul(0.1).bfloat16()
gs = torch.randn((B, H, D, D), device="cuda") * 0.05
bw = la.lasp_prefill_backward(q, k, v, g, state_in=sin, dstate_out=gs)
bref = la.prefill_backward(q, k, v, g, state_in=sin, dstate_out=gs)
same = same and all(torch.equal(x, y) for x, y in zip(bw[:3], bref[:3]))
rel_ds = float((bw[3] - bref[3]).norm() / bref[3].norm())
dist.destroy_process_group()
print("RESULT", int(same), rel, la.get_device_status(), rel_ds)
"""


def test_lasp_prefill_under_one_rank_nccl_group():
    """With one rank the global prefix is the carried-in state itself, so the
    output must equal la_prefill's bit for bit (and the packed form's outputs
    and states those of la_prefill_varlen, the gradients dq, dk, dv those of
    la_prefill_backward); the final state of the equal-length form, and dS_in
    (la_kv_aggregate's sum here, the reversed sweep's final state there),
    differ only in summation order."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    env = dict(os.environ, LA_ROOT=ROOT, LA_PORT=str(port), NCCL_NVLS_ENABLE="0")
    res = subprocess.run([sys.executable, "-c", _ONE_RANK], env=env, capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stderr[-2000:]
    line = [x for x in res.stdout.splitlines() if x.startswith("RESULT")][-1].split()
    assert line[1] == "1", "output differs from la_prefill / la_prefill_varlen / la_prefill_backward"
    assert float(line[2]) <= 1e-5
    assert int(line[3]) == la.LA_OK
    assert float(line[4]) <= 1e-5
