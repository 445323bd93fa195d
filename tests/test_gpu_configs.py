"""GPU parity at the full sizes of the five target workloads, through the C ABI,
against the fp64 oracle on the same seeded inputs.

  1. prefill B=1 H=2 N=1024, fp32 out         -> every output (test_gpu_prefill.py)
  2. prefill B=1 H=64 N=32768, bf16 out+state -> every output and state, all 64 heads
  3. packed varlen, 8 sequences U[1024, 65536], H=64, bf16 out
                                              -> every output of 16 of the 64 heads
  4. prefill B=1 H=8 N=1048576                -> bf16 run: 2 heads; fp32 run: 2 heads
  5. decode 256 seqs x 64 heads from a 4096-token prefill, 1024 steps
                                              -> 32 seeded (seq, head) pairs, every step
"""
import numpy as np
import pytest
import torch

import la_inputs
import linear_attention_blocked_b200 as la
from parity_util import check_out, check_state, to_np

pytestmark = pytest.mark.gpu

D = 128


def _bits(t):
    return la_inputs.bits(t)


def test_config2_prefill_32k_all_heads(oracle_mod):
    B, N, H = 1, 32768, 64
    q, k, v = la_inputs.qkv((B, N, H, D), seed=20250101, device="cuda")
    out, st = la.prefill(q, k, v, out_dtype=torch.bfloat16)
    assert la.get_device_status() == la.LA_OK
    ref, rst = oracle_mod.recurrent(_bits(q[0]), _bits(k[0]), _bits(v[0]), np.array([0, N], np.int32))
    check_out(to_np(out[0]), ref, bf16_out=True, what="config 2 outputs")
    check_state(to_np(st[0]), rst[0], what="config 2 final states")


def test_config3_varlen_packed(oracle_mod):
    H = 64
    lens = la_inputs.varlen_lengths(8, 1024, 65536, seed=3)
    cu = la_inputs.cu_seqlens_from_lengths(lens)
    T = int(cu[-1])
    q, k, v = la_inputs.qkv((T, H, D), seed=303, device="cuda")
    out, st = la.prefill_varlen(q, k, v, torch.from_numpy(cu).cuda(), int(lens.max()), out_dtype=torch.bfloat16)
    assert la.get_device_status() == la.LA_OK
    heads = np.random.default_rng(33).choice(H, 16, replace=False).astype(np.int32)
    hsel = torch.from_numpy(heads.astype(np.int64)).cuda()
    ref, rst = oracle_mod.recurrent(_bits(q), _bits(k), _bits(v), cu, heads=heads)
    check_out(to_np(out[:, hsel]), ref, bf16_out=True, what="config 3 outputs (16 heads)")
    check_state(to_np(st[:, hsel]), rst, what="config 3 final states (16 heads)")


def test_config4_one_million_tokens(oracle_mod):
    B, N, H = 1, 1048576, 8
    q, k, v = la_inputs.qkv((B, N, H, D), seed=404, device="cuda")
    hsel = torch.tensor([0, 5], device="cuda")
    ref, rst = oracle_mod.recurrent(_bits(q[0][:, hsel]), _bits(k[0][:, hsel]), _bits(v[0][:, hsel]),
                                    np.array([0, N], np.int32))
    for dtype in (torch.bfloat16, torch.float32):
        out, st = la.prefill(q, k, v, out_dtype=dtype)
        assert la.get_device_status() == la.LA_OK
        check_out(to_np(out[0][:, hsel]), ref, bf16_out=dtype == torch.bfloat16, what=f"config 4 outputs ({dtype})")
        check_state(to_np(st[0][hsel]), rst[0], what="config 4 states")
        del out, st
        torch.cuda.empty_cache()


def test_config5_batched_decode(oracle_mod):
    S, H, NP, STEPS = 256, 64, 4096, 1024
    rng = np.random.default_rng(55)
    pairs = [(int(s), int(h)) for s, h in zip(rng.choice(S, 32, replace=False), rng.integers(0, H, 32))]
    state = torch.empty((S, H, D, D), dtype=torch.float32, device="cuda")
    chunk = 32
    pq = []
    for s0 in range(0, S, chunk):
        qp, kp, vp = la_inputs.qkv((chunk, NP, H, D), seed=5000 + s0, device="cuda")
        la.prefill(qp, kp, vp, state_out=state[s0:s0 + chunk])
        for (s, h) in pairs:
            if s0 <= s < s0 + chunk:
                pq.append((s, h, _bits(qp[s - s0, :, h]), _bits(kp[s - s0, :, h]), _bits(vp[s - s0, :, h])))
        del qp, kp, vp
    assert la.get_device_status() == la.LA_OK
    pq.sort(key=lambda e: pairs.index((e[0], e[1])))
    # oracle states after the prefill, one (seq, head) pair per "sequence" of length NP
    Qp = np.stack([e[2] for e in pq], 0).reshape(-1, 1, D)
    Kp = np.stack([e[3] for e in pq], 0).reshape(-1, 1, D)
    Vp = np.stack([e[4] for e in pq], 0).reshape(-1, 1, D)
    cu = la_inputs.cu_seqlens_from_lengths([NP] * len(pairs))
    _, rstate = oracle_mod.recurrent(Qp, Kp, Vp, cu)          # [32, 1, D, D]
    ref_state = rstate[:, 0][None]                               # [1, 32, D, D]
    ss = torch.tensor([p[0] for p in pairs], device="cuda")
    hs = torch.tensor([p[1] for p in pairs], device="cuda")
    check_state(to_np(state[ss, hs]), ref_state[0], what="state after 4096-token prefill")
    out = torch.empty((S, H, D), dtype=torch.bfloat16, device="cuda")
    for step in range(STEPS):
        q, k, v = la_inputs.qkv((S, H, D), la_inputs.decode_seed(55, step), device="cuda")
        la.decode_step(q, k, v, state, out=out)
        ro, ref_state = oracle_mod.decode_step(_bits(q[ss, hs])[None], _bits(k[ss, hs])[None],
                                               _bits(v[ss, hs])[None], ref_state)
        check_out(to_np(out[ss, hs]), ro[0], bf16_out=True, what=f"decode step {step}")
    assert la.get_device_status() == la.LA_OK
    check_state(to_np(state[ss, hs]), ref_state[0], what="state after 1024 decode steps")
