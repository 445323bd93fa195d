"""GPU parity of prefill_from_host (pinned host inputs, chunks of tokens
pipelined over copy-in, scan and copy-out streams, the state carried from
chunk to chunk) against the fp64 oracle's prefill of the whole sequences."""
import numpy as np
import pytest
import torch

import la_inputs
import linear_attention_blocked_b200 as la
from parity_util import check_out, check_state, to_np

pytestmark = pytest.mark.gpu

D = 128


def _host(shape, seed):
    return [t.cpu().pin_memory() for t in la_inputs.qkv(shape, seed=seed)]


@pytest.mark.parametrize("B,N,H,chunk,dtype", [(2, 3000, 4, 1024, torch.float32), (1, 5000, 8, 4096, torch.bfloat16),
                                               (3, 700, 2, 256, torch.float32), (1, 128, 2, 4096, torch.float32)])
def test_prefill_from_host_matches_oracle(oracle_mod, B, N, H, chunk, dtype):
    q, k, v = _host((B, N, H, D), seed=1200 + N)
    gen = torch.Generator(device="cuda").manual_seed(1201)
    sin = torch.randn((B, H, D, D), generator=gen, device="cuda") * 0.1
    out, st = la.prefill_from_host(q, k, v, chunk_tokens=chunk, state_in=sin, out_dtype=dtype)
    torch.cuda.synchronize()
    assert la.get_device_status() == la.LA_OK
    assert not out.is_cuda and out.dtype == dtype
    cu = (np.arange(B + 1) * N).astype(np.int32)
    flat = lambda t: la_inputs.bits(t.reshape(B * N, H, D))  # noqa: E731
    ref, rst = oracle_mod.recurrent(flat(q), flat(k), flat(v), cu, state_in=to_np(sin))
    check_out(to_np(out).reshape(B * N, H, D), ref, bf16_out=dtype == torch.bfloat16, what="streamed outputs")
    check_state(to_np(st), rst, what="final state")


def test_prefill_from_host_reuses_buffers_and_host_state():
    """Buffers made once serve repeated calls; the final state can land in
    pinned host memory; a call with no tokens returns the carried-in state."""
    B, N, H = 1, 2500, 4
    q, k, v = _host((B, N, H, D), seed=1210)
    bufs = la.make_buffers(B, 1024, H)
    sh = torch.empty((B, H, D, D), dtype=torch.float32, pin_memory=True)
    o1, _ = la.prefill_from_host(q, k, v, chunk_tokens=1024, buffers=bufs, state_out=sh)
    torch.cuda.synchronize()
    s1 = sh.clone()
    o2, s2 = la.prefill_from_host(q, k, v, chunk_tokens=1024, buffers=bufs)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(s1, s2.cpu())
    e = torch.empty((B, 0, H, D), dtype=torch.bfloat16).pin_memory()
    sin = torch.randn((B, H, D, D), device="cuda")
    o3, s3 = la.prefill_from_host(e, e, e, state_in=sin)
    torch.cuda.synchronize()
    assert o3.shape == (B, 0, H, D) and torch.equal(s3, sin)
    assert la.get_device_status() == la.LA_OK
