"""la_prefill_noalloc: the prefill entry point for callers that cannot allocate
device memory (a plugin whose host framework owns the allocator, a server
that reserved all GPU memory up front and forbids cudaMalloc on its request
path).  It uses a fixed scratch array inside the library instead of a
caller-provided workspace.  Called here through the C ABI (ctypes) and
compared with la_prefill on the same inputs, two calls in a row, with the
tolerances of the other parity tests.  This file is collected last on purpose."""
import ctypes

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


@pytest.mark.parametrize("shape", [(2, 1500, 4), (1, 32768, 64)])
def test_noalloc_matches_prefill_twice(shape):
    la.set_segment_len(0)
    B, N, H = shape
    for call in range(2):                     # two calls in a row share the scratch
        q, k, v = la_inputs.qkv((B, N, H, D), seed=700 + call, device="cuda")
        gen = torch.Generator(device="cuda").manual_seed(800 + call)
        s_in = torch.randn((B, H, D, D), generator=gen, device="cuda") * 0.1
        ref_out, ref_st = la.prefill(q, k, v, state_in=s_in, out_dtype=torch.float32)
        out = torch.empty((B, N, H, D), dtype=torch.float32, device="cuda")
        st = torch.empty((B, H, D, D), dtype=torch.float32, device="cuda")
        assert _noalloc(q, k, v, out, st, s_in) == la.LA_OK
        assert la.get_device_status() == la.LA_OK
        check_out(to_np(out), to_np(ref_out), bf16_out=False, what=f"call {call}")
        check_state(to_np(st), to_np(ref_st), what=f"call {call}")


def test_noalloc_rejects_problems_beyond_its_scratch():
    B, N, H = 8, 128, 64                      # 512 (sequence, head) pairs: needs > 32 MiB
    q, k, v = la_inputs.qkv((B, N, H, D), seed=9, device="cuda")
    out = torch.full((B, N, H, D), 3.0, dtype=torch.float32, device="cuda")
    st = torch.zeros((B, H, D, D), dtype=torch.float32, device="cuda")
    assert _noalloc(q, k, v, out, st) == la.LA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(out == 3.0)              # nothing was launched
    assert la.get_device_status() == la.LA_OK
