"""Lightning Attention (blocked causal linear attention) for NVIDIA B200.

The computation runs in the in-tree CUDA library (sm_100a, tcgen05/TMEM
tensor-core MMAs, TMA-staged tiles); this package is the Python face of its C
ABI (include/lightning_attn.h).  Entry points:

  prefill(q, k, v, ...)                      la_prefill          [B, N, H, 128]
  prefill_varlen(q, k, v, cu_seqlens, ...)   la_prefill_varlen   [T, H, 128] packed
  decode_step(q, k, v, state, ...)           la_decode_step      [B, H, 128]
                                             (each of the three with decay=<fp32 [H] on the
                                             device>: la_*_decay, per-head decay lambda_h)
  prefill_varlen_slots / decode_step_slots   the same on a pool of per-request states
  mixed_step(q, k, v, cu_seqlens, ...)       la_mixed_step: prefill chunks and decode tokens
                                             of one batch on two streams (plan with
                                             serving.plan_batch)
  kv_aggregate(k, v)                         la_kv_aggregate: sum_t k_t^T v_t per (sequence, head)
  state_prefix(parts, count, state_in)       la_state_prefix: state_in + parts[0] + ... + parts[count-1]
  lasp_prefill(q, k, v, group=...)           sequence parallelism across ranks (seqpar.py)
  lasp_prefill_varlen(q, k, v, cu, bounds)   the same for a packed batch cut at any token
  lasp_prefill_backward(q, k, v, dout, ...)  gradients of lasp_prefill across ranks
  lasp_prefill_backward_varlen(...)          gradients of lasp_prefill_varlen across ranks
  prefill_backward(q, k, v, dout, ...)       la_prefill_backward: dq, dk, dv, dS_in
  prefill_backward_varlen(q, k, v, dout, cu, ...)  la_prefill_backward_varlen: the same per packed sequence
  prefill_from_host(q, k, v, ...)            la_prefill of pinned host tensors, chunks pipelined
                                             over copy-in / scan / copy-out streams
  get_device_status()                        la_get_device_status
"""
from ._binding import (D, DEFAULT_BLOCK, backward_workspace_size, backward_varlen_workspace_size,  # noqa: F401
                       prefill_backward, prefill_backward_varlen, EXPORTED, LA_BF16, LA_ERR_CUDA,
                       LA_ERR_INVALID_ARGUMENT, LA_ERR_TIMEOUT, LA_ERR_UNSUPPORTED,
                       LA_ERR_WORKSPACE, LA_FP32, LA_INJECT_NONE, LA_INJECT_SKIP_PUBLISH, LA_OK,
                       LAError, debug_inject, decode_step, decode_step_slots, get_device_status,
                       kernel_launches, kv_aggregate, last_segment_len, lib, library_path, mixed_step,
                       prefill, prefill_varlen, prefill_varlen_slots,
                       set_segment_len, set_wait_limit_ns, state_prefix, status_string,
                       varlen_workspace_size, workspace_size)
from .seqpar import (lasp_prefill, lasp_prefill_backward, lasp_prefill_backward_varlen,  # noqa: F401,E402
                     lasp_prefill_varlen, plan_varlen_rank,
                     split_tokens)
from .serving import BatchPlan, plan_batch  # noqa: F401,E402
from .streaming import make_buffers, prefill_from_host  # noqa: F401,E402
