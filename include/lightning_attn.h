/*
 * lightning_attn.h -- C ABI of the B200 (sm_100a) Lightning Attention library.
 *
 * Lightning Attention is blocked causal linear attention.  Per sequence and
 * head, with q_t, k_t, v_t row vectors of length d:
 *
 *     o_t = sum_{s <= t} (q_t . k_s) v_s + q_t S_in          O = (Q K^T ⊙ M) V
 *     S   = S_in + sum_s k_s^T v_s        S[i][j] = S_in[i][j] + sum_s k_s[i] v_s[j]
 *
 * computed blockwise: inside a block of rows the left product (Q_b K_b^T ⊙ M) V_b,
 * across blocks the right product Q_b S_{<b}, with the running d x d state
 * updated by S += K_b^T V_b ("MiniMax-01技术报告解读", §2.2 线性注意力: the
 * right-product kernel trick, the recursively updated KV product, intra-block
 * left product and inter-block right product over row blocks of Q/K/V).
 * No scale, feature map or normalisation is applied inside the operation:
 * callers pass q/k/v already scaled.  A per-head decay is applied only by the
 * *_decay entry points below.
 *
 * Conventions shared by every entry point
 *   - Ownership: the caller allocates and owns every buffer (inputs, outputs,
 *     states, workspace).  Only the functions that say so read host memory.
 *   - Asynchrony: device work is enqueued on `stream` and the call returns
 *     without waiting.  Nothing synchronises except la_get_device_status.
 *   - Errors: argument, shape and size errors are returned synchronously with
 *     nothing launched.  A failed launch returns LA_ERR_CUDA.  Problems found
 *     on the device (an invalid cu_seqlens array, a bounded wait that ran out)
 *     are recorded in a sticky per-device word that la_get_device_status
 *     returns; the kernels never trap and every device-side wait is bounded.
 *   - Shapes: only head dimension d = 128 is built (other d: LA_ERR_UNSUPPORTED).
 *     Every device pointer must be 16-byte aligned, the workspace 256-byte aligned.
 *   - Dtypes: q, k, v are bf16; accumulation is fp32 on the tensor cores; the
 *     output is bf16 or fp32 (la_dtype); states are fp32.
 */
#ifndef LIGHTNING_ATTN_H
#define LIGHTNING_ATTN_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define LA_API __attribute__((visibility("default")))
#else
#define LA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LA_OK = 0,
    LA_ERR_INVALID_ARGUMENT = 1, /* bad pointer, shape, alignment or dtype        */
    LA_ERR_UNSUPPORTED = 2,      /* valid but not built (d != 128, block not 0/64/128/256, decay at block 64 or 256) */
    LA_ERR_CUDA = 3,             /* a CUDA runtime call or launch failed          */
    LA_ERR_TIMEOUT = 4,          /* a bounded device-side wait ran out            */
    LA_ERR_WORKSPACE = 5         /* workspace missing or smaller than required    */
} la_status;

typedef enum { LA_BF16 = 0, LA_FP32 = 1 } la_dtype;

/* Row-block length the kernels use when `block` is 0.  Row blocks are the
 * units of the blocked algorithm; the result does not depend on the block
 * length except through rounding. */
#define LA_DEFAULT_BLOCK 128

/* ---------------------------------------------------------------------------
 * Prefill of B equal-length sequences.
 *
 *   q, k, v    device, bf16, [B, N, H, d] contiguous (token-major, heads inner).
 *   block      row-block length: 0 (= LA_DEFAULT_BLOCK) or 128.
 *   state_in   device fp32 [B, H, d, d] (row i = key feature, column j = value
 *              feature) carried-in state, or NULL for a zero state.
 *   out        device, [B, N, H, d], dtype out_dtype.
 *   state_out  device fp32 [B, H, d, d] final state, or NULL.  May be the same
 *              pointer as state_in (updated in place); any other overlap with
 *              an input or output is an error.
 *   workspace  device scratch of at least la_prefill_workspace_size(...)
 *              bytes, owned by the caller; its contents on entry do not matter
 *              and it must not be used by another call that overlaps on the GPU.
 *
 * Splits every (sequence, head) scan into segments that run on different SMs,
 * combining them with the local-prefix / gather / global-prefix recipe of
 * LASP+ ("MiniMax-01技术报告解读", §3.2 item 3) applied to SMs instead of ranks.
 * ------------------------------------------------------------------------- */
LA_API size_t la_prefill_workspace_size(int B, int N, int H, int d, int block);

LA_API la_status la_prefill(const void *q, const void *k, const void *v,
                     int B, int N, int H, int d, int block,
                     const float *state_in, void *out, la_dtype out_dtype,
                     float *state_out, void *workspace, size_t ws_bytes,
                     cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Prefill of nseq packed sequences of different lengths (data packing:
 * "MiniMax-01技术报告解读", §3.2 item 1 -- samples joined end to end along the
 * sequence; §3.2 item 4 pads each to a block of 256 in memory, which is not
 * done here: a short last block is masked in the kernel instead).
 *
 *   q, k, v      device, bf16, [total_tokens, H, d] packed.
 *   cu_seqlens   DEVICE int32 [nseq + 1]: cu_seqlens[0] = 0, non-decreasing,
 *                cu_seqlens[nseq] = total_tokens; sequence i owns tokens
 *                [cu_seqlens[i], cu_seqlens[i+1]).  Zero-length sequences are
 *                allowed.  It is checked on the device; a bad array computes
 *                nothing and records LA_ERR_INVALID_ARGUMENT in the sticky word.
 *   max_seqlen   an upper bound on every length (checked on the device too).
 *   state_in     device fp32 [nseq, H, d, d] or NULL;  state_out likewise.
 *   out          device [total_tokens, H, d], dtype out_dtype.
 *   Other arguments as for la_prefill.
 * ------------------------------------------------------------------------- */
LA_API size_t la_prefill_varlen_workspace_size(int nseq, int total_tokens, int max_seqlen,
                                        int H, int d, int block);

LA_API la_status la_prefill_varlen(const void *q, const void *k, const void *v,
                            const int *cu_seqlens, int nseq, int total_tokens,
                            int max_seqlen, int H, int d, int block,
                            const float *state_in, void *out, la_dtype out_dtype,
                            float *state_out, void *workspace, size_t ws_bytes,
                            cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * One fused decode step on a persistent fp32 state ("MiniMax-01技术报告解读",
 * §3.3 items 1-2: length-1 tokens run in their own kernel, whose KV
 * computation is fused with the update of the prefix-KV cache).
 * For every (b, h):   S <- S + k^T v,   o = q S   (the new token sees itself).
 *
 *   q, k, v   device bf16 [B, H, d].
 *   state     device fp32 [B, H, d, d], read and updated in place.
 *   out       device [B, H, d], dtype out_dtype.
 * ------------------------------------------------------------------------- */
LA_API la_status la_decode_step(const void *q, const void *k, const void *v, float *state,
                         void *out, la_dtype out_dtype, int B, int H, int d,
                         cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Per-head decay.  "MiniMax-01技术报告解读" §3.3 item 1 names a decay value
 * computation fused into the prefill but gives no formula; these entry points
 * take the reading of the TransNormer / Lightning Attention line: one constant
 * lambda_h in (0, 1] per head h and the decayed recurrence
 *
 *     S_t = lambda_h S_{t-1} + k_t^T v_t,   o_t = q_t S_t,   S_{-1} = S_in
 *   i.e.
 *     o_t = sum_{s <= t} lambda^{t-s} (q_t . k_s) v_s + lambda^{t+1} q_t S_in
 *     S   = lambda^{n} S_in + sum_s lambda^{n-1-s} k_s^T v_s     (n tokens)
 *
 * with t counted from the start of each sequence.  lambda_h = 1 on every head
 * is the undecayed operation (to rounding).  The blocked form keeps the
 * decayed keys of the state update exact to ~2^-16 (a bf16 hi + lo pair), so
 * the fp32 state meets the same error bound as without decay.
 *
 *   decay   DEVICE fp32 [H], 4-byte aligned, read only.  Checked on the device:
 *           a value outside (0, 1] (or NaN) computes nothing and records
 *           LA_ERR_INVALID_ARGUMENT in the sticky word (la_prefill_*_decay:
 *           the whole call; la_decode_step_decay: the rows of that head).
 *   block   0 or 128.  Other arguments, layouts, workspace sizes (those of
 *           la_prefill / la_prefill_varlen) and errors as without decay;
 *           decay = NULL is LA_ERR_INVALID_ARGUMENT.
 * ------------------------------------------------------------------------- */
LA_API la_status la_prefill_decay(const void *q, const void *k, const void *v,
                                  int B, int N, int H, int d, int block, const float *decay,
                                  const float *state_in, void *out, la_dtype out_dtype,
                                  float *state_out, void *workspace, size_t ws_bytes,
                                  cudaStream_t stream);

LA_API la_status la_prefill_varlen_decay(const void *q, const void *k, const void *v,
                                         const int *cu_seqlens, int nseq, int total_tokens,
                                         int max_seqlen, int H, int d, int block,
                                         const float *decay, const float *state_in, void *out,
                                         la_dtype out_dtype, float *state_out, void *workspace,
                                         size_t ws_bytes, cudaStream_t stream);

/* S <- lambda_h S + k^T v, o = q S for every (b, h); as la_decode_step otherwise. */
LA_API la_status la_decode_step_decay(const void *q, const void *k, const void *v,
                                      const float *decay, float *state, void *out,
                                      la_dtype out_dtype, int B, int H, int d,
                                      cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * State slots and the mixed prefill/decode step ("MiniMax-01技术报告解读",
 * §3.3 item 2: prefill and decode requests are served on separate CUDA
 * streams, with the length-1 tokens routed to the decode kernel; item 1: the
 * decode kernel updates the prefix-KV cache in place).
 *
 * A state pool is device fp32 [n_slots, H, d, d]: one running state per
 * request.  `slots` (DEVICE int32) maps each sequence or decode row to its
 * slot; a slot outside [0, n_slots) computes nothing for that sequence or
 * row and records LA_ERR_INVALID_ARGUMENT in the sticky device word.  Two
 * sequences or rows of one call must not name the same slot (the results
 * are then undefined; nothing checks it).
 *
 * la_prefill_varlen_slots: la_prefill_varlen where sequence i starts from
 *   state_pool[slots[i]] and leaves its final state there (in place).
 *   A zero-length sequence leaves its slot unchanged.
 * la_decode_step_slots: la_decode_step where row b updates state_pool[slots[b]].
 * la_mixed_step: one batch of requests, rows [0, prefill_tokens) of q, k, v
 *   and out packed as prefill chunks (cu_seqlens, prefill_slots), rows
 *   [prefill_tokens, prefill_tokens + n_decode) one decode token each
 *   (decode_slots).  The prefill is launched on prefill_stream and the
 *   decode on decode_stream; when the two streams differ, prefill_stream
 *   then waits (cudaStreamWaitEvent) for the decode, so work queued on
 *   prefill_stream after the call sees both results.  The workspace is the
 *   la_prefill_varlen workspace for (n_prefill, prefill_tokens).  Argument
 *   errors of either part are returned before anything is launched.
 * ------------------------------------------------------------------------- */
LA_API la_status la_prefill_varlen_slots(const void *q, const void *k, const void *v,
                                  const int *cu_seqlens, const int *slots, int nseq,
                                  int total_tokens, int max_seqlen, int H, int d, int block,
                                  float *state_pool, int n_slots, void *out,
                                  la_dtype out_dtype, void *workspace, size_t ws_bytes,
                                  cudaStream_t stream);

LA_API la_status la_decode_step_slots(const void *q, const void *k, const void *v,
                               float *state_pool, int n_slots, const int *slots, void *out,
                               la_dtype out_dtype, int B, int H, int d, cudaStream_t stream);

LA_API la_status la_mixed_step(const void *q, const void *k, const void *v,
                        const int *cu_seqlens, const int *prefill_slots, int n_prefill,
                        int prefill_tokens, int max_seqlen, const int *decode_slots,
                        int n_decode, int H, int d, float *state_pool, int n_slots, void *out,
                        la_dtype out_dtype, void *workspace, size_t ws_bytes,
                        cudaStream_t prefill_stream, cudaStream_t decode_stream);

/* ---------------------------------------------------------------------------
 * Prefill of inputs that live in pinned host memory.  When q, k, v are on the
 * host the host link, not the kernel, sets the pace (at B=1, H=64, N=32768:
 * 1.61 GB in and 0.54 GB out, tens of milliseconds against half a
 * millisecond of compute), so the sequence is cut into chunks of
 * chunk_tokens tokens pipelined over three streams: chunk c+1 is copied in
 * on copy_in while chunk c is scanned on compute and chunk c-1 is copied out
 * on copy_out.  Each chunk is an la_prefill from the state the previous
 * chunk left.  This is the state-carry identity of the recurrent form
 * ("MiniMax-01技术报告解读", §2.2 线性注意力: the running KV state summarises
 * every earlier token), so the result equals one prefill of the whole
 * sequence, to rounding.
 *
 *   q, k, v     PINNED HOST bf16 [B, N, H, d] (cudaHostAlloc / registered).
 *   out         PINNED HOST [B, N, H, d] in out_dtype.
 *   state_in    device fp32 [B, H, d, d] or NULL (zero state).
 *   state_out   fp32 [B, H, d, d], device or pinned host, or NULL.
 *   buffers     device scratch of la_prefill_from_host_buffer_size(B,
 *               chunk_tokens, H, d, out_dtype) bytes, 256-byte aligned,
 *               caller-owned: two chunk slots of q, k, v and out, the
 *               running state and a prefill workspace.
 *   copy_in, compute, copy_out   three streams (may be the same stream, which
 *               serialises the pipeline).  The copy streams first wait for the
 *               work already queued on compute; on return, work queued on
 *               compute after the call sees every result (outputs copied out,
 *               state_out written).  Nothing is synchronised; the host buffers
 *               must stay valid until compute reaches that point.
 * Errors before any work is queued: argument and shape errors, a host buffer
 * that is not pinned (LA_ERR_INVALID_ARGUMENT), a short buffer
 * (LA_ERR_WORKSPACE).  The call keeps a few CUDA events per host thread
 * (created on its first call, reused afterwards) and allocates no memory.
 * ------------------------------------------------------------------------- */
LA_API size_t la_prefill_from_host_buffer_size(int B, int chunk_tokens, int H, int d, la_dtype out_dtype);

LA_API la_status la_prefill_from_host(const void *q, const void *k, const void *v,
                                      int B, int N, int H, int d, int chunk_tokens,
                                      const float *state_in, void *out, la_dtype out_dtype,
                                      float *state_out, void *buffers, size_t buffer_bytes,
                                      cudaStream_t copy_in, cudaStream_t compute,
                                      cudaStream_t copy_out);

/* ---------------------------------------------------------------------------
 * la_prefill without a workspace argument, for callers that cannot allocate
 * device memory when they call: e.g. a plugin inside a host framework that
 * owns the allocator and offers no allocation hook, or a serving process that
 * reserved all device memory up front and forbids cudaMalloc (a slow call
 * that may synchronise the device) on its request path.  This entry point has
 * no counterpart on the pages; it is a convenience of this library.
 *
 * Arguments, layouts and results are those of la_prefill minus the workspace.
 * Scratch is a fixed 32 MiB array inside the library, reserved on every GPU
 * the process uses from library load until exit; the call allocates and frees
 * nothing.  To fit, it may use longer cross-SM segments than la_prefill
 * (changing only speed and rounding).  A problem whose scratch needs exceed
 * 32 MiB even with one segment per sequence -- B * H above 511 (sequence,
 * head) pairs -- is rejected with LA_ERR_WORKSPACE before any launch.  The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call before
 * any stream capture.  Every call uses the same array and the kernels reset
 * the parts that must start at zero, so leftover contents do not matter, but
 * calls that overlap on the GPU (other streams, other host threads) race on
 * it: serialise them.
 * ------------------------------------------------------------------------- */
LA_API la_status la_prefill_noalloc(const void *q, const void *k, const void *v,
                                    int B, int N, int H, int d, int block,
                                    const float *state_in, void *out, la_dtype out_dtype,
                                    float *state_out, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Sequence parallelism across ranks ("MiniMax-01技术报告解读", §3.2 item 3,
 * LASP+: each rank forms the local prefix of its part of the sequence, the
 * local prefixes are all-gathered, and each rank adds up the global prefix
 * of the ranks before it, then runs its own blocked scan from there).
 * Rank r holds tokens [n_0 + ... + n_{r-1}, + n_r) of every sequence of the
 * batch.  Per rank:
 *
 *   la_kv_aggregate(k_r, v_r) -> A_r           (local prefix, this library)
 *   AllGather(A_r) -> A_0 ... A_{W-1}          (the caller's collective)
 *   la_state_prefix(A, r, S_in) -> P_r         (global prefix, this library)
 *   la_prefill(q_r, k_r, v_r, state_in = P_r)  (the local scan)
 *
 * and la_state_prefix(A, W, S_in) is the final state of the whole sequence.
 * The rank's outputs equal the rows of the single-GPU result for its tokens.
 *
 * la_kv_aggregate: A[b][h][i][j] = sum_t k[b][t][h][i] * v[b][t][h][j] over
 *   the N tokens of each sequence (the state increment S_out - S_in of a
 *   prefill of those tokens).  k, v: bf16 [B, N, H, d] contiguous (read
 *   only; may be NULL when N == 0).  agg: fp32 [B, H, d, d] row-major, fully
 *   written (zeros when N == 0), must not overlap k, v or the workspace.
 *   workspace: at least la_kv_aggregate_workspace_size(B, N, H, d) bytes
 *   (at most 2 x 148 x 64 KiB), 16-byte aligned, caller-owned scratch whose
 *   contents before and after the call do not matter; may be NULL when the
 *   size is 0.  fp32 accumulation on the tensor cores, summed in a fixed
 *   order (the result does not depend on timing).  Asynchronous on `stream`;
 *   argument errors are returned before any launch; a device-side wait that
 *   ran out is reported by la_get_device_status.
 * la_state_prefix: out = (state_in or 0) + parts[0] + ... + parts[count-1],
 *   elementwise in that order, in fp32.  parts: fp32 [count][nstates][d][d]
 *   contiguous (NULL when count == 0); state_in: fp32 [nstates][d][d] or
 *   NULL; out: fp32 [nstates][d][d], may equal state_in, must not overlap
 *   parts or partially overlap state_in.  nstates = B * H.  Asynchronous on
 *   `stream`.  With count == 0 it copies state_in into out (or zeroes out).
 * Errors of both, returned before any launch: d != 128 -> LA_ERR_UNSUPPORTED;
 * a negative size or count, a needed pointer that is NULL or not 16-byte
 * aligned, or overlapping buffers -> LA_ERR_INVALID_ARGUMENT; a missing or
 * short workspace -> LA_ERR_WORKSPACE.
 * ------------------------------------------------------------------------- */
LA_API size_t la_kv_aggregate_workspace_size(int B, int N, int H, int d);

LA_API la_status la_kv_aggregate(const void *k, const void *v, int B, int N, int H, int d,
                                 float *agg, void *workspace, size_t ws_bytes,
                                 cudaStream_t stream);

LA_API la_status la_state_prefix(const float *parts, int count, const float *state_in,
                                 float *out, int nstates, int d, cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Gradients of la_prefill.  The pages train the model with LASP+
 * ("MiniMax-01技术报告解读", §3.2 item 3) but give no backward formulas; these
 * are the derivatives of the forward definition at the top of this file for
 * a loss L with dL/do_t = g_t (dout) and dL/dS_out = G (dstate_out):
 *
 *   dq_t  = sum_{s <= t} (g_t . v_s) k_s + g_t S_in^T
 *   dk_s  = sum_{t >= s} (g_t . v_s) q_t + v_s G^T
 *   dv_s  = sum_{t >= s} (q_t . k_s) g_t + k_s G
 *   dS_in = sum_t q_t^T g_t + G
 *
 * computed as two blocked sweeps: dq is a forward sweep of (dout, v, k)
 * from S_in^T; dv and dk, sums over the later tokens, are one reversed sweep
 * (segments and row blocks from the end of each sequence, the mask keeping
 * t >= s) of the paired problems (k, q, dout) and (v, dout, q) from G,
 * whose final state is dS_in.
 *
 * q, k, v, dout: bf16 [B, N, H, d] contiguous (read only).  state_in,
 * dstate_out: fp32 [B, H, d, d] row-major or NULL (= 0).  dq, dk, dv: [B, N,
 * H, d] in grad_dtype (bf16 or fp32), fully written; they must not overlap
 * each other, the inputs, the states or the workspace.  dstate_in: fp32
 * [B, H, d, d] or NULL (not computed).  workspace: at least
 * la_prefill_backward_workspace_size(B, N, H, d) bytes, 256-byte aligned,
 * caller-owned scratch.  fp32 accumulation on the tensor cores.  Enqueues
 * four kernels (five with a state_in) on `stream` and returns; argument
 * errors are
 * returned before any launch; device-side problems are reported by
 * la_get_device_status.
 * ------------------------------------------------------------------------- */
LA_API size_t la_prefill_backward_workspace_size(int B, int N, int H, int d);

LA_API la_status la_prefill_backward(const void *q, const void *k, const void *v,
                                     const void *dout, int B, int N, int H, int d,
                                     const float *state_in, const float *dstate_out,
                                     void *dq, void *dk, void *dv, la_dtype grad_dtype,
                                     float *dstate_in, void *workspace, size_t ws_bytes,
                                     cudaStream_t stream);

/* la_prefill_backward_varlen: the gradients of la_prefill_varlen -- the
 * same derivatives for every sequence of a packed batch (the pages train on
 * packed sequences: "MiniMax-01技术报告解读" §3.2 item 1).  q, k, v, dout,
 * dq, dk, dv: [total_tokens, H, d]; cu_seqlens: device int32 [nseq + 1],
 * validated on the device as for la_prefill_varlen (an invalid table sets
 * LA_ERR_INVALID_ARGUMENT in the device word and computes nothing);
 * state_in, dstate_out, dstate_in: fp32 [nseq, H, d, d] or NULL.  The
 * gradients of an empty sequence are empty and its dS_in is its dS_out.
 * Workspace: la_prefill_backward_varlen_workspace_size bytes, 256-byte
 * aligned.  Otherwise as la_prefill_backward. */
LA_API size_t la_prefill_backward_varlen_workspace_size(int nseq, int total_tokens, int max_seqlen,
                                                        int H, int d);

LA_API la_status la_prefill_backward_varlen(const void *q, const void *k, const void *v,
                                            const void *dout, const int *cu_seqlens, int nseq,
                                            int total_tokens, int max_seqlen, int H, int d,
                                            const float *state_in, const float *dstate_out,
                                            void *dq, void *dk, void *dv, la_dtype grad_dtype,
                                            float *dstate_in, void *workspace, size_t ws_bytes,
                                            cudaStream_t stream);

/* ---------------------------------------------------------------------------
 * Status.
 * la_get_device_status synchronises `stream`, then returns and clears the
 * sticky device word of the current device (LA_ERR_TIMEOUT,
 * LA_ERR_INVALID_ARGUMENT from a device-side check), or LA_ERR_CUDA when the
 * synchronisation itself reports an error.  LA_OK when nothing was recorded.
 * ------------------------------------------------------------------------- */
LA_API la_status la_get_device_status(cudaStream_t stream);

/* Static English text for a status code (never NULL). */
LA_API const char *la_status_string(la_status status);

/* ---------------------------------------------------------------------------
 * Controls and diagnostics (process-wide, host side; not thread-safe against
 * concurrent launches).
 *
 * la_set_wait_limit_ns: upper bound for every device-side wait (mbarrier
 *   phases, the cross-SM segment hand-off).  Default 2e9 ns.  A wait that runs
 *   out records LA_ERR_TIMEOUT and the kernel finishes without hanging.
 *   0 restores the default.
 * la_set_segment_len: tokens per segment of the cross-SM scan; 0 = automatic,
 *   otherwise a positive multiple of 128.  Changes only speed and rounding.
 * la_debug_inject: fault injection made on the host side, for tests.
 *   LA_INJECT_NONE (0): normal operation.
 *   LA_INJECT_SKIP_PUBLISH (1): segments never publish their prefix, so every
 *   segment with a predecessor waits until the limit runs out; outputs are
 *   then meaningless and la_get_device_status returns LA_ERR_TIMEOUT.
 * la_last_segment_len: the segment length the last prefill launch used.
 * la_kernel_launches: cumulative number of kernels this library has
 *   launched in this process (all entry points), for launch accounting.
 * ------------------------------------------------------------------------- */
#define LA_INJECT_NONE 0
#define LA_INJECT_SKIP_PUBLISH 1

LA_API la_status la_set_wait_limit_ns(unsigned long long ns);
LA_API la_status la_set_segment_len(int tokens);
LA_API la_status la_debug_inject(int mode);
LA_API int la_last_segment_len(void);
LA_API unsigned long long la_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* LIGHTNING_ATTN_H */
