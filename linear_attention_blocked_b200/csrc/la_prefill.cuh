// la_prefill.cuh -- blocked causal linear attention prefill for sm_100a.
//
// What one CTA does ("MiniMax-01技术报告解读", §2.2 线性注意力; §3.2 item 3 LASP+):
// the token range of every (sequence, head) is cut into segments of
// `seg_len` tokens; a work item is one (segment, head).  CTAs are persistent
// and take items in ticket order from a device counter.  For an item
//
//   phase A (only if a later segment of the same sequence exists):
//       local KV sum  A_j = sum_b K_b^T V_b    (tcgen05, fp32, in an O buffer)
//   phase L (look-back, LASP+ "gather + global prefix" on SMs instead of ranks):
//       E_j = state_in (j = 0)  or  INCL_{j-1} published by the item that
//       owns segment j-1 (bounded spin on its flag);  INCL_j = E_j + A_j is
//       published for segment j+1.
//   phase O (blocked scan over the segment's row blocks, starting from E_j):
//       Sc  = Q_b K_b^T                    a2   (SS MMA, M=N=128, K=d)
//       P   = bf16(Sc ⊙ M), inclusive mask a3   (TMEM -> regs -> TMEM)
//       O   = Q_b S_{<b}                   a5   (S as one bf16 term, or as
//                                               bf16 hi + lo for long sequences)
//       O  += P V_b                        a4   (TS MMA, P read from TMEM)
//       S  += K_b^T V_b                    a6   (SS MMA, both MN-major)
//       out = O (bf16 or fp32)             a7
//   and, for the last segment, the final state S goes to state_out.
//
// The kernel is a template.  DECAY adds a per-head decay lambda_h in (0, 1]
// (the "decay value computation" of "MiniMax-01技术报告解读" §3.3 item 1, read
// as the decayed recurrence S_t = lambda S_{t-1} + k_t^T v_t, o_t = q_t S_t).
// With r the row in a block of nb rows:
//       P[r][c] = bf16(Sc[r][c] lambda^{r-c})           a3 (decay in the mask)
//       O       = P V + lambda^{r+1} Q S_{<b}           a4 into O buffer 0, a5 into
//                                                       buffer 1, combined by the
//                                                       store warps in fp32
//       S      <- lambda^{nb} S + (Lambda K)^T V        a6, Lambda = lambda^{nb-1-r}
//       A_j     = sum_b (Lambda_b K_b)^T V_b            phase A, rows scaled to the
//                                                       segment end
//       INCL_j  = lambda^{len_j} E_j + A_j              phase L
// The row-scaled keys Lambda K are split into a bf16 pair hi + lo (x = hi +
// lo to within 2^-16 |x|), so the state sees the decayed keys as exactly as
// the undecayed state sees the raw ones: hi is written over the K tile once
// the scores have read it, lo into the block's Q slot once a5 has read it (in
// phase A: into the snapshot buffer, idle there), and a6 is the two products
// hi^T V + lo^T V.  The state warps rescale S by lambda^{nb} in TMEM when they
// take each snapshot.
//
// REV makes the sweep run backwards: the scheduler lists each sequence's
// segments from its end, every item visits its row blocks from the last, and
// the mask keeps key t for row s iff t >= s, so from a state S_0 passed as
// state_in
//       o_s = q_s (S_0 + sum_{t >= s} k_t^T v_t)
// with the final state S_0 + sum_t k_t^T v_t -- sums over later tokens from
// a sweep that adds.
//
// PAIR (with REV) runs two problems that share their keys, values and state
// in one sweep: problem 1 is (q, k, v) and problem 2 is (q2, v, k), whose
// state sum v^T k is the transpose of problem 1's.  Each row block b becomes
// two sub-blocks, u = 2b (problem 1) and u = 2b + 1 (problem 2), which take
// turns in the score buffer, in the Q ring (q tile, then q2 tile) and in the
// two O buffers (sub-block u in buffer u & 1; problem 1 writes `out`, problem
// 2 `out2`).  a5 of problem 2 reads the same state snapshot through K-major
// descriptors, which present it transposed (with S as hi + lo, the snapshot
// holds one column half at a time, and both problems read each half before
// it is released); a6 runs once per block.  With (q, k, v, q2) = (K, Q, dO,
// V) the two outputs are the gradients dV and dK, Q and dO are read once for
// both, and the final state is dS_in.
//
// Warp roles (448 threads):
//   warp 0      TMA producers: lane 0 takes tickets and loads K and V, lane 1
//               loads Q
//   warp 1      TMEM allocator + MMA issuer (the whole warp runs the schedule;
//               elect.sync picks the lane that issues each MMA or commit)
//   warps 2-5   causal mask (a3)
//   warps 6-9   output store (a7) and the flag that publishes INCL_j
//   warps 10-13 segment hand-off (phase L), state snapshots for a5, final state
// A warp may only touch the 32 TMEM lanes of its quarter (warp % 4), so each
// group of four covers all 128 rows.  Every group has its own chain of TMEM
// loads and barrier arrivals, so the mask of block b+1, the output of block b
// and the state snapshot for block b+1 proceed independently.
//
// Shared memory (1024-byte aligned, 128-byte swizzle everywhere):
//   K ring 2 x 32 KiB | V ring 2 x 32 KiB | Q ring 2 x 32 KiB | S snapshot
//   2 x 16 KiB | barriers + item queue.
// A [128 x 128] bf16 tile is two 16 KiB halves (columns 0-63, 64-127), each
// 128 rows of 128 bytes, written by one TMA box {64, 1, 128, 2} of the 4-D
// view {64, H, T, 2} of the [T, H, 128] tensor (the halves are its outer
// dimension).
// TMEM (512 columns x 128 lanes x 32 bit): Sc [0,128) (scores; P overwrites
//   the first 64 columns in place) | O0 [128,256) | O1 [256,384) (block b
//   accumulates in O_{b&1}, so O of block b is read out while b+1 runs) |
//   S [384,512).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include "la_ptx.cuh"
#include "lightning_attn.h"

namespace la {

constexpr int D = 128;                      // head dimension (d_k = d_v)
constexpr int BLK = 128;                    // rows per block (= MMA M)
constexpr int HALF_BYTES = BLK * 128;       // [128 rows x 64 bf16]
constexpr int TILE_BYTES = 2 * HALF_BYTES;  // [128 x 128] bf16
constexpr int KV_STAGES = 2;
constexpr int Q_STAGES = 2;
constexpr int PREFILL_THREADS = 448;
constexpr int W_MASK = 2, W_STORE = 6, W_STATE = 10;  // first warp of each four-warp group

// L2 prefetch distance of the Q tiles, in row blocks ahead of their
// shared-memory loads.  Q is the one tile phase O reads from DRAM (K and V
// come back from L2 after phase A); prefetching it two or four blocks ahead
// measured slower, so the default is 0 (off).
#ifndef LA_PREFETCH_Q
#define LA_PREFETCH_Q 0
#endif
constexpr int PF_Q = LA_PREFETCH_Q;

// The scores a2(b+1) are issued only after a4(b): they fill the gap while
// the tensor pipe waits on the next a5 instead of delaying it, and, since the
// pipe runs MMAs in issue order, a4(b) has read P(b) before a2(b+1)
// overwrites the score buffer -- one score buffer suffices, which leaves the
// TMEM for two O buffers.

constexpr int SM_K = 0;
constexpr int SM_V = SM_K + KV_STAGES * TILE_BYTES;
constexpr int SM_Q = SM_V + KV_STAGES * TILE_BYTES;
constexpr int SM_SHI = SM_Q + Q_STAGES * TILE_BYTES;  // S snapshot: bf16 hi of one half, or columns 0-63
constexpr int SM_SLO = SM_SHI + HALF_BYTES;           // ... bf16 lo residual of that half, or columns 64-127
constexpr int SM_CTRL = SM_SLO + HALF_BYTES;          // 229376
constexpr int SM_CTRL_BYTES = 1024;
constexpr int PREFILL_SMEM = SM_CTRL + SM_CTRL_BYTES + 1024;  // + alignment slack

constexpr uint32_t TM_SC = 0, TM_O = 128, TM_S = 384, TM_COLS = 512;  // O buffer 1 = TM_O + 128

// device status codes (match la_status)
constexpr int ST_INVALID = 1;
constexpr int ST_TIMEOUT = 4;

// workspace header words
constexpr int HDR_TOTAL = 0;   // number of work items (G * H)
constexpr int HDR_TICKET = 1;  // ticket counter
constexpr int HDR_G = 2;       // number of segments
constexpr int HDR_BYTES = 256;

constexpr int SEG_LAST = 1 << 30;  // flag bit in SegInfo::jinfo

struct PrefillParams {
    const float *state_in;  // [nseq, H, D, D] or null (or a pool of states, see slots)
    float *state_out;       // [nseq, H, D, D] or null (or a pool of states, see slots)
    const int *slots;       // null, or [nseq]: sequence i reads and writes state slots[i]
    void *out;              // [T, H, D]
    void *out2;             // PAIR: [T, H, D], the second problem's output (same dtype)
    int out_fp32;
    int out_al32;           // out is 32-byte aligned: rows are written with 32-byte stores
    int H;
    int *hdr;               // workspace header
    const int4 *segs;       // [G] {seq, tok0, tok1, jinfo}
    int *flags;             // [G*H] 0 = empty, 2 = inclusive prefix published
    float *incl;            // [G*H][D*D] inclusive prefixes, column-quad interleaved
    int seg_len;            // tokens per segment (the last one of a sequence may be shorter)
    unsigned long long wait_limit_ns;
    int inject;
    const float *decay;     // DECAY: lambda_h per head, [H] (validated by the scheduler)
    int *status;            // sticky device status word
};

// mbarriers (arrival counts in brackets)
struct CtrlBlock {
    uint64_t kv_full[KV_STAGES];  // [1] producer expect_tx
    uint64_t kv_empty[KV_STAGES]; // [1] MMA commit after the last MMA reading the stage
    uint64_t q_full[Q_STAGES];    // [1] producer expect_tx
    uint64_t q_empty[Q_STAGES];   // [1] MMA commit after a5 of the block
    uint64_t sc_full;             // [1] a2 done: scores in the score buffer
    uint64_t p_full;              // [4] mask warps: P written over the scores
    uint64_t o_full[2];           // [1] a5 + a4 of a block done, O in buffer b & 1
    uint64_t o_empty[2];          // [4] store warps have O buffer b & 1 in registers
    uint64_t s_done;              // [1] a6 done
    uint64_t snap_full;           // [4] state warps: snapshot of S in shared memory (S read)
    uint64_t snap_empty;          // [1] a5 has read the snapshot
    uint64_t agg_full;            // [1] phase A done: A_j in the first block's O buffer
    uint64_t a_free;              // [4] state warps: A_j read, that O buffer is free
    uint64_t incl_stored;         // [4] state warps: their rows of INCL_j are in the workspace
    uint64_t item_full[2];        // [1] producer
    uint64_t item_empty[2];       // [14] Q producer lane + MMA lane 0 + 3 x 4 warps
    uint64_t fin;                 // [1] tear-down: every MMA done
    uint64_t a5_done;             // [1] DECAY: a5 of a block done (its Q slot may take K lo)
    uint64_t alo_free;            // [1] DECAY: the phase-A lo tile (snapshot buffer) is free
    uint64_t alo_ready;           // [4] DECAY: a phase-A K tile is scaled (hi in place, lo)
    int item[2][8];
    uint32_t tmem_base;
    volatile int abort;
};
static_assert(sizeof(CtrlBlock) <= SM_CTRL_BYTES, "control block too large");

// item fields
enum { IT_T = 0, IT_H, IT_TOK0, IT_TOK1, IT_J, IT_FLAGS, IT_SEQ, IT_VALID };
constexpr int ITF_LAST = 1;  // last segment of its sequence (no successor, no phase A)
constexpr int ITF_LO = 2;    // inter-block product uses S = S_hi + S_lo

// Precision of the inter-block product Q_b S_{<b}.  S is rounded to bf16 for
// the tensor cores (relative error 2^-9).  S grows like sqrt(position) for the
// unit-scaled inputs this operation sees, and so does the error of that
// rounding: measured on the fp32 output, max abs 1.27e-2 over the first 32768
// tokens and 2.02e-2 (past the 2e-2 bound) near 64K tokens of one sequence.
// Up to LA_LO_SPLIT_FROM tokens into a sequence a single bf16 term is used;
// segments that reach past it use S = S_hi + S_lo, two bf16 terms with
// ~2^-16 relative error, at twice the tensor-core and shared-memory cost of
// that product.
#ifndef LA_LO_SPLIT_FROM
#define LA_LO_SPLIT_FROM 32768
#endif

__device__ __forceinline__ void record_status(int *status, int code) {
    atomicCAS(status, 0, code);
}

// Bounded wait on an mbarrier phase; on failure flag the CTA and the device.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity,
                                              const PrefillParams &p, CtrlBlock *cb) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t deadline = globaltimer_ns() + p.wait_limit_ns;
    if (la_wait(bar, parity, deadline, &cb->abort)) return true;
    cb->abort = 1;
    record_status(p.status, ST_TIMEOUT);
    return false;
}

// Every lane waits itself (each needs the acquire), then the warp agrees on
// one result so that control flow stays uniform around .sync.aligned ops.
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, const PrefillParams &p,
                                          CtrlBlock *cb) {
    return __all_sync(0xffffffffu, wait_or_abort(bar, parity, p, cb)) != 0;
}

// K-major operand (Q or K tile, K dim = head features): step kk covers
// features [16kk, 16kk+16): half kk/4, byte offset 32*(kk%4) inside the row.
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t tile, int kk) {
    return smem_desc_sw128(tile + (kk >> 2) * HALF_BYTES + (kk & 3) * 32, 16, 1024);
}
// MN-major operand (K^T, V, S halves; K dim = rows): step kk covers rows
// [16kk, 16kk+16) = two 8-row atoms; the 64-column halves are HALF_BYTES apart.
__device__ __forceinline__ uint64_t desc_mnmajor(uint32_t tile, int kk) {
    return smem_desc_sw128(tile + kk * 2048, HALF_BYTES, 1024);
}

// Byte offset of (row r, 16-byte chunk c in 0..15) in a swizzled [128 x 128] bf16 tile.
__device__ __forceinline__ uint32_t sw_off(int r, int c) {
    return (uint32_t)((c >> 3) * HALF_BYTES + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

// Interleaved layout of a D x D fp32 state in the scratch: element (r, c) at
// ((c/4) * D + r) * 4 + c%4, so a warp reading 4 columns of 32 rows touches
// 512 contiguous bytes.
__device__ __forceinline__ size_t incl_off(int r, int c4) {  // c4 = column / 4
    return ((size_t)c4 * D + r) * 4;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&b);
}

// fp32 pair (bit patterns) -> packed bf16 pair (first value in the low half),
// rounding the magnitude to nearest with ties away from zero: adding half an
// ulp of bf16 to the sign-magnitude bits and keeping the upper 16.  Error
// <= half an ulp like round-to-nearest-even (they differ only on exact ties);
// integer-pipe work only, for finite inputs.
__device__ __forceinline__ uint32_t bf16x2_round(uint32_t u0, uint32_t u1) {
    return __byte_perm(u0 + 0x8000u, u1 + 0x8000u, 0x7632);
}

// Split two fp32 values (bit patterns u0, u1) into a bf16 pair `hi` (rounded
// as in bf16x2_round) and a bf16 pair `lo` holding the exact fp32 residual
// x - hi truncated to bf16, so that x = hi + lo to within 2^-16 |x|.
// Integer and fp32-add work only (finite inputs).
__device__ __forceinline__ void split_hi_lo(uint32_t u0, uint32_t u1, uint32_t &hi, uint32_t &lo) {
    const uint32_t r0 = u0 + 0x8000u;
    const uint32_t r1 = u1 + 0x8000u;
    hi = __byte_perm(r0, r1, 0x7632);
    const float l0 = __uint_as_float(u0) - __uint_as_float(r0 & 0xffff0000u);
    const float l1 = __uint_as_float(u1) - __uint_as_float(r1 & 0xffff0000u);
    lo = __byte_perm(__float_as_uint(l0), __float_as_uint(l1), 0x7632);
}

// Load 32 consecutive TMEM columns of this warp's lanes and wait for them.
__device__ __forceinline__ void tmem_ld_wait32(uint32_t taddr, uint32_t (&x)[32]) {
    tmem_ld32(taddr, x);
    tmem_wait_ld();
    reg_fence(x);
}

// Multiply 32 fp32 words (bit patterns) by c in place.
__device__ __forceinline__ void scale32(uint32_t (&x)[32], float c) {
#pragma unroll
    for (int i = 0; i < 32; ++i) x[i] = __float_as_uint(__uint_as_float(x[i]) * c);
}

// Read S from TMEM and hand it to a5 through the snapshot buffer: either the
// whole state as bf16 (one arrival; columns 0-63 in `shi`, 64-127 in `slo`),
// or, when `lo`, as bf16 hi + lo one 64-column half at a time (two arrivals).
// The last arrival also tells the MMA warp that S has been read, so a6 may
// overwrite it.  DECAY: S is also written back multiplied by `wb` (the decay
// lambda^{nb} of the block whose update a6 adds next) before the arrival.
template <bool DECAY>
__device__ __forceinline__ bool snapshot_state(uint32_t trow, uint8_t *shi, uint8_t *slo, int r, int lane, bool lo,
                                            uint32_t &snap_n, const PrefillParams &p, CtrlBlock *cb,
                                            float wb = 1.f) {
    if (!lo) {
#pragma unroll 1
        for (int hf = 0; hf < 2; ++hf) {  // columns [64 hf, 64 hf + 64) -> shi (hf = 0) or slo (hf = 1)
            uint32_t x[64];
            tmem_ld_cols<64>(trow + TM_S + hf * 64, x);
            if (hf == 0 && !warp_wait(&cb->snap_empty, (snap_n & 1) ^ 1, p, cb)) return false;
            uint8_t *half = hf ? slo : shi;
#pragma unroll
            for (int q = 0; q < 8; ++q)  // 16-byte chunks of 8 columns
                *reinterpret_cast<uint4 *>(half + r * 128 + ((q ^ (r & 7)) << 4)) =
                    make_uint4(bf16x2_round(x[8 * q], x[8 * q + 1]), bf16x2_round(x[8 * q + 2], x[8 * q + 3]),
                               bf16x2_round(x[8 * q + 4], x[8 * q + 5]), bf16x2_round(x[8 * q + 6], x[8 * q + 7]));
            if (DECAY) {
#pragma unroll
                for (int c2 = 0; c2 < 2; ++c2) {
                    scale32(*reinterpret_cast<uint32_t(*)[32]>(&x[32 * c2]), wb);
                    tmem_st32(trow + TM_S + hf * 64 + 32 * c2, *reinterpret_cast<uint32_t(*)[32]>(&x[32 * c2]));
                }
            }
        }
        if (DECAY) tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&cb->snap_full);
        ++snap_n;
        return true;
    }
    // hi + lo, one 64-column half per arrival; a6 is issued only after a5 has
    // used both halves, so S may be read half by half
#pragma unroll 1
    for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
        for (int qq = 0; qq < 2; ++qq) {
            uint32_t x[32];
            tmem_ld_wait32(trow + TM_S + hf * 64 + qq * 32, x);
            if (qq == 0 && !warp_wait(&cb->snap_empty, (snap_n & 1) ^ 1, p, cb)) return false;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t hv[4], lv[4];
#pragma unroll
                for (int w = 0; w < 4; ++w) split_hi_lo(x[8 * c + 2 * w], x[8 * c + 2 * w + 1], hv[w], lv[w]);
                const uint32_t off = (uint32_t)(r * 128 + (((qq * 4 + c) ^ (r & 7)) << 4));
                *reinterpret_cast<uint4 *>(shi + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
                *reinterpret_cast<uint4 *>(slo + off) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
            }
            if (DECAY) {
                scale32(x, wb);
                tmem_st32(trow + TM_S + hf * 64 + qq * 32, x);
            }
        }
        if (DECAY) tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&cb->snap_full);
        ++snap_n;
    }
    return true;
}

// Release the hand-off flag of a segment once all four state warps have
// stored their rows of its inclusive prefix (incl_stored); `leader` is the one
// thread that waits and releases.  Its acquire on the barrier orders the other
// warps' stores before the gpu-scope release of the flag.
__device__ __forceinline__ bool publish_incl(bool leader, uint32_t pub_n, int *flag, const PrefillParams &p,
                                          CtrlBlock *cb) {
    if (!leader) return true;
    const bool all_in = wait_or_abort(&cb->incl_stored, pub_n & 1, p, cb);
    if (all_in && p.inject != LA_INJECT_SKIP_PUBLISH) {
        const int two = 2;
        asm volatile("fence.acq_rel.gpu;" ::: "memory");
        asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(flag), "r"(two) : "memory");
    }
    return all_in;
}

// lambda^n for n >= 0 from log2(lambda) (lambda in (0, 1]: exact 1 for n = 0
// or lambda = 1; underflows to 0 where the true power is below fp32 range).
__device__ __forceinline__ float decay_pow(float l2, int n) { return exp2f(l2 * (float)n); }

// DECAY: scale row r of a swizzled [128 x 128] bf16 tile by c and split the
// fp32 products into bf16 hi (written back in place) and lo (written at the
// same offsets of `lo_tile`): x = hi + lo with |x - hi - lo| <= 2^-17 |x|.
// One thread per row; every 16-byte chunk is read once and written twice.
__device__ __forceinline__ void scale_row_hi_lo(uint8_t *tile, uint8_t *lo_tile, int r, float c) {
#pragma unroll 4
    for (int ch = 0; ch < 16; ++ch) {
        const uint32_t off = sw_off(r, ch);
        const uint4 x = *reinterpret_cast<const uint4 *>(tile + off);
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float a = __uint_as_float(w[i] << 16) * c;           // low bf16 of the pair
            const float b = __uint_as_float(w[i] & 0xffff0000u) * c;   // high bf16
            const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
            const float2 hf = __bfloat1622float2(h);
            const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
            hi[i] = *reinterpret_cast<const uint32_t *>(&h);
            lo[i] = *reinterpret_cast<const uint32_t *>(&l);
        }
        *reinterpret_cast<uint4 *>(tile + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4 *>(lo_tile + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
}

// First row of the b-th row block a sweep visits in an item of nblk blocks
// starting at tok0: in token order, or, for a reversed sweep, from the last.
template <bool REV>
__device__ __forceinline__ int block_row(int tok0, int nblk, int b) {
    return tok0 + (REV ? nblk - 1 - b : b) * BLK;
}

// Every role reads the same item from the two-slot queue the producer fills.
__device__ __forceinline__ bool next_item(uint32_t &it, int (&item)[8], int lane, const PrefillParams &p,
                                          CtrlBlock *cb) {
    const int islot = it & 1;
    if (!warp_wait(&cb->item_full[islot], (it >> 1) & 1, p, cb)) return false;
    // broadcast from lane 0, so that the compiler knows the fields are warp-uniform
#pragma unroll
    for (int f = 0; f < 8; ++f) item[f] = __shfl_sync(0xffffffffu, cb->item[islot][f], 0);
    if (lane == 0) mbar_arrive(&cb->item_empty[islot]);
    ++it;
    return item[IT_VALID] != 0;
}

template <bool DECAY, int BK, bool PAIR = false, bool REV = false>
__global__ void __launch_bounds__(PREFILL_THREADS, 1)
la_prefill_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmq2,
                  const __grid_constant__ PrefillParams p) {
    static_assert(BK == 64 || BK == 128 || BK == 256, "row blocks of 64, 128 or 256 tokens");
    static_assert(BK == 128 || !DECAY, "64- and 256-row blocks: the plain forward only");
    static_assert(!PAIR || REV, "PAIR: two problems in a reversed sweep");
    static_assert(!REV || (!DECAY && BK == 128), "REV: the plain operation at 128-row blocks");
    constexpr bool B64 = BK == 64;  // two 64-row blocks per 128-row tile
    constexpr int SUBS = PAIR ? 2 : 1;  // sub-blocks per row block (PAIR: problem 1, problem 2)
    // BK == 256: one row block per pair of 128-row tiles (see the MMA warp)
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    CtrlBlock *cb = reinterpret_cast<CtrlBlock *>(smem + SM_CTRL);
    // warp index and TMEM base through a shuffle: provably warp-uniform values,
    // so role branches and MMA operands stay in uniform registers
    const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0), lane = threadIdx.x & 31;
    const uint32_t sbase = smem_u32(smem);

    if (threadIdx.x == 0) {
        for (int s = 0; s < KV_STAGES; ++s) {
            mbar_init(&cb->kv_full[s], 1);
            mbar_init(&cb->kv_empty[s], 1);
        }
        for (int s = 0; s < Q_STAGES; ++s) {
            mbar_init(&cb->q_full[s], 1);
            mbar_init(&cb->q_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&cb->o_full[s], 1);
            mbar_init(&cb->o_empty[s], 4);
            mbar_init(&cb->item_full[s], 1);
            mbar_init(&cb->item_empty[s], 14);
        }
        mbar_init(&cb->sc_full, 1);
        mbar_init(&cb->p_full, 4);
        mbar_init(&cb->s_done, 1);
        mbar_init(&cb->snap_full, 4);
        mbar_init(&cb->snap_empty, 1);
        mbar_init(&cb->agg_full, 1);
        mbar_init(&cb->a_free, 4);
        mbar_init(&cb->incl_stored, 4);
        mbar_init(&cb->fin, 1);
        mbar_init(&cb->a5_done, 1);
        mbar_init(&cb->alo_free, 1);
        mbar_init(&cb->alo_ready, 4);
        cb->abort = 0;
        fence_mbarrier_init();
        tma_prefetch_desc(&tmq);
        tma_prefetch_desc(&tmk);
        tma_prefetch_desc(&tmv);
        if (PAIR) tma_prefetch_desc(&tmq2);
    }
    if (warp == 1) {
        tmem_alloc(&cb->tmem_base, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = __shfl_sync(0xffffffffu, cb->tmem_base, 0);
    const int H = p.H;

    if (warp == 0) {
        // ===================== producers =====================
        // lane 0: tickets, K and V tiles (phase A and phase O)
        // lane 1: Q tiles of phase O, which may run ahead of K and V (for
        //         instance into the previous item's phase A)
        if (lane == 0) {
            const uint64_t pol_first = policy_evict_first();
            const uint64_t pol_last = policy_evict_last();
            uint32_t it = 0, kv_n = 0;
            int kv_last_fill[KV_STAGES] = {-1, -1};
            const int total = *reinterpret_cast<volatile int *>(&p.hdr[HDR_TOTAL]);
            bool ok = true;
            for (;;) {
                const int islot = it & 1;
                if (!wait_or_abort(&cb->item_empty[islot], ((it >> 1) & 1) ^ 1, p, cb)) { ok = false; break; }
                int t = atomicAdd(&p.hdr[HDR_TICKET], 1);
                int *item = cb->item[islot];
                item[IT_T] = t;
                item[IT_VALID] = t < total;
                int4 seg = make_int4(0, 0, 0, 0);
                int h = 0;
                if (t < total) {
                    seg = p.segs[t / H];
                    h = t % H;
                    item[IT_H] = h;
                    item[IT_SEQ] = seg.x;
                    item[IT_TOK0] = seg.y;
                    item[IT_TOK1] = seg.z;
                    item[IT_J] = seg.w & (SEG_LAST - 1);
                    const int jj = seg.w & (SEG_LAST - 1);
                    const long long seg_end = (long long)jj * p.seg_len + (seg.z - seg.y);
                    item[IT_FLAGS] = ((seg.w & SEG_LAST) ? ITF_LAST : 0) |
                                     (seg_end > LA_LO_SPLIT_FROM ? ITF_LO : 0);
                }
                mbar_arrive(&cb->item_full[islot]);
                ++it;
                if (t >= total) break;
                const int tok0 = seg.y, tok1 = seg.z;
                const int nblk = (tok1 - tok0 + BLK - 1) / BLK;
                const bool last = (seg.w & SEG_LAST) != 0;
                // phase A (K and V, kept in L2 for phase O), then phase O
                for (int pass = last ? 1 : 0; pass < 2 && ok; ++pass) {
                    const uint64_t pol = pass == 0 ? pol_last : pol_first;
                    for (int b = 0; b < nblk; ++b) {
                        if (cb->abort) { ok = false; break; }
                        const int s = kv_n % KV_STAGES;
                        if (!wait_or_abort(&cb->kv_empty[s], ((kv_n / KV_STAGES) & 1) ^ 1, p, cb)) { ok = false; break; }
                        mbar_expect_tx(&cb->kv_full[s], 2 * TILE_BYTES);
                        const int row = block_row<REV>(tok0, nblk, b);
                        tma_load_4d(smem + SM_K + s * TILE_BYTES, &tmk, &cb->kv_full[s], 0, h, row, 0, pol);
                        tma_load_4d(smem + SM_V + s * TILE_BYTES, &tmv, &cb->kv_full[s], 0, h, row, 0, pol);
                        kv_last_fill[s] = kv_n / KV_STAGES;
                        ++kv_n;
                    }
                }
                if (!ok) break;
            }
            // Tear-down: every issued TMA copy must land before the CTA exits.
            for (int s = 0; s < KV_STAGES; ++s)
                if (kv_last_fill[s] >= 0) {
                    const uint64_t dl = globaltimer_ns() + p.wait_limit_ns;
                    int dummy = 0;
                    la_wait(&cb->kv_full[s], kv_last_fill[s] & 1, dl, &dummy);
                }
            if (!ok) cb->abort = 1;
        } else if (lane == 1) {
            const uint64_t pol_first = policy_evict_first();
            const uint64_t pol_last = policy_evict_last();
            uint32_t it = 0, q_n = 0;
            int q_last_fill[Q_STAGES] = {-1, -1};
            bool ok = true;
            for (;;) {
                const int islot = it & 1;
                if (!wait_or_abort(&cb->item_full[islot], (it >> 1) & 1, p, cb)) { ok = false; break; }
                int item[8];
#pragma unroll
                for (int f = 0; f < 8; ++f) item[f] = cb->item[islot][f];
                mbar_arrive(&cb->item_empty[islot]);
                ++it;
                if (!item[IT_VALID]) break;
                const int h = item[IT_H], tok0 = item[IT_TOK0];
                const int nblk = (item[IT_TOK1] - tok0 + BLK - 1) / BLK;
                for (int u = 0; u < SUBS * nblk; ++u) {  // PAIR: q and q2 tiles of each block in turn
                    const int b = u / SUBS;
                    if (cb->abort) { ok = false; break; }
                    if (PF_Q > 0 && b + PF_Q < nblk) tma_prefetch_4d(&tmq, 0, h, tok0 + (b + PF_Q) * BLK, 0, pol_last);
                    const int qs = q_n % Q_STAGES;
                    if (!wait_or_abort(&cb->q_empty[qs], ((q_n / Q_STAGES) & 1) ^ 1, p, cb)) { ok = false; break; }
                    mbar_expect_tx(&cb->q_full[qs], TILE_BYTES);
                    tma_load_4d(smem + SM_Q + qs * TILE_BYTES, (PAIR && (u & 1)) ? &tmq2 : &tmq, &cb->q_full[qs], 0, h,
                                block_row<REV>(tok0, nblk, b), 0, pol_first);
                    q_last_fill[qs] = q_n / Q_STAGES;
                    ++q_n;
                }
                if (!ok) break;
            }
            for (int s = 0; s < Q_STAGES; ++s)
                if (q_last_fill[s] >= 0) {
                    const uint64_t dl = globaltimer_ns() + p.wait_limit_ns;
                    int dummy = 0;
                    la_wait(&cb->q_full[s], q_last_fill[s] & 1, dl, &dummy);
                }
            if (!ok) cb->abort = 1;
        }
    } else if (warp == 1) {
        // ===================== MMA issuer =====================
        // Phase O runs three dependency chains per block b:
        //   intra chain:  a4(b-1) -> a2(b) -> [mask] -> a4(b)   (needs Q, K, V tiles)
        //   O chain:      a5(b) -> a4(b) -> [O_{b&1} read out] -> a5(b+2)
        //   state chain:  [snapshot S_{<b}] -> a5(b), a6(b) -> [snapshot S_{<b+1}]
        // a5(b) initialises the block's O buffer and a4(b) accumulates onto it,
        // so every accumulator receives its MMAs in a fixed order and the result
        // is deterministic.  a5 comes first so that the Q tile is released as
        // soon as possible (a2 and a5 are its only readers) and so that a6, the
        // state update, follows the snapshot without waiting for the mask.
        // Instead of a fixed program order, the warp polls the barriers and
        // issues whatever is ready; a2(b) waits for a4(b-1) (see TM_O).
        constexpr uint32_t ID_QK = idesc_bf16_f32(BLK, BLK, 0, 0);    // Q (K-major) x K (K-major)
        constexpr uint32_t ID_QS = idesc_bf16_f32(BLK, D / 2, 0, 1);  // Q (K-major) x S half (MN-major)
        constexpr uint32_t ID_QF = idesc_bf16_f32(BLK, D, 0, 1);      // Q (K-major) x S (MN-major)
        constexpr uint32_t ID_KV = idesc_bf16_f32(D, D, 1, 1);  // K^T (MN) x V (MN)
        constexpr uint32_t ID_PV = idesc_bf16_f32(BLK, D, 0, 1);  // P (TMEM) x V (MN)
        // The whole warp runs this loop in step: every lane holds the same
        // counters, barrier probes are combined with __all_sync, and each MMA or
        // commit is issued by the lane that elect.sync picks.
        uint32_t it = 0, kv_n = 0, q_n = 0, blk_n = 0, snap_n = 0, afree_n = 0, a_n = 0, stp_n = 0;
        bool ok = true;
        int item[8];
        auto ready = [&](uint64_t *bar, uint32_t parity) -> bool {
            return __all_sync(0xffffffffu, mbar_test(bar, parity)) != 0;
        };
        // O buffers: block bn accumulates in buffer bn & 1 (double-buffered);
        // under DECAY a block uses both (P V in buffer 0, Q S in buffer 1), so
        // one block is in flight and the barrier phase advances every block.
        auto ob = [&](uint32_t bn) -> uint32_t { return DECAY ? 0u : (bn & 1); };
        auto obpar = [&](uint32_t bn) -> uint32_t { return DECAY ? (bn & 1) : ((bn >> 1) & 1); };
        const uint32_t tm_a = DECAY ? TM_O + 128 : 0;  // DECAY: phase A sums in O buffer 1
        while (ok && next_item(it, item, lane, p, cb)) {
            const int tok0 = item[IT_TOK0], tok1 = item[IT_TOK1];
            const int nblk = (tok1 - tok0 + BLK - 1) / BLK;
            const bool last = (item[IT_FLAGS] & ITF_LAST) != 0;
            const bool lo = (item[IT_FLAGS] & ITF_LO) != 0;
            if (!last) {
                // phase A: A_j = sum_b K_b^T V_b, accumulated in the O buffer of this
                // item's first block once the block two before it has been read out
                // (DECAY: in O buffer 1 once the previous block has been read out)
                if (!warp_wait(&cb->o_empty[ob(blk_n)], obpar(blk_n) ^ 1, p, cb)) break;
                tc_fence_after();
                const uint32_t ta = DECAY ? tmem + tm_a : tmem + TM_O + (blk_n & 1) * 128;
                for (int b = 0; b < nblk; ++b) {
                    if (cb->abort) { ok = false; break; }
                    const int s = kv_n % KV_STAGES;
                    if (DECAY) tc_commit_w(&cb->alo_free);  // every MMA so far has read the lo tile
                    if (!warp_wait(&cb->kv_full[s], (kv_n / KV_STAGES) & 1, p, cb)) { ok = false; break; }
                    if (DECAY && !warp_wait(&cb->alo_ready, a_n & 1, p, cb)) { ok = false; break; }
                    if (REV) {
                        // a reversed sweep starts at a sequence's last segment, which may
                        // end inside its first tile and still has a successor: rows past
                        // the sequence end (the next sequence's tokens) must add nothing
                        // to A_j, so they are zeroed in the K tile (in token order only
                        // full segments have successors)
                        const int valid = min(BLK, tok1 - block_row<REV>(tok0, nblk, b));
                        if (valid < BLK) {
                            uint8_t *kp = smem + SM_K + s * TILE_BYTES;
                            const int nbytes = (BLK - valid) * 128;
                            for (int hh = 0; hh < 2; ++hh)
                                for (int o = lane * 16; o < nbytes; o += 32 * 16)
                                    *reinterpret_cast<uint4 *>(kp + hh * HALF_BYTES + valid * 128 + o) = make_uint4(0, 0, 0, 0);
                            fence_proxy_async_smem();
                            __syncwarp();
                        }
                    }
                    tc_fence_after();
                    const uint32_t kt = sbase + SM_K + s * TILE_BYTES;
                    const uint32_t vt = sbase + SM_V + s * TILE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BLK / 16; ++kk)
                        mma_ss_w(ta, desc_mnmajor(kt, kk), desc_mnmajor(vt, kk), ID_KV, (b > 0 || kk > 0) ? 1u : 0u);
                    if (DECAY) {  // + (Lambda K)_lo^T V, lo tile in the snapshot buffer
                        const uint32_t kl = sbase + SM_SHI;
#pragma unroll
                        for (int kk = 0; kk < BLK / 16; ++kk)
                            mma_ss_w(ta, desc_mnmajor(kl, kk), desc_mnmajor(vt, kk), ID_KV, 1u);
                    }
                    tc_commit_w(&cb->kv_empty[s]);
                    ++kv_n;
                    ++a_n;
                }
                if (!ok) break;
                tc_commit_w(&cb->agg_full);
            }
            // ---------------- phase O: polled three-chain schedule ----------------
            const bool want_final = last && p.state_out != nullptr;
            const uint32_t kv0 = kv_n, q0 = q_n, blk0 = blk_n;
            int i2 = 0, i4 = 0, i5 = 0, sub = 0;  // next block of a2 / a4 / a5; a5 sub-step pending
            const int nsub = SUBS * nblk;         // PAIR: i2, i4, i5 count sub-blocks
            uint32_t spins = 0;
            uint64_t deadline = 0;
            if constexpr (BK == 256) {
                // Row blocks of 256 tokens = pairs of 128-row tiles (2m, 2m+1)
                // sharing one state snapshot.  Score steps, in order: (2m, 2m),
                // (2m+1, 2m+1) with the causal mask, and (2m+1, 2m) unmasked -- the
                // second tile's queries against the first tile's keys, inside the
                // block -- each a2 -> [mask] -> a4 through the one score buffer.
                // a5 of both tiles reads the pair's snapshot S_{<block}; a6 adds
                // K^T V of both tiles once per pair.  A pair keeps both K/V stages
                // until its last score step.
                const int npair = (nblk + 1) / 2, nsteps = 3 * (nblk / 2) + (nblk & 1);
                const int nch = lo ? 2 : 1;
                int u2 = 0, u4 = 0, a6n = 0;  // next score step of a2 / a4; pairs whose a6 is issued
                while (u4 < nsteps) {
                    bool prog = false;
                    // a4(u4): P of the step ready, a5 of its query tile issued
                    if (u4 < u2) {
                        const int m = u4 / 3, w = u4 % 3, ti = 2 * m + (w > 0), tj = 2 * m + (w == 1);
                        const bool pair_last = w == 2 || 2 * m + 1 >= nblk;
                        // (the pair's last step releases its stages: its a6 must be issued)
                        if (ti < i5 && (!pair_last || a6n > m) && ready(&cb->p_full, (stp_n + u4) & 1)) {
                            tc_fence_after();
                            const uint32_t vt = sbase + SM_V + ((kv0 + tj) % KV_STAGES) * TILE_BYTES;
                            const uint32_t bn = blk0 + ti;
#pragma unroll
                            for (int kk = 0; kk < BLK / 16; ++kk)
                                mma_ts_w(tmem + TM_O + (bn & 1) * 128, tmem + TM_SC + kk * 8, desc_mnmajor(vt, kk), ID_PV, 1u);
                            const bool pair_full = 2 * m + 1 < nblk;
                            if (w != 1) tc_commit_w(&cb->o_full[bn & 1]);  // tile 2m (step 0) or 2m+1 (step 2) done
                            if (w == 2 || !pair_full) {  // the pair's last step: both stages are free
                                tc_commit_w(&cb->kv_empty[(kv0 + 2 * m) % KV_STAGES]);
                                if (pair_full) tc_commit_w(&cb->kv_empty[(kv0 + 2 * m + 1) % KV_STAGES]);
                            }
                            ++u4;
                            prog = true;
                        }
                    }
                    // a5 sub-step: one column half (hi + lo) of one tile of the pair
                    if (i5 < nblk) {
                        const int m = i5 / 2, ntp = (2 * m + 1 < nblk) ? 2 : 1;
                        const int tp = sub % ntp, ch = sub / ntp, ti = 2 * m + tp;
                        const uint32_t bn = blk0 + ti;
                        const uint32_t qn = q0 + ti;
                        const bool a_read = last || ti > 0 || ready(&cb->a_free, afree_n & 1);
                        // the tile's Q landed (checked directly: with hi + lo halves the
                        // second tile reads the first half of the snapshot before the
                        // first tile's a5 -- and so the second tile's a2 -- can complete)
                        if (a_read && ready(&cb->q_full[qn % Q_STAGES], (qn / Q_STAGES) & 1) &&
                            ready(&cb->snap_full, snap_n & 1) && ready(&cb->o_empty[bn & 1], ((bn >> 1) & 1) ^ 1)) {
                            tc_fence_after();
                            const uint32_t qt = sbase + SM_Q + (qn % Q_STAGES) * TILE_BYTES;
                            const uint32_t sh = sbase + SM_SHI, sl = sbase + SM_SLO;
                            const uint32_t tq = tmem + TM_O + (bn & 1) * 128;
                            if (!lo) {
#pragma unroll
                                for (int kk = 0; kk < D / 16; ++kk)
                                    mma_ss_w(tq, desc_kmajor(qt, kk), desc_mnmajor(sh, kk), ID_QF, kk > 0 ? 1u : 0u);
                            } else {
                                const uint32_t to = tq + ch * 64;
#pragma unroll
                                for (int kk = 0; kk < D / 16; ++kk)
                                    mma_ss_w(to, desc_kmajor(qt, kk), desc_mnmajor(sh, kk), ID_QS, kk > 0 ? 1u : 0u);
#pragma unroll
                                for (int kk = 0; kk < D / 16; ++kk)
                                    mma_ss_w(to, desc_kmajor(qt, kk), desc_mnmajor(sl, kk), ID_QS, 1u);
                            }
                            if (tp == ntp - 1) {  // every tile of the pair has read this snapshot
                                tc_commit_w(&cb->snap_empty);
                                ++snap_n;
                            }
                            if (ch == nch - 1) {  // the tile's a5 is complete
                                if (!last && ti == 0) ++afree_n;
                                // a first tile's Q is free once its a2 is issued too
                                if ((ti & 1) == 0 && u2 > 3 * (ti / 2)) tc_commit_w(&cb->q_empty[qn % Q_STAGES]);
                                ++i5;
                            }
                            sub = (tp == ntp - 1 && ch == nch - 1) ? 0 : sub + 1;
                            prog = true;
                        }
                    }
                    // a6 of pair a6n: S += K^T V over both tiles, once the pair's a5 is
                    // complete (S has been read out) and its last tile's diagonal a2 is
                    // issued (rows past the sequence end are zeroed by then)
                    if (a6n < npair) {
                        const int m = a6n, ntp = (2 * m + 1 < nblk) ? 2 : 1;
                        if (i5 >= 2 * m + ntp && u2 > 3 * m + ntp - 1) {
                            if ((m < npair - 1) || want_final) {
                                for (int t2 = 0; t2 < ntp; ++t2) {
                                    const int s2 = (kv0 + 2 * m + t2) % KV_STAGES;
                                    const uint32_t kt = sbase + SM_K + s2 * TILE_BYTES;
                                    const uint32_t vt = sbase + SM_V + s2 * TILE_BYTES;
#pragma unroll
                                    for (int kk = 0; kk < BLK / 16; ++kk)
                                        mma_ss_w(tmem + TM_S, desc_mnmajor(kt, kk), desc_mnmajor(vt, kk), ID_KV, 1u);
                                }
                                tc_commit_w(&cb->s_done);
                            }
                            ++a6n;
                            prog = true;
                        }
                    }
                    // a2(u2): the score buffer free (a4 of the previous step issued),
                    // query tile and key tile landed
                    if (u2 < nsteps && u2 <= u4) {
                        const int m = u2 / 3, w = u2 % 3, ti = 2 * m + (w > 0), tj = 2 * m + (w == 1);
                        const int sj = (kv0 + tj) % KV_STAGES;
                        const uint32_t kn = (kv0 + tj) / KV_STAGES, qn = q0 + ti;
                        if (ready(&cb->kv_full[sj], kn & 1) && ready(&cb->q_full[qn % Q_STAGES], (qn / Q_STAGES) & 1)) {
                            if (w < 2) {  // a tile's first use: rows past the sequence end add nothing
                                const int valid = min(BLK, tok1 - (tok0 + tj * BLK));
                                if (valid < BLK) {
                                    uint8_t *kp = smem + SM_K + sj * TILE_BYTES;
                                    uint8_t *vp = smem + SM_V + sj * TILE_BYTES;
                                    const int nbytes = (BLK - valid) * 128;
                                    for (int hh = 0; hh < 2; ++hh)
                                        for (int o = lane * 16; o < nbytes; o += 32 * 16) {
                                            *reinterpret_cast<uint4 *>(kp + hh * HALF_BYTES + valid * 128 + o) = make_uint4(0, 0, 0, 0);
                                            *reinterpret_cast<uint4 *>(vp + hh * HALF_BYTES + valid * 128 + o) = make_uint4(0, 0, 0, 0);
                                        }
                                    fence_proxy_async_smem();
                                    __syncwarp();
                                }
                            }
                            tc_fence_after();
                            const uint32_t qt = sbase + SM_Q + (qn % Q_STAGES) * TILE_BYTES;
                            const uint32_t kt = sbase + SM_K + sj * TILE_BYTES;
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk)
                                mma_ss_w(tmem + TM_SC, desc_kmajor(qt, kk), desc_kmajor(kt, kk), ID_QK, kk > 0 ? 1u : 0u);
                            tc_commit_w(&cb->sc_full);
                            if (w == 2) tc_commit_w(&cb->q_empty[qn % Q_STAGES]);  // Q of tile 2m+1: last reader
                            if (w == 0 && i5 > ti) tc_commit_w(&cb->q_empty[qn % Q_STAGES]);  // tile 2m: a5 came first
                            ++u2;
                            prog = true;
                        }
                    }
                    if (prog) {
                        spins = 0;
                        deadline = 0;
                    } else if (((++spins) & 255u) == 0u) {
                        int stop = 0;
                        if (lane == 0) {
                            const uint64_t now = globaltimer_ns();
                            if (deadline == 0) deadline = now + p.wait_limit_ns;
                            if (now > deadline || cb->abort) {
                                cb->abort = 1;
                                record_status(p.status, ST_TIMEOUT);
                                stop = 1;
                            }
                        }
                        if (__shfl_sync(0xffffffffu, stop, 0)) {
                            ok = false;
                            break;
                        }
                    }
                }
                stp_n += nsteps;
            } else
            while (i4 < nsub) {
                bool prog = false;
                // O chain, a4(i4): P ready, a5 of the block issued
                // (DECAY: P ready also means the block's K rows are scaled into
                // hi + lo, and a6 follows a4)
                if (i4 < i5) {
                    const uint32_t bn = blk0 + i4;
                    if (ready(&cb->p_full, bn & 1)) {
                        tc_fence_after();
                        const bool second = PAIR && (i4 & 1);  // problem 2: its values are the K tile
                        const int s = (kv0 + i4 / SUBS) % KV_STAGES;
                        const uint32_t vt = sbase + (second ? SM_K : SM_V) + s * TILE_BYTES;
#pragma unroll
                        for (int kk = 0; kk < BLK / 16; ++kk)  // P: first 64 score columns; DECAY: P V
                            mma_ts_w(tmem + TM_O + ob(bn) * 128, tmem + TM_SC + kk * 8, desc_mnmajor(vt, kk), ID_PV,
                                     (DECAY && kk == 0) ? 0u : 1u);  // has buffer 0 to itself and starts it
                        if (DECAY) {
                            const uint32_t qn = q0 + i4;
                            if ((i4 < nblk - 1) || want_final) {  // a6: S += (Lambda K)_hi^T V + (Lambda K)_lo^T V
                                const uint32_t kt = sbase + SM_K + s * TILE_BYTES;
                                const uint32_t kl = sbase + SM_Q + (qn % Q_STAGES) * TILE_BYTES;
#pragma unroll
                                for (int kk = 0; kk < BLK / 16; ++kk)
                                    mma_ss_w(tmem + TM_S, desc_mnmajor(kt, kk), desc_mnmajor(vt, kk), ID_KV, 1u);
#pragma unroll
                                for (int kk = 0; kk < BLK / 16; ++kk)
                                    mma_ss_w(tmem + TM_S, desc_mnmajor(kl, kk), desc_mnmajor(vt, kk), ID_KV, 1u);
                                tc_commit_w(&cb->s_done);
                            }
                            tc_commit_w(&cb->q_empty[qn % Q_STAGES]);  // a5 and a6 have read the Q slot
                        }
                        tc_commit_w(&cb->o_full[ob(bn)]);
                        if (!PAIR || second) tc_commit_w(&cb->kv_empty[s]);  // a2, a6 and a4 of this block are issued
                        ++i4;
                        prog = true;
                    }
                }
                // state and O chains, a5(i5) (one full-width pass, or one half of
                // the hi + lo pair) then a6(i5): Q landed (a2 issued), snapshot
                // ready, the block's O buffer free (block i5 - 2 read out; for the
                // first block of a segment with a successor, A_j read out of it)
                // DECAY: a5 goes to O buffer 1 and a6 waits for the scaled keys
                // PAIR: the second sub-block reads the snapshot the first one waited
                // for (released after both), into the other O buffer
                // PAIR with S as hi + lo: the snapshot holds one column half at a
                // time, which both problems read before it is released, so a5 of
                // the two sub-blocks runs as one step per half (both O buffers
                // free, the second q tile landed; i5 advances by two)
                const bool pair_lo = PAIR && lo;
                if (i5 < i2) {
                    const uint32_t bn = blk0 + i5;
                    const bool second = PAIR && (i5 & 1);  // (never with pair_lo)
                    const bool a_read = last || i5 > 0 || ready(&cb->a_free, afree_n & 1);
                    const uint32_t qn2 = q0 + i5 + 1;     // pair_lo: the second sub-block's q tile
                    if (a_read && (second || ready(&cb->snap_full, snap_n & 1)) &&
                        ready(&cb->o_empty[ob(bn)], obpar(bn) ^ 1) &&
                        (!pair_lo || (ready(&cb->o_empty[ob(bn + 1)], obpar(bn + 1) ^ 1) &&
                                      ready(&cb->q_full[qn2 % Q_STAGES], (qn2 / Q_STAGES) & 1)))) {
                        tc_fence_after();
                        const int bi = i5 / SUBS;  // row block
                        const int s = (kv0 + bi) % KV_STAGES;
                        const uint32_t qn = q0 + i5;
                        const uint32_t qt = sbase + SM_Q + (qn % Q_STAGES) * TILE_BYTES;
                        const uint32_t sh = sbase + SM_SHI, sl = sbase + SM_SLO;
                        const uint32_t kt = sbase + SM_K + s * TILE_BYTES;
                        const uint32_t vt = sbase + SM_V + s * TILE_BYTES;
                        const uint32_t tq = DECAY ? tmem + TM_O + 128 : tmem + TM_O + ob(bn) * 128;
                        const bool upd = (bi < nblk - 1) || want_final;
                        // sub-step: one snapshot arrival = one column half (hi + lo
                        // mode) of one row half (64-row blocks) of the tile
                        const int nch = lo ? 2 : 1;
                        const int rh = B64 ? sub / nch : 0;  // 64-row blocks: rows 64 rh .. 64 rh + 63
                        const int ch = sub % nch;            // hi + lo: columns 64 ch .. 64 ch + 63
                        // 64-row blocks: only the lanes (rows) of this block are written
                        const uint32_t m_lo = (B64 && rh == 1) ? ~0u : 0u, m_hi = (B64 && rh == 0) ? ~0u : 0u;
                        if (second) {  // O = Q2 S^T: K-major reads of the snapshot give S transposed
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk)
                                mma_ss_w(tq, desc_kmajor(qt, kk), desc_kmajor(sh, kk), ID_QK, kk > 0 ? 1u : 0u);
                        } else if (!lo) {  // O = Q S, S = the whole [128 x 128] snapshot
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                if (B64)
                                    mma_ss_w_lanes(tq, desc_kmajor(qt, kk), desc_mnmajor(sh, kk), ID_QF, kk > 0 ? 1u : 0u,
                                                   m_lo, m_lo, m_hi, m_hi);
                                else
                                    mma_ss_w(tq, desc_kmajor(qt, kk), desc_mnmajor(sh, kk), ID_QF, kk > 0 ? 1u : 0u);
                            }
                        } else {  // one 64-column half of O = Q (S_hi + S_lo)
                            const uint32_t to = tq + ch * 64;
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                if (B64)
                                    mma_ss_w_lanes(to, desc_kmajor(qt, kk), desc_mnmajor(sh, kk), ID_QS, kk > 0 ? 1u : 0u,
                                                   m_lo, m_lo, m_hi, m_hi);
                                else
                                    mma_ss_w(to, desc_kmajor(qt, kk), desc_mnmajor(sh, kk), ID_QS, kk > 0 ? 1u : 0u);
                            }
#pragma unroll
                            for (int kk = 0; kk < D / 16; ++kk) {
                                if (B64)
                                    mma_ss_w_lanes(to, desc_kmajor(qt, kk), desc_mnmajor(sl, kk), ID_QS, 1u,
                                                   m_lo, m_lo, m_hi, m_hi);
                                else
                                    mma_ss_w(to, desc_kmajor(qt, kk), desc_mnmajor(sl, kk), ID_QS, 1u);
                            }
                            if (pair_lo) {
                                // problem 2: O2 += Q2[:, half ch] (S_hi + S_lo)^T[half ch, :] --
                                // the half read K-major is rows 64 ch .. 64 ch + 63 of S^T
                                const uint32_t tq2 = tmem + TM_O + ob(bn + 1) * 128;
                                const uint32_t qt2 = sbase + SM_Q + (qn2 % Q_STAGES) * TILE_BYTES;
#pragma unroll
                                for (int kk = 0; kk < D / 32; ++kk)
                                    mma_ss_w(tq2, desc_kmajor(qt2, 4 * ch + kk), desc_kmajor(sh, kk), ID_QK,
                                             (ch > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
                                for (int kk = 0; kk < D / 32; ++kk)
                                    mma_ss_w(tq2, desc_kmajor(qt2, 4 * ch + kk), desc_kmajor(sl, kk), ID_QK, 1u);
                            }
                        }
                        if (!PAIR || second || pair_lo) {  // every reader of this snapshot (half) is issued
                            tc_commit_w(&cb->snap_empty);
                            ++snap_n;
                        }
                        const bool rh_done = ch == nch - 1;
                        const bool tile_done = rh_done && (!B64 || rh == 1);
                        if (!last && i5 == 0 && tile_done) ++afree_n;
                        if (B64 && rh_done && rh == 0) {
                            // S += K_lo^T V_lo over rows 0-63: S_{<b1} for the second block
#pragma unroll
                            for (int kk = 0; kk < BLK / 32; ++kk)
                                mma_ss_w(tmem + TM_S, desc_mnmajor(kt, kk), desc_mnmajor(vt, kk), ID_KV, 1u);
                            tc_commit_w(&cb->s_done);
                        }
                        if (tile_done) {
                            if (DECAY) {
                                tc_commit_w(&cb->a5_done);  // the Q slot may now take the block's K lo
                            } else {
                                tc_commit_w(&cb->q_empty[qn % Q_STAGES]);  // a2 and a5 have read the Q tile
                                // PAIR: a6 after the first sub-block's a5 (S has been read
                                // out of TMEM; the snapshot in shared memory stays for the
                                // second)
                                if (upd && !second) {  // a6: S += K^T V (S_{<b} has been read out); 64-row blocks: rows 64-127
#pragma unroll
                                    for (int kk = B64 ? BLK / 32 : 0; kk < BLK / 16; ++kk)
                                        mma_ss_w(tmem + TM_S, desc_mnmajor(kt, kk), desc_mnmajor(vt, kk), ID_KV, 1u);
                                    tc_commit_w(&cb->s_done);
                                }
                            }
                            i5 += pair_lo ? 2 : 1;  // (pair_lo: the second q tile is released after its a2)
                        }
                        sub = tile_done ? 0 : sub + 1;
                        prog = true;
                    }
                }
                // intra chain, a2(i2): its score buffer free (a4 of block i2 - 1
                // issued), tiles landed
                if (i2 < nsub && i2 <= i4) {
                    const int bi = i2 / SUBS;
                    const bool second = PAIR && (i2 & 1);  // problem 2: its keys are the V tile
                    const int s = (kv0 + bi) % KV_STAGES;
                    const uint32_t kn = (kv0 + bi) / KV_STAGES, qn = q0 + i2;
                    if (ready(&cb->kv_full[s], kn & 1) && ready(&cb->q_full[qn % Q_STAGES], (qn / Q_STAGES) & 1)) {
                        const int valid = min(BLK, tok1 - block_row<REV>(tok0, nblk, bi));
                        if (valid < BLK && !second) {  // (PAIR: the first sub-block's a2 reads the tiles first)
                            // rows past the end of the sequence must add nothing to S or O:
                            // zero them in K and V (they may hold the next sequence's tokens)
                            uint8_t *kp = smem + SM_K + s * TILE_BYTES;
                            uint8_t *vp = smem + SM_V + s * TILE_BYTES;
                            const int nbytes = (BLK - valid) * 128;
                            for (int hh = 0; hh < 2; ++hh)
                                for (int o = lane * 16; o < nbytes; o += 32 * 16) {
                                    *reinterpret_cast<uint4 *>(kp + hh * HALF_BYTES + valid * 128 + o) = make_uint4(0, 0, 0, 0);
                                    *reinterpret_cast<uint4 *>(vp + hh * HALF_BYTES + valid * 128 + o) = make_uint4(0, 0, 0, 0);
                                }
                            fence_proxy_async_smem();
                            __syncwarp();
                        }
                        tc_fence_after();
                        const uint32_t qt = sbase + SM_Q + (qn % Q_STAGES) * TILE_BYTES;
                        const uint32_t kt = sbase + (second ? SM_V : SM_K) + s * TILE_BYTES;
#pragma unroll
                        for (int kk = 0; kk < D / 16; ++kk)  // a2: Sc = Q K^T
                            mma_ss_w(tmem + TM_SC, desc_kmajor(qt, kk), desc_kmajor(kt, kk), ID_QK,
                                     kk > 0 ? 1u : 0u);
                        tc_commit_w(&cb->sc_full);
                        if (PAIR && lo && second) tc_commit_w(&cb->q_empty[qn % Q_STAGES]);  // its a5 came first
                        ++i2;
                        prog = true;
                    }
                }
                if (prog) {
                    spins = 0;
                    deadline = 0;
                } else if (((++spins) & 255u) == 0u) {
                    int stop = 0;
                    if (lane == 0) {
                        const uint64_t now = globaltimer_ns();
                        if (deadline == 0) deadline = now + p.wait_limit_ns;
                        if (now > deadline || cb->abort) {
                            cb->abort = 1;
                            record_status(p.status, ST_TIMEOUT);
                            stop = 1;
                        }
                    }
                    if (__shfl_sync(0xffffffffu, stop, 0)) {
                        ok = false;
                        break;
                    }
                }
            }
            kv_n = kv0 + nblk;
            q_n = q0 + nsub;
            blk_n = blk0 + nsub;
        }
        // Tear-down: all MMAs issued by this thread must finish before TMEM is freed.
        __syncwarp();
        tc_commit_w(&cb->fin);
        if (lane == 0) {
            const uint64_t dl = globaltimer_ns() + p.wait_limit_ns;
            int dummy = 0;
            la_wait(&cb->fin, 0, dl, &dummy);
        }
        __syncwarp();
    } else if (warp < W_STORE) {
        // ===================== warps 2-5: causal mask (a3) =====================
        const int q4 = warp & 3;               // TMEM lane quarter this warp may access
        const int r = q4 * 32 + lane;          // tile row = TMEM lane
        const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16);
        // key s kept for row t iff s <= t (REV: iff s >= t)
        uint32_t it = 0, blk_n = 0, kv_n = 0, q_n = 0, a_n = 0;
        bool ok = true;
        int item[8];
        while (ok && next_item(it, item, lane, p, cb)) {
            const int tok0 = item[IT_TOK0], tok1 = item[IT_TOK1];
            const int nblk = (tok1 - tok0 + BLK - 1) / BLK;
            const bool last = (item[IT_FLAGS] & ITF_LAST) != 0;
            const float l2 = DECAY ? log2f(__ldg(p.decay + item[IT_H])) : 0.f;
            const float lam = DECAY ? exp2f(l2) : 1.f;
            if (DECAY && !last) {
                // phase A: scale each K tile's rows to the segment end, row r of
                // the block starting at token t0 by lambda^{tok1-1-t0-r}, hi in
                // place, lo into the snapshot buffer (free: every MMA that read it
                // has completed)
                for (int b = 0; b < nblk; ++b) {
                    const int s = kv_n % KV_STAGES;
                    if (!warp_wait(&cb->alo_free, a_n & 1, p, cb)) { ok = false; break; }
                    if (!warp_wait(&cb->kv_full[s], (kv_n / KV_STAGES) & 1, p, cb)) { ok = false; break; }
                    scale_row_hi_lo(smem + SM_K + s * TILE_BYTES, smem + SM_SHI, r,
                                    decay_pow(l2, tok1 - 1 - block_row<REV>(tok0, nblk, b) - r));
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&cb->alo_ready);
                    ++kv_n;
                    ++a_n;
                }
                if (!ok) break;
            }
            const bool want_final = last && p.state_out != nullptr;
            // score steps: one per tile, or, with 256-row blocks, three per pair of
            // tiles (the third, the second tile's queries against the first tile's
            // keys, is not masked)
            // (PAIR: two per block, one per problem, the same mask)
            const int nsteps = BK == 256 ? 3 * (nblk / 2) + (nblk & 1) : SUBS * nblk;
            for (int b = 0; b < nsteps; ++b) {
                // P = bf16(Sc ⊙ M), inclusive mask, packed
                // two per 32-bit column over the first 64 score columns
                // (DECAY: P = bf16(Sc lambda^{r-c}) for c <= r)
                const uint32_t bn = blk_n + b, tsc = trow + TM_SC;
                const bool full = BK == 256 && b % 3 == 2;  // every key precedes every query
                if (!warp_wait(&cb->sc_full, bn & 1, p, cb)) { ok = false; break; }
                tc_fence_after();
#pragma unroll
                for (int hf = 0; hf < 2; ++hf) {
                    uint32_t x[64];
                    if (!full && (REV ? (hf == 0 && q4 >= 2) : ((hf == 1 && q4 < 2) || (B64 && hf == 0 && q4 >= 2)))) {
                        // rows 0-63 see none of the keys 64-127; with 64-row blocks,
                        // rows 64-127 (the second block) see none of the keys 0-63;
                        // reversed, rows 64-127 see none of the keys 0-63
#pragma unroll
                        for (int w = 0; w < 32; ++w) x[w] = 0u;
                    } else {
                        tmem_ld_cols<64>(tsc + hf * 64, x);
                        if (DECAY) {
                            // x[i] *= lambda^{r-c}, c = 64 hf + i, from the top column
                            // down: the factor restarts at 1 on the diagonal and
                            // gains one factor lambda per column below it
                            const int ctop = hf * 64 + 63;
                            float f = r > ctop ? decay_pow(l2, r - ctop - 1) : 0.f;
#pragma unroll
                            for (int i = 63; i >= 0; --i) {
                                f = (hf * 64 + i == r) ? 1.f : f * lam;
                                x[i] = __float_as_uint(__uint_as_float(x[i]) * f);
                            }
                        }
                        // in place: x[w] <- (x[2w], x[2w+1]) only overwrites words already read
#pragma unroll
                        for (int w = 0; w < 32; ++w) {
                            const int c = hf * 64 + 2 * w;
                            const bool k0 = REV ? c >= r : (full || c <= r);
                            const bool k1 = REV ? c + 1 >= r : (full || c + 1 <= r);
                            x[w] = bf16x2_round(k0 ? x[2 * w] : 0u, k1 ? x[2 * w + 1] : 0u);
                        }
                    }
                    tmem_st32(tsc + hf * 32, *reinterpret_cast<uint32_t(*)[32]>(&x[0]));
                }
                if (DECAY && ((b < nblk - 1) || want_final)) {
                    // keys of the state update: row r scaled by lambda^{nb-1-r} (rows past
                    // the block's end are zero), hi over the K tile, lo into the Q slot
                    // once a5 has read it
                    const int valid = min(BLK, tok1 - (tok0 + b * BLK));
                    const int s = (kv_n + b) % KV_STAGES;
                    const uint32_t qn = q_n + b;
                    if (!warp_wait(&cb->a5_done, bn & 1, p, cb)) { ok = false; break; }
                    scale_row_hi_lo(smem + SM_K + s * TILE_BYTES, smem + SM_Q + (qn % Q_STAGES) * TILE_BYTES, r,
                                    r < valid ? decay_pow(l2, valid - 1 - r) : 0.f);
                    fence_proxy_async_smem();
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&cb->p_full);
            }
            blk_n += nsteps;
            kv_n += nblk;
            q_n += nblk;
        }
    } else if (warp < W_STATE) {
        // ====== warps 6-9: output store (a7), publication of inclusive prefixes ======
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16);
        uint32_t it = 0, blk_n = 0, pub_n = 0;
        bool ok = true;
        int item[8];
        while (ok && next_item(it, item, lane, p, cb)) {
            const int h = item[IT_H], tok0 = item[IT_TOK0], tok1 = item[IT_TOK1];
            const int nblk = (tok1 - tok0 + BLK - 1) / BLK;
            if (!(item[IT_FLAGS] & ITF_LAST)) {
                // the state warps have written INCL_j: release the flag the next
                // segment's look-back waits for
                publish_incl(r == 0, pub_n, p.flags + item[IT_T], p, cb);
                ++pub_n;
            }
            // DECAY: the inter-block term of row r carries lambda^{r+1}
            const float fq = DECAY ? decay_pow(log2f(__ldg(p.decay + h)), r + 1) : 1.f;
            for (int u = 0; u < SUBS * nblk && ok; ++u) {  // PAIR: out, then out2, per block
                const int b = u / SUBS;
                const uint32_t bn = blk_n + u;
                void *const outp = (PAIR && (u & 1)) ? p.out2 : p.out;
                const int row0 = block_row<REV>(tok0, nblk, b);
                const int valid = min(BLK, tok1 - row0);
                const uint32_t obuf = DECAY ? 0u : (bn & 1), opar = DECAY ? (bn & 1) : ((bn >> 1) & 1);
                if (!warp_wait(&cb->o_full[obuf], opar, p, cb)) { ok = false; break; }
                const uint32_t tob = trow + TM_O + obuf * 128;  // this block's O buffer
                tc_fence_after();
                const size_t orow = ((size_t)(row0 + r) * H + h) * D;
                if (DECAY) {
                    // out = (P V, buffer 0) + lambda^{r+1} (Q S, buffer 1) in fp32, 32
                    // columns at a time, each chunk stored as soon as it is formed
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t xi[32], xq[32];
                        tmem_ld32(tob + 32 * c, xi);
                        tmem_ld32(tob + 128 + 32 * c, xq);
                        tmem_wait_ld();
                        reg_fence(xi);
                        reg_fence(xq);
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            xi[i] = __float_as_uint(fmaf(fq, __uint_as_float(xq[i]), __uint_as_float(xi[i])));
                        if (c == 3) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&cb->o_empty[0]);
                        }
                        if (r < valid) {
                            if (!p.out_fp32) {
                                uint32_t w[16];
#pragma unroll
                                for (int i = 0; i < 16; ++i) w[i] = bf16x2_round(xi[2 * i], xi[2 * i + 1]);
                                uint32_t *o = reinterpret_cast<uint32_t *>(reinterpret_cast<__nv_bfloat16 *>(outp) + orow) + 16 * c;
                                if (p.out_al32) {
                                    st_global_cs_v8(o, &w[0]);
                                    st_global_cs_v8(o + 8, &w[8]);
                                } else {
#pragma unroll
                                    for (int q = 0; q < 4; ++q)
                                        __stcs(reinterpret_cast<uint4 *>(o + 4 * q), make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]));
                                }
                            } else {
                                uint32_t *o = reinterpret_cast<uint32_t *>(reinterpret_cast<float *>(outp) + orow) + 32 * c;
                                if (p.out_al32) {
#pragma unroll
                                    for (int q = 0; q < 4; ++q) st_global_cs_v8(o + 8 * q, &xi[8 * q]);
                                } else {
#pragma unroll
                                    for (int q = 0; q < 8; ++q)
                                        __stcs(reinterpret_cast<uint4 *>(o + 4 * q), make_uint4(xi[4 * q], xi[4 * q + 1], xi[4 * q + 2], xi[4 * q + 3]));
                                }
                            }
                        }
                    }
                } else if (!p.out_fp32) {
                    // both 64-column rounds into registers (packed to bf16 as they
                    // arrive), release the O buffer, then write the row with 32-byte
                    // stores: full sectors, and no store queued ahead of the TMEM loads
                    uint32_t w[64];
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        uint32_t x[64];
                        tmem_ld_cols<64>(tob + hf * 64, x);
#pragma unroll
                        for (int c = 0; c < 32; ++c) w[hf * 32 + c] = bf16x2_round(x[2 * c], x[2 * c + 1]);
                    }
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&cb->o_empty[bn & 1]);
                    if (r < valid) {
                        uint32_t *o = reinterpret_cast<uint32_t *>(reinterpret_cast<__nv_bfloat16 *>(outp) + orow);
                        if (p.out_al32) {
#pragma unroll
                            for (int q = 0; q < 8; ++q) st_global_cs_v8(o + 8 * q, &w[8 * q]);
                        } else {
#pragma unroll
                            for (int q = 0; q < 16; ++q)
                                __stcs(reinterpret_cast<uint4 *>(o + 4 * q), make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]));
                        }
                    }
                } else {
#pragma unroll
                    for (int hf = 0; hf < 2; ++hf) {
                        uint32_t x[64];
                        tmem_ld_cols<64>(tob + hf * 64, x);
                        if (hf == 1) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&cb->o_empty[bn & 1]);
                        }
                        if (r < valid) {
                            uint32_t *o = reinterpret_cast<uint32_t *>(reinterpret_cast<float *>(outp) + orow + hf * 64);
                            if (p.out_al32) {
#pragma unroll
                                for (int q = 0; q < 8; ++q) st_global_cs_v8(o + 8 * q, &x[8 * q]);
                            } else {
#pragma unroll
                                for (int q = 0; q < 16; ++q)
                                    __stcs(reinterpret_cast<uint4 *>(o + 4 * q), make_uint4(x[4 * q], x[4 * q + 1], x[4 * q + 2], x[4 * q + 3]));
                            }
                        }
                    }
                }
            }
            blk_n += SUBS * nblk;
        }
    } else {
        // ===== warps 10-13: segment hand-off (phase L), state snapshots, final state =====
        const int q4 = warp & 3;
        const int r = q4 * 32 + lane;
        const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16);
        uint32_t it = 0, snap_n = 0, upd_n = 0, agg_n = 0, blk_n = 0;
        uint8_t *shi = smem + SM_SHI;
        uint8_t *slo = smem + SM_SLO;
        int item[8];
        while (next_item(it, item, lane, p, cb)) {
            const int t = item[IT_T], h = item[IT_H], seq = item[IT_SEQ];
            const int tok0 = item[IT_TOK0], tok1 = item[IT_TOK1], j = item[IT_J];
            const bool last = (item[IT_FLAGS] & ITF_LAST) != 0;
            const bool lo = (item[IT_FLAGS] & ITF_LO) != 0;
            const int nblk = (tok1 - tok0 + BLK - 1) / BLK;
            bool ok = true;
            const float l2 = DECAY ? log2f(__ldg(p.decay + h)) : 0.f;
            // DECAY: lambda^{nb} of block b (its rows), the factor S takes before a6(b)
            auto block_decay = [&](int b) -> float { return decay_pow(l2, min(BLK, tok1 - (tok0 + b * BLK))); };

            // ---------------- phase L: prefix of this segment ----------------
            const float *src_state = nullptr;  // row-major [D][D] (state_in) ...
            const float *src_incl = nullptr;   // ... or interleaved (predecessor)
            if (j == 0) {
                if (p.state_in) src_state = p.state_in + ((size_t)(p.slots ? p.slots[seq] : seq) * H + h) * D * D;
            } else {
                const int pred = t - H;
                const int *fl = p.flags + pred;
                uint32_t n = 0;
                uint64_t deadline = 0;
                for (;;) {
                    int f;
                    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(f) : "l"(fl) : "memory");
                    if (f == 2) break;
                    if (((++n) & 63u) == 0u) {
                        const uint64_t now = globaltimer_ns();
                        if (deadline == 0) deadline = now + p.wait_limit_ns;
                        if (now > deadline || cb->abort) {
                            cb->abort = 1;
                            record_status(p.status, ST_TIMEOUT);
                            ok = false;
                            break;
                        }
                        __nanosleep(256);
                    }
                }
                ok = __all_sync(0xffffffffu, ok) != 0;
                src_incl = p.incl + (size_t)pred * D * D;
            }
            // E_j -> S (TMEM); INCL_j = E_j + A_j -> workspace straight from registers;
            // E_j as bf16 -> the snapshot buffer for a5 of the first block (one
            // bf16 term: written here; hi + lo: through snapshot_state below).
            // With one bf16 term (and no decay) the prefix and its snapshot go out
            // while phase A still runs, and INCL_j is formed afterwards from S and
            // A_j in TMEM, so that only the sum remains between the end of phase A
            // and the first block's a5.
            const bool snap_here = !lo;
            const bool early = snap_here && !DECAY;
            if (!last && !early) {
                if (!warp_wait(&cb->agg_full, agg_n & 1, p, cb)) ok = false;
                ++agg_n;
                tc_fence_after();
            }
            if (snap_here && !warp_wait(&cb->snap_empty, (snap_n & 1) ^ 1, p, cb)) ok = false;
            float *dst_incl = p.incl + (size_t)t * D * D;
#pragma unroll 1
            for (int hf = 0; hf < 2; ++hf) {  // two halves of 64 columns
                uint32_t e[64];
                if (src_incl && ok) {
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const uint4 x = __ldcg(reinterpret_cast<const uint4 *>(src_incl + incl_off(r, hf * 16 + q)));
                        e[4 * q] = x.x; e[4 * q + 1] = x.y; e[4 * q + 2] = x.z; e[4 * q + 3] = x.w;
                    }
                } else if (src_state) {
#pragma unroll
                    for (int q = 0; q < 16; ++q) {
                        const uint4 x = __ldg(reinterpret_cast<const uint4 *>(src_state + (size_t)r * D + hf * 64 + 4 * q));
                        e[4 * q] = x.x; e[4 * q + 1] = x.y; e[4 * q + 2] = x.z; e[4 * q + 3] = x.w;
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 64; ++q) e[q] = 0u;
                }
                if (!DECAY || !snap_here) {  // (DECAY with a direct snapshot: stored decayed below)
                    tmem_st32(trow + TM_S + hf * 64, *reinterpret_cast<uint32_t(*)[32]>(&e[0]));
                    tmem_st32(trow + TM_S + hf * 64 + 32, *reinterpret_cast<uint32_t(*)[32]>(&e[32]));
                }
                if (snap_here) {
                    uint8_t *half = hf ? slo : shi;
#pragma unroll
                    for (int q = 0; q < 8; ++q)  // 16-byte chunks of 8 columns
                        *reinterpret_cast<uint4 *>(half + r * 128 + ((q ^ (r & 7)) << 4)) =
                            make_uint4(bf16x2_round(e[8 * q], e[8 * q + 1]), bf16x2_round(e[8 * q + 2], e[8 * q + 3]),
                                       bf16x2_round(e[8 * q + 4], e[8 * q + 5]), bf16x2_round(e[8 * q + 6], e[8 * q + 7]));
                }
                if (!last && !early) {
                    // A_j: the first block's O buffer (DECAY: O buffer 1);
                    // DECAY: INCL_j = lambda^{len} E_j + A_j
                    const uint32_t ta = DECAY ? TM_O + 128 : TM_O + (blk_n & 1) * 128;
                    const float fl = DECAY ? decay_pow(l2, tok1 - tok0) : 1.f;
#pragma unroll
                    for (int qq = 0; qq < 2; ++qq) {
                        uint32_t a[32];
                        tmem_ld_wait32(trow + ta + hf * 64 + qq * 32, a);
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            float4 v;
                            if (DECAY) {
                                v = make_float4(fmaf(fl, __uint_as_float(e[qq * 32 + 4 * c]), __uint_as_float(a[4 * c])),
                                                fmaf(fl, __uint_as_float(e[qq * 32 + 4 * c + 1]), __uint_as_float(a[4 * c + 1])),
                                                fmaf(fl, __uint_as_float(e[qq * 32 + 4 * c + 2]), __uint_as_float(a[4 * c + 2])),
                                                fmaf(fl, __uint_as_float(e[qq * 32 + 4 * c + 3]), __uint_as_float(a[4 * c + 3])));
                            } else {
                                v = make_float4(__uint_as_float(e[qq * 32 + 4 * c]) + __uint_as_float(a[4 * c]),
                                                __uint_as_float(e[qq * 32 + 4 * c + 1]) + __uint_as_float(a[4 * c + 1]),
                                                __uint_as_float(e[qq * 32 + 4 * c + 2]) + __uint_as_float(a[4 * c + 2]),
                                                __uint_as_float(e[qq * 32 + 4 * c + 3]) + __uint_as_float(a[4 * c + 3]));
                            }
                            __stcg(reinterpret_cast<float4 *>(dst_incl + incl_off(r, hf * 16 + qq * 8 + c)), v);
                        }
                    }
                }
                if (DECAY && snap_here) {  // S = lambda^{nb} E_j, ready for a6 of the first block
                    const float f0 = block_decay(0);
#pragma unroll
                    for (int c2 = 0; c2 < 2; ++c2) {
                        scale32(*reinterpret_cast<uint32_t(*)[32]>(&e[32 * c2]), f0);
                        tmem_st32(trow + TM_S + hf * 64 + 32 * c2, *reinterpret_cast<uint32_t(*)[32]>(&e[32 * c2]));
                    }
                }
            }
            if (!last && !early) {  // A_j has been read: its O buffer is free for a5 of the first block
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&cb->a_free);
                    mbar_arrive(&cb->incl_stored);  // this warp's rows of INCL_j are stored
                }
            }
            // (the store warps release the flag once all four warps have arrived)
            tmem_wait_st();
            if (snap_here) {
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&cb->snap_full);
                ++snap_n;
            } else if (!snapshot_state<DECAY>(trow, shi, slo, r, lane, lo, snap_n, p, cb, DECAY ? block_decay(0) : 1.f)) {
                ok = false;
            }
            if (!last && early) {
                // INCL_j = E_j + A_j from TMEM once phase A is done (a5 of the first
                // block, which overwrites A_j, waits for a_free; a6, which changes S,
                // follows that a5)
                if (!warp_wait(&cb->agg_full, agg_n & 1, p, cb)) ok = false;
                ++agg_n;
                tc_fence_after();
                const uint32_t ta = TM_O + (blk_n & 1) * 128;
#pragma unroll 1
                for (int qq = 0; qq < 4 && ok; ++qq) {
                    uint32_t e[32], a[32];
                    tmem_ld32(trow + TM_S + qq * 32, e);
                    tmem_ld32(trow + ta + qq * 32, a);
                    tmem_wait_ld();
                    reg_fence(e);
                    reg_fence(a);
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        __stcg(reinterpret_cast<float4 *>(dst_incl + incl_off(r, qq * 8 + c)),
                               make_float4(__uint_as_float(e[4 * c]) + __uint_as_float(a[4 * c]),
                                           __uint_as_float(e[4 * c + 1]) + __uint_as_float(a[4 * c + 1]),
                                           __uint_as_float(e[4 * c + 2]) + __uint_as_float(a[4 * c + 2]),
                                           __uint_as_float(e[4 * c + 3]) + __uint_as_float(a[4 * c + 3])));
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&cb->a_free);
                    mbar_arrive(&cb->incl_stored);
                }
            }
            if (!__all_sync(0xffffffffu, ok && !cb->abort)) break;

            // ------------- phase O: state snapshots and the final state -------------
            const bool want_final = last && p.state_out != nullptr;
            const int nupd = BK == 256 ? (nblk + 1) / 2 : nblk;  // state updates: one per row block
            for (int b = 0; b < nupd; ++b) {
                if (B64) {  // S_{<b1} after the update over the tile's first 64 rows
                    if (!warp_wait(&cb->s_done, upd_n & 1, p, cb)) { ok = false; break; }
                    ++upd_n;
                    tc_fence_after();
                    if (!snapshot_state<DECAY>(trow, shi, slo, r, lane, lo, snap_n, p, cb)) { ok = false; break; }
                }
                const bool update = (b < nupd - 1) || want_final;
                if (!update) continue;
                if (!warp_wait(&cb->s_done, upd_n & 1, p, cb)) { ok = false; break; }
                ++upd_n;
                tc_fence_after();
                if (b < nupd - 1) {
                    if (!snapshot_state<DECAY>(trow, shi, slo, r, lane, lo, snap_n, p, cb,
                                               DECAY ? block_decay(b + 1) : 1.f)) {  // S_{<b+1}
                        ok = false;
                        break;
                    }
                } else {
                    // final state of the sequence -> state_out (row-major fp32)
                    float *so = p.state_out + ((size_t)(p.slots ? p.slots[seq] : seq) * H + h) * D * D + (size_t)r * D;
#pragma unroll 1
                    for (int qq = 0; qq < 4; ++qq) {
                        uint32_t x[32];
                        tmem_ld_wait32(trow + TM_S + qq * 32, x);
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            *reinterpret_cast<float4 *>(so + qq * 32 + 4 * c) =
                                make_float4(__uint_as_float(x[4 * c]), __uint_as_float(x[4 * c + 1]),
                                            __uint_as_float(x[4 * c + 2]), __uint_as_float(x[4 * c + 3]));
                    }
                }
            }
            blk_n += SUBS * nblk;  // (O buffers count sub-blocks)
            if (!ok) break;
        }
    }

    // ===================== tear-down =====================
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, TM_COLS);
}

// ---------------------------------------------------------------------------
// Scheduler: validates cu_seqlens, builds the segment table, resets the
// ticket counter and the hand-off flags, and handles empty sequences.
// One block of 1024 threads.
// ---------------------------------------------------------------------------
constexpr int SCHED_THREADS = 1024;

struct ScheduleParams {
    const int *cu;          // device cu_seqlens [nseq+1] or null (equal lengths)
    int fixed_len;          // length of every sequence when cu is null
    int nseq, T, max_seqlen, H, seg_len, Gmax;
    int *hdr;
    int4 *segs;
    int *flags;
    const float *state_in;
    float *state_out;
    const int *slots;       // null, or [nseq] state slots in a pool of n_slots
    int n_slots;
    const float *decay;     // null, or [H] per-head decays, each must lie in (0, 1]
    int reverse;            // list each sequence's segments from its end (reversed sweep)
    int *status;
};

__device__ __forceinline__ int cu_at(const ScheduleParams &s, int i) {
    return s.cu ? s.cu[i] : i * s.fixed_len;
}

__global__ void __launch_bounds__(SCHED_THREADS, 1) la_schedule_kernel(const ScheduleParams s) {
    __shared__ int warp_sums[SCHED_THREADS / 32];
    __shared__ int carry_sh;
    const int tid = threadIdx.x;
    // 1. validation
    int bad = 0;
    if (s.cu) {
        if (tid == 0 && (s.cu[0] != 0 || s.cu[s.nseq] != s.T)) bad = 1;
        for (int i = tid; i < s.nseq; i += SCHED_THREADS) {
            const int len = s.cu[i + 1] - s.cu[i];
            if (len < 0 || len > s.max_seqlen) bad = 1;
        }
    }
    if (s.slots)
        for (int i = tid; i < s.nseq; i += SCHED_THREADS)
            if (s.slots[i] < 0 || s.slots[i] >= s.n_slots) bad = 1;
    if (s.decay)
        for (int h = tid; h < s.H; h += SCHED_THREADS) {
            const float lam = s.decay[h];
            if (!(lam > 0.f && lam <= 1.f)) bad = 1;  // also rejects NaN
        }
    bad = __syncthreads_or(bad);
    if (bad) {
        if (tid == 0) {
            s.hdr[HDR_TOTAL] = 0;
            s.hdr[HDR_TICKET] = 0;
            s.hdr[HDR_G] = 0;
            atomicCAS(s.status, 0, ST_INVALID);
        }
        return;
    }
    // 2. segment table: exclusive scan of per-sequence segment counts
    if (tid == 0) carry_sh = 0;
    __syncthreads();
    for (int base = 0; base < s.nseq; base += SCHED_THREADS) {
        const int i = base + tid;
        int a = 0, len = 0, nseg = 0;
        if (i < s.nseq) {
            a = cu_at(s, i);
            len = cu_at(s, i + 1) - a;
            nseg = (len + s.seg_len - 1) / s.seg_len;
        }
        int x = nseg;  // inclusive warp scan
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if ((tid & 31) >= o) x += y;
        }
        if ((tid & 31) == 31) warp_sums[tid >> 5] = x;
        __syncthreads();
        if (tid < 32) {
            int w = warp_sums[tid];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, w, o);
                if (tid >= o) w += y;
            }
            warp_sums[tid] = w;  // inclusive over warps
        }
        __syncthreads();
        const int excl = carry_sh + x - nseg + ((tid >> 5) ? warp_sums[(tid >> 5) - 1] : 0);
        for (int jj = 0; jj < nseg; ++jj) {
            // jj: position in the sweep; reversed, the sweep starts at the last segment
            const int t0 = a + (s.reverse ? nseg - 1 - jj : jj) * s.seg_len;
            const int t1 = min(t0 + s.seg_len, a + len);
            s.segs[excl + jj] = make_int4(i, t0, t1, jj | (jj == nseg - 1 ? SEG_LAST : 0));
        }
        __syncthreads();
        if (tid == 0) carry_sh += warp_sums[SCHED_THREADS / 32 - 1];
        __syncthreads();
    }
    const int G = carry_sh;
    // 3. reset the hand-off flags of this launch's items
    for (int e = tid; e < G * s.H; e += SCHED_THREADS) s.flags[e] = 0;
    // 4. empty sequences: the final state is the carried-in state (nothing to
    //    do when the states are updated in place)
    if (s.state_out && s.state_out != s.state_in) {
        for (int i = 0; i < s.nseq; ++i) {
            if (cu_at(s, i + 1) != cu_at(s, i)) continue;
            const size_t n = (size_t)s.H * D * D, off = (size_t)i * n;
            for (size_t e = tid; e < n; e += SCHED_THREADS)
                s.state_out[off + e] = s.state_in ? s.state_in[off + e] : 0.f;
        }
    }
    if (tid == 0) {
        s.hdr[HDR_TOTAL] = G * s.H;
        s.hdr[HDR_TICKET] = 0;
        s.hdr[HDR_G] = G;
    }
}

}  // namespace la
