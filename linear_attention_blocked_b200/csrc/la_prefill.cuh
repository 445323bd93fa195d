// la_prefill.cuh -- blocked causal linear attention prefill for sm_100a.
//
// What one CTA does ("MiniMax-01技术报告解读", §2.2 线性注意力; §3.2 item 3 LASP+):
// the token range of every (sequence, head) is cut into segments of
// `seg_len` tokens; a work item is one (segment, head).  CTAs are persistent
// and take items in ticket order from a device counter.  For an item
//
//   phase A (only if a later segment of the same sequence exists):
//       local KV sum  A_j = sum_b K_b^T V_b    (tcgen05, fp32, in the O columns)
//   phase L (look-back, LASP+ "gather + global prefix" on SMs instead of ranks):
//       E_j = state_in (j = 0)  or  INCL_{j-1} published by the item that
//       owns segment j-1 (bounded spin on its flag);  INCL_j = E_j + A_j is
//       published for segment j+1.
//   phase O (blocked scan over the segment's row blocks, starting from E_j):
//       Sc  = Q_b K_b^T                    a2   (SS MMA, M=N=128, K=d)
//       P   = bf16(Sc ⊙ M), inclusive mask a3   (TMEM -> regs -> TMEM)
//       O   = Q_b S_hi + Q_b S_lo          a5   (S split in two bf16 terms)
//       S  += K_b^T V_b                    a6   (SS MMA, both MN-major)
//       O  += P V_b                        a4   (TS MMA, P read from TMEM)
//       out = O (bf16 or fp32)             a7
//   and, for the last segment, the final state S goes to state_out.
//
// Warp roles (192 threads): warp 0 = TMA producer + ticket fetch, warp 1 =
// TMEM allocator + MMA issuer (lane 0 issues), warps 2-5 = TMEM-lane owners
// doing masking, state snapshots, look-back and output stores.
//
// Shared memory (1024-byte aligned, 128-byte swizzle everywhere):
//   K ring 2 x 32 KiB | V ring 2 x 32 KiB | Q 32 KiB | S_hi 32 KiB | S_lo 32 KiB
//   | barriers + item queue.
// A [128 x 128] bf16 tile is two 16 KiB halves (columns 0-63, 64-127), each
// 128 rows of 128 bytes as TMA writes them with a {64, 1, 128} box.
// TMEM (512 columns x 128 lanes x 32 bit): Sc [0,128) | P [128,192) |
//   O [256,384) | S [384,512).
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
constexpr int PREFILL_THREADS = 192;

constexpr int SM_K = 0;
constexpr int SM_V = SM_K + KV_STAGES * TILE_BYTES;
constexpr int SM_Q = SM_V + KV_STAGES * TILE_BYTES;
constexpr int SM_SHI = SM_Q + TILE_BYTES;
constexpr int SM_SLO = SM_SHI + TILE_BYTES;
constexpr int SM_CTRL = SM_SLO + TILE_BYTES;  // 229376
constexpr int SM_CTRL_BYTES = 1024;
constexpr int PREFILL_SMEM = SM_CTRL + SM_CTRL_BYTES + 1024;  // + alignment slack

constexpr uint32_t TM_SC = 0, TM_P = 128, TM_O = 256, TM_S = 384, TM_COLS = 512;

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
    const float *state_in;  // [nseq, H, D, D] or null
    float *state_out;       // [nseq, H, D, D] or null
    void *out;              // [T, H, D]
    int out_fp32;
    int H;
    int *hdr;               // workspace header
    const int4 *segs;       // [G] {seq, tok0, tok1, jinfo}
    int *flags;             // [G*H] 0 = empty, 2 = inclusive prefix published
    float *incl;            // [G*H][D*D] inclusive prefixes, column-quad interleaved
    unsigned long long wait_limit_ns;
    int inject;
    int *status;            // sticky device status word
};

struct CtrlBlock {
    uint64_t kv_full[KV_STAGES], kv_empty[KV_STAGES];
    uint64_t q_full, q_empty;
    uint64_t sc_full, p_full, o_full, o_empty;
    uint64_t s_done, snap_full, snap_empty, agg_full;
    uint64_t item_full[2], item_empty[2];
    uint64_t fin, pub;
    int item[2][8];
    uint32_t tmem_base;
    volatile int abort;
};
static_assert(sizeof(CtrlBlock) <= SM_CTRL_BYTES, "control block too large");

// item fields
enum { IT_T = 0, IT_H, IT_TOK0, IT_TOK1, IT_J, IT_LAST, IT_SEQ, IT_VALID };

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

__global__ void __launch_bounds__(PREFILL_THREADS, 1)
la_prefill_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const __grid_constant__ CUtensorMap tmv, const __grid_constant__ PrefillParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    CtrlBlock *cb = reinterpret_cast<CtrlBlock *>(smem + SM_CTRL);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sbase = smem_u32(smem);

    if (threadIdx.x == 0) {
        for (int s = 0; s < KV_STAGES; ++s) {
            mbar_init(&cb->kv_full[s], 1);
            mbar_init(&cb->kv_empty[s], 1);
        }
        mbar_init(&cb->q_full, 1);
        mbar_init(&cb->q_empty, 1);
        mbar_init(&cb->sc_full, 1);
        mbar_init(&cb->p_full, 4);
        mbar_init(&cb->o_full, 1);
        mbar_init(&cb->o_empty, 4);
        mbar_init(&cb->s_done, 1);
        mbar_init(&cb->snap_full, 4);
        mbar_init(&cb->snap_empty, 1);
        mbar_init(&cb->agg_full, 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(&cb->item_full[s], 1);
            mbar_init(&cb->item_empty[s], 5);
        }
        mbar_init(&cb->fin, 1);
        mbar_init(&cb->pub, 4);
        cb->abort = 0;
        fence_mbarrier_init();
        tma_prefetch_desc(&tmq);
        tma_prefetch_desc(&tmk);
        tma_prefetch_desc(&tmv);
    }
    if (warp == 1) {
        tmem_alloc(&cb->tmem_base, TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = cb->tmem_base;
    const int H = p.H;

    if (warp == 0) {
        // ===================== producer: tickets + TMA =====================
        if (lane == 0) {
            const uint64_t pol_first = policy_evict_first();
            const uint64_t pol_last = policy_evict_last();
            uint32_t it = 0, kv_n = 0, q_n = 0;
            int kv_last_fill[KV_STAGES] = {-1, -1};
            int q_last_fill = -1;
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
                    item[IT_LAST] = (seg.w & SEG_LAST) ? 1 : 0;
                }
                mbar_arrive(&cb->item_full[islot]);
                ++it;
                if (t >= total) break;
                const int tok0 = seg.y, tok1 = seg.z;
                const int nblk = (tok1 - tok0 + BLK - 1) / BLK;
                const bool last = (seg.w & SEG_LAST) != 0;
                if (!last) {  // phase A: K and V only; kept in L2 for phase O
                    for (int b = 0; b < nblk && ok; ++b) {
                        if (cb->abort) { ok = false; break; }
                        const int s = kv_n % KV_STAGES;
                        if (!wait_or_abort(&cb->kv_empty[s], ((kv_n / KV_STAGES) & 1) ^ 1, p, cb)) { ok = false; break; }
                        mbar_expect_tx(&cb->kv_full[s], 2 * TILE_BYTES);
                        const int row = tok0 + b * BLK;
                        uint8_t *kt = smem + SM_K + s * TILE_BYTES;
                        uint8_t *vt = smem + SM_V + s * TILE_BYTES;
                        tma_load_3d(kt, &tmk, &cb->kv_full[s], 0, h, row, pol_last);
                        tma_load_3d(kt + HALF_BYTES, &tmk, &cb->kv_full[s], 64, h, row, pol_last);
                        tma_load_3d(vt, &tmv, &cb->kv_full[s], 0, h, row, pol_last);
                        tma_load_3d(vt + HALF_BYTES, &tmv, &cb->kv_full[s], 64, h, row, pol_last);
                        kv_last_fill[s] = kv_n / KV_STAGES;
                        ++kv_n;
                    }
                }
                for (int b = 0; b < nblk && ok; ++b) {  // phase O: Q, K, V
                    if (cb->abort) { ok = false; break; }
                    const int row = tok0 + b * BLK;
                    if (!wait_or_abort(&cb->q_empty, (q_n & 1) ^ 1, p, cb)) { ok = false; break; }
                    mbar_expect_tx(&cb->q_full, TILE_BYTES);
                    uint8_t *qt = smem + SM_Q;
                    tma_load_3d(qt, &tmq, &cb->q_full, 0, h, row, pol_first);
                    tma_load_3d(qt + HALF_BYTES, &tmq, &cb->q_full, 64, h, row, pol_first);
                    q_last_fill = q_n;
                    ++q_n;
                    const int s = kv_n % KV_STAGES;
                    if (!wait_or_abort(&cb->kv_empty[s], ((kv_n / KV_STAGES) & 1) ^ 1, p, cb)) { ok = false; break; }
                    mbar_expect_tx(&cb->kv_full[s], 2 * TILE_BYTES);
                    uint8_t *kt = smem + SM_K + s * TILE_BYTES;
                    uint8_t *vt = smem + SM_V + s * TILE_BYTES;
                    tma_load_3d(kt, &tmk, &cb->kv_full[s], 0, h, row, pol_first);
                    tma_load_3d(kt + HALF_BYTES, &tmk, &cb->kv_full[s], 64, h, row, pol_first);
                    tma_load_3d(vt, &tmv, &cb->kv_full[s], 0, h, row, pol_first);
                    tma_load_3d(vt + HALF_BYTES, &tmv, &cb->kv_full[s], 64, h, row, pol_first);
                    kv_last_fill[s] = kv_n / KV_STAGES;
                    ++kv_n;
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
            if (q_last_fill >= 0) {
                const uint64_t dl = globaltimer_ns() + p.wait_limit_ns;
                int dummy = 0;
                la_wait(&cb->q_full, q_last_fill & 1, dl, &dummy);
            }
            if (!ok) {
                // unblock the consumers waiting for an item: hand them a stop item
                cb->abort = 1;
            }
        }
    } else if (warp == 1) {
        // ===================== MMA issuer =====================
        constexpr uint32_t ID_QK = idesc_bf16_f32(BLK, BLK, 0, 0);  // Q (K-major) x K (K-major)
        constexpr uint32_t ID_QS = idesc_bf16_f32(BLK, D, 0, 1);    // Q (K-major) x S (MN-major)
        constexpr uint32_t ID_KV = idesc_bf16_f32(D, D, 1, 1);      // K^T (MN) x V (MN)
        constexpr uint32_t ID_PV = idesc_bf16_f32(BLK, D, 0, 1);    // P (TMEM) x V (MN)
        uint32_t it = 0, kv_n = 0, q_n = 0, blk_n = 0, snap_n = 0;
        bool ok = true;
        while (ok) {
            const int islot = it & 1;
            if (!warp_wait(&cb->item_full[islot], (it >> 1) & 1, p, cb)) break;
            int item[8];
#pragma unroll
            for (int f = 0; f < 8; ++f) item[f] = cb->item[islot][f];
            __syncwarp();
            if (lane == 0) mbar_arrive(&cb->item_empty[islot]);
            ++it;
            if (!item[IT_VALID]) break;
            const int tok0 = item[IT_TOK0], tok1 = item[IT_TOK1];
            const int nblk = (tok1 - tok0 + BLK - 1) / BLK;
            const bool last = item[IT_LAST] != 0;
            if (!last) {  // phase A: A_j = sum_b K_b^T V_b, accumulated in the O columns
                // (S may still be read by the previous item's final-state store; O is
                // free once the previous block's output has been read out)
                if (!warp_wait(&cb->o_empty, (blk_n & 1) ^ 1, p, cb)) break;
                for (int b = 0; b < nblk; ++b) {
                    if (cb->abort) { ok = false; break; }
                    const int s = kv_n % KV_STAGES;
                    if (!warp_wait(&cb->kv_full[s], (kv_n / KV_STAGES) & 1, p, cb)) { ok = false; break; }
                    tc_fence_after();
                    if (lane == 0) {
                        const uint32_t kt = sbase + SM_K + s * TILE_BYTES;
                        const uint32_t vt = sbase + SM_V + s * TILE_BYTES;
#pragma unroll
                        for (int kk = 0; kk < BLK / 16; ++kk)
                            mma_ss(tmem + TM_O, desc_mnmajor(kt, kk), desc_mnmajor(vt, kk), ID_KV,
                                   (b > 0 || kk > 0) ? 1u : 0u);
                        tc_commit(&cb->kv_empty[s]);
                    }
                    __syncwarp();
                    ++kv_n;
                }
                if (!ok) break;
                if (lane == 0) tc_commit(&cb->agg_full);
                __syncwarp();
            }
            const bool want_final = last && p.state_out != nullptr;
            for (int b = 0; b < nblk; ++b) {  // phase O
                const int valid = min(BLK, tok1 - (tok0 + b * BLK));
                const bool update = (b < nblk - 1) || want_final;
                const int s = kv_n % KV_STAGES;
                if (cb->abort) { ok = false; break; }
                if (!warp_wait(&cb->q_full, q_n & 1, p, cb)) { ok = false; break; }
                if (!warp_wait(&cb->kv_full[s], (kv_n / KV_STAGES) & 1, p, cb)) { ok = false; break; }
                tc_fence_after();
                const uint32_t qt = sbase + SM_Q;
                const uint32_t kt = sbase + SM_K + s * TILE_BYTES;
                const uint32_t vt = sbase + SM_V + s * TILE_BYTES;
                if (valid < BLK) {
                    // rows past the end of the sequence must add nothing to S or O:
                    // zero them in K and V (they may hold the next sequence's tokens)
                    uint8_t *kp = smem + SM_K + s * TILE_BYTES;
                    uint8_t *vp = smem + SM_V + s * TILE_BYTES;
                    const int nbytes = (BLK - valid) * 128;
                    for (int half = 0; half < 2; ++half)
                        for (int o = lane * 16; o < nbytes; o += 32 * 16) {
                            *reinterpret_cast<uint4 *>(kp + half * HALF_BYTES + valid * 128 + o) = make_uint4(0, 0, 0, 0);
                            *reinterpret_cast<uint4 *>(vp + half * HALF_BYTES + valid * 128 + o) = make_uint4(0, 0, 0, 0);
                        }
                    fence_proxy_async_smem();
                    __syncwarp();
                }
                if (lane == 0) {  // a2: Sc = Q K^T
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_ss(tmem + TM_SC, desc_kmajor(qt, kk), desc_kmajor(kt, kk), ID_QK, kk > 0 ? 1u : 0u);
                    tc_commit(&cb->sc_full);
                }
                __syncwarp();
                if (!warp_wait(&cb->snap_full, snap_n & 1, p, cb)) { ok = false; break; }
                if (!warp_wait(&cb->o_empty, (blk_n & 1) ^ 1, p, cb)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {  // a5: O = Q S_hi + Q S_lo
                    const uint32_t sh = sbase + SM_SHI, sl = sbase + SM_SLO;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_ss(tmem + TM_O, desc_kmajor(qt, kk), desc_mnmajor(sh, kk), ID_QS, kk > 0 ? 1u : 0u);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_ss(tmem + TM_O, desc_kmajor(qt, kk), desc_mnmajor(sl, kk), ID_QS, 1u);
                    tc_commit(&cb->snap_empty);
                    tc_commit(&cb->q_empty);
                    if (update) {  // a6: S += K^T V
#pragma unroll
                        for (int kk = 0; kk < BLK / 16; ++kk)
                            mma_ss(tmem + TM_S, desc_mnmajor(kt, kk), desc_mnmajor(vt, kk), ID_KV, 1u);
                        tc_commit(&cb->s_done);
                    }
                }
                __syncwarp();
                ++q_n;
                ++snap_n;
                if (!warp_wait(&cb->p_full, blk_n & 1, p, cb)) { ok = false; break; }
                tc_fence_after();
                if (lane == 0) {  // a4: O += P V
#pragma unroll
                    for (int kk = 0; kk < BLK / 16; ++kk)
                        mma_ts(tmem + TM_O, tmem + TM_P + kk * 8, desc_mnmajor(vt, kk), ID_PV, 1u);
                    tc_commit(&cb->o_full);
                    tc_commit(&cb->kv_empty[s]);
                }
                __syncwarp();
                ++kv_n;
                ++blk_n;
            }
        }
        // Tear-down: all MMAs issued by this thread must finish before TMEM is freed.
        if (lane == 0) {
            tc_commit(&cb->fin);
            const uint64_t dl = globaltimer_ns() + p.wait_limit_ns;
            int dummy = 0;
            la_wait(&cb->fin, 0, dl, &dummy);
        }
        __syncwarp();
    } else {
        // ===================== TMEM-lane owners (warps 2-5) =====================
        const int q4 = warp & 3;               // TMEM lane quarter this warp may access
        const int r = q4 * 32 + lane;          // tile row = TMEM lane
        const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16);
        uint32_t it = 0, blk_n = 0, snap_n = 0, upd_n = 0, agg_n = 0, pub_n = 0;
        uint8_t *shi = smem + SM_SHI;
        uint8_t *slo = smem + SM_SLO;
        while (true) {
            const int islot = it & 1;
            if (!warp_wait(&cb->item_full[islot], (it >> 1) & 1, p, cb)) break;
            int item[8];
#pragma unroll
            for (int f = 0; f < 8; ++f) item[f] = cb->item[islot][f];
            __syncwarp();
            if (lane == 0) mbar_arrive(&cb->item_empty[islot]);
            ++it;
            if (!item[IT_VALID]) break;
            const int t = item[IT_T], h = item[IT_H], seq = item[IT_SEQ];
            const int tok0 = item[IT_TOK0], tok1 = item[IT_TOK1], j = item[IT_J];
            const bool last = item[IT_LAST] != 0;
            const int nblk = (tok1 - tok0 + BLK - 1) / BLK;
            bool ok = true;

            // ---------------- phase L: prefix of this segment ----------------
            const float *src_state = nullptr;  // row-major [D][D] (state_in) ...
            const float *src_incl = nullptr;   // ... or interleaved (predecessor)
            if (j == 0) {
                if (p.state_in) src_state = p.state_in + ((size_t)seq * H + h) * D * D;
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
            if (!last) {
                if (!warp_wait(&cb->agg_full, agg_n & 1, p, cb)) ok = false;
                ++agg_n;
                tc_fence_after();
            }
            // the snapshot buffer must be free (a5 of the previous block done)
            if (!warp_wait(&cb->snap_empty, (snap_n & 1) ^ 1, p, cb)) ok = false;
            float *dst_incl = p.incl + (size_t)t * D * D;
#pragma unroll 1
            for (int c = 0; c < D / 32; ++c) {
                float e[32];
                if (src_incl && ok) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 x = __ldcg(reinterpret_cast<const float4 *>(src_incl + incl_off(r, c * 8 + q)));
                        e[4 * q] = x.x; e[4 * q + 1] = x.y; e[4 * q + 2] = x.z; e[4 * q + 3] = x.w;
                    }
                } else if (src_state) {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 x = __ldg(reinterpret_cast<const float4 *>(src_state + (size_t)r * D + c * 32 + 4 * q));
                        e[4 * q] = x.x; e[4 * q + 1] = x.y; e[4 * q + 2] = x.z; e[4 * q + 3] = x.w;
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 32; ++q) e[q] = 0.f;
                }
                if (!last) {  // INCL_j = E_j + A_j  (A_j sits in the O columns)
                    uint32_t a[32];
                    tmem_ld32(trow + TM_O + c * 32, a);
                    tmem_wait_ld();
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        float4 x;
                        x.x = e[4 * q] + __uint_as_float(a[4 * q]);
                        x.y = e[4 * q + 1] + __uint_as_float(a[4 * q + 1]);
                        x.z = e[4 * q + 2] + __uint_as_float(a[4 * q + 2]);
                        x.w = e[4 * q + 3] + __uint_as_float(a[4 * q + 3]);
                        __stcg(reinterpret_cast<float4 *>(dst_incl + incl_off(r, c * 8 + q)), x);
                    }
                }
                // S (TMEM) = E_j for the scan, and its bf16 hi/lo split for a5
                uint32_t eu[32];
#pragma unroll
                for (int q = 0; q < 32; ++q) eu[q] = __float_as_uint(e[q]);
                tmem_st32(trow + TM_S + c * 32, eu);
#pragma unroll
                for (int q = 0; q < 4; ++q) {  // 4 chunks of 8 columns
                    uint32_t hv[4], lv[4];
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const float x0 = e[8 * q + 2 * w], x1 = e[8 * q + 2 * w + 1];
                        const __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
                        hv[w] = pack_bf16x2(__bfloat162float(h0), __bfloat162float(h1));
                        lv[w] = pack_bf16x2(x0 - __bfloat162float(h0), x1 - __bfloat162float(h1));
                    }
                    const uint32_t off = sw_off(r, c * 4 + q);
                    *reinterpret_cast<uint4 *>(shi + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
                    *reinterpret_cast<uint4 *>(slo + off) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
                }
            }
            fence_proxy_async_smem();
            tmem_wait_st();
            tc_fence_before();
            if (!last) {
                // publish INCL_j: every warp fences its stores and arrives; the
                // owner of row 0 waits (bounded) for all four, then releases the flag
                __threadfence();
                __syncwarp();
                if (lane == 0) mbar_arrive(&cb->pub);
                if (r == 0) {
                    const bool all_in = wait_or_abort(&cb->pub, pub_n & 1, p, cb);
                    if (all_in && ok && p.inject != LA_INJECT_SKIP_PUBLISH) {
                        const int two = 2;
                        int *fl = p.flags + t;
                        asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(fl), "r"(two) : "memory");
                    }
                }
                ++pub_n;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&cb->snap_full);
            ++snap_n;
            if (!__all_sync(0xffffffffu, ok && !cb->abort)) break;

            // ---------------- phase O: blocked scan ----------------
            const bool want_final = last && p.state_out != nullptr;
            for (int b = 0; b < nblk; ++b) {
                const int row0 = tok0 + b * BLK;
                const int valid = min(BLK, tok1 - row0);
                const bool update = (b < nblk - 1) || want_final;
                // a3: P = bf16(Sc ⊙ M), inclusive causal mask inside the block
                if (!warp_wait(&cb->sc_full, blk_n & 1, p, cb)) { ok = false; break; }
                tc_fence_after();
#pragma unroll 1
                for (int c = 0; c < BLK / 32; ++c) {
                    uint32_t x[32];
                    tmem_ld32(trow + TM_SC + c * 32, x);
                    tmem_wait_ld();
                    uint32_t pk[16];
#pragma unroll
                    for (int w = 0; w < 16; ++w) {
                        const int s0 = c * 32 + 2 * w;
                        const float a0 = (s0 <= r) ? __uint_as_float(x[2 * w]) : 0.f;
                        const float a1 = (s0 + 1 <= r) ? __uint_as_float(x[2 * w + 1]) : 0.f;
                        pk[w] = pack_bf16x2(a0, a1);
                    }
                    tmem_st16(trow + TM_P + c * 16, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&cb->p_full);
                if (update) {
                    if (!warp_wait(&cb->s_done, upd_n & 1, p, cb)) { ok = false; break; }
                    ++upd_n;
                    tc_fence_after();
                    if (b < nblk - 1) {
                        // snapshot S_{<b+1} as bf16 hi + lo for the next block's a5
                        if (!warp_wait(&cb->snap_empty, (snap_n & 1) ^ 1, p, cb)) { ok = false; break; }
#pragma unroll 1
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t x[32];
                            tmem_ld32(trow + TM_S + c * 32, x);
                            tmem_wait_ld();
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                uint32_t hv[4], lv[4];
#pragma unroll
                                for (int w = 0; w < 4; ++w) {
                                    const float x0 = __uint_as_float(x[8 * q + 2 * w]);
                                    const float x1 = __uint_as_float(x[8 * q + 2 * w + 1]);
                                    const __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
                                    hv[w] = pack_bf16x2(__bfloat162float(h0), __bfloat162float(h1));
                                    lv[w] = pack_bf16x2(x0 - __bfloat162float(h0), x1 - __bfloat162float(h1));
                                }
                                const uint32_t off = sw_off(r, c * 4 + q);
                                *reinterpret_cast<uint4 *>(shi + off) = make_uint4(hv[0], hv[1], hv[2], hv[3]);
                                *reinterpret_cast<uint4 *>(slo + off) = make_uint4(lv[0], lv[1], lv[2], lv[3]);
                            }
                        }
                        fence_proxy_async_smem();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&cb->snap_full);
                        ++snap_n;
                    } else {
                        // final state of the sequence -> state_out (row-major fp32)
                        float *so = p.state_out + ((size_t)seq * H + h) * D * D + (size_t)r * D;
#pragma unroll 1
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t x[32];
                            tmem_ld32(trow + TM_S + c * 32, x);
                            tmem_wait_ld();
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                *reinterpret_cast<float4 *>(so + c * 32 + 4 * q) =
                                    make_float4(__uint_as_float(x[4 * q]), __uint_as_float(x[4 * q + 1]),
                                                __uint_as_float(x[4 * q + 2]), __uint_as_float(x[4 * q + 3]));
                        }
                    }
                }
                // a7: O -> out
                if (!warp_wait(&cb->o_full, blk_n & 1, p, cb)) { ok = false; break; }
                tc_fence_after();
                const size_t orow = ((size_t)(row0 + r) * H + h) * D;
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t x[32];
                    tmem_ld32(trow + TM_O + c * 32, x);
                    tmem_wait_ld();
                    if (r < valid) {
                        if (p.out_fp32) {
                            float *o = reinterpret_cast<float *>(p.out) + orow + c * 32;
#pragma unroll
                            for (int q = 0; q < 8; ++q)
                                __stcs(reinterpret_cast<float4 *>(o + 4 * q),
                                       make_float4(__uint_as_float(x[4 * q]), __uint_as_float(x[4 * q + 1]),
                                                   __uint_as_float(x[4 * q + 2]), __uint_as_float(x[4 * q + 3])));
                        } else {
                            __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(p.out) + orow + c * 32;
#pragma unroll
                            for (int q = 0; q < 4; ++q) {
                                uint4 u;
                                u.x = pack_bf16x2(__uint_as_float(x[8 * q]), __uint_as_float(x[8 * q + 1]));
                                u.y = pack_bf16x2(__uint_as_float(x[8 * q + 2]), __uint_as_float(x[8 * q + 3]));
                                u.z = pack_bf16x2(__uint_as_float(x[8 * q + 4]), __uint_as_float(x[8 * q + 5]));
                                u.w = pack_bf16x2(__uint_as_float(x[8 * q + 6]), __uint_as_float(x[8 * q + 7]));
                                __stcs(reinterpret_cast<uint4 *>(o + 8 * q), u);
                            }
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&cb->o_empty);
                ++blk_n;
            }
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
            const int t0 = a + jj * s.seg_len;
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
    // 4. empty sequences: the final state is the carried-in state
    if (s.state_out) {
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
