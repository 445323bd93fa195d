// la_aggregate.cuh -- the two device steps of sequence parallelism across
// ranks ("MiniMax-01技术报告解读", §3.2 item 3, LASP+):
//
//   local prefix   A_r = sum over this rank's tokens of k_t^T v_t, per
//                  (sequence, head)                     la_kv_aggregate_kernel
//                                                       + la_agg_reduce_kernel
//   global prefix  P_r = S_in + sum_{i<r} A_i, from the gathered A_i
//                                                       la_state_prefix_kernel
//
// The exchange between them (an AllGather of the A_r) is the caller's
// collective; the local scan that follows is la_prefill seeded with P_r.
//
// la_kv_aggregate_kernel: the (sequence, head) pairs are laid end to end as a
// list of 128-row blocks, pair by pair, and the list is cut into equal
// contiguous ranges, one per CTA, so every CTA streams the same number of
// K and V tiles (one wave, no tail).  A CTA accumulates K_b^T V_b in TMEM
// (fp32, tcgen05, both operands MN-major -- no transpose) over each run of
// blocks that belongs to one pair (a "piece").  A piece that covers its whole
// pair is written straight to the output; a piece cut by a range boundary can
// only be the first or the last piece of its CTA's range, and goes to one of
// the CTA's two partial slots.  la_agg_reduce_kernel then sums, for every pair
// that was cut, its partials in range order, so the result does not depend
// on timing.
//
// Warp roles (192 threads):
//   warp 0      TMA producer (lane 0): K and V tiles into a three-stage ring
//   warp 1      TMEM allocator + MMA issuer (elect.sync picks the issuing lane)
//   warps 2-5   read-out: TMEM -> registers -> fp32 rows in global memory
// Two TMEM accumulators (columns [0,128) and [128,256)) let the read-out of
// one piece overlap the MMAs of the next.
#pragma once
#include "la_prefill.cuh"

namespace la {

constexpr int AGG_STAGES = 3;
constexpr int AGG_THREADS = 192;
constexpr int AGG_CTAS = 148;  // ranges per launch (one wave on a B200)
constexpr int AGG_SM_K = 0;
constexpr int AGG_SM_V = AGG_SM_K + AGG_STAGES * TILE_BYTES;
constexpr int AGG_SM_CTRL = AGG_SM_V + AGG_STAGES * TILE_BYTES;  // 196608
constexpr int AGG_SMEM = AGG_SM_CTRL + 1024 + 1024;              // + alignment slack
constexpr uint32_t AGG_TM_COLS = 256;

struct AggParams {
    float *out;               // [npairs][D*D] row-major fp32
    float *partial;           // [2 * ctas][D*D]
    int N;                    // tokens per sequence
    int H;
    int nblk;                 // row blocks per sequence, ceil(N / BLK)
    long long total;          // npairs * nblk
    long long per_cta;        // blocks per CTA range
    unsigned long long wait_limit_ns;
    int *status;
};

struct AggCtrl {
    uint64_t full[AGG_STAGES];   // [1] producer expect_tx
    uint64_t empty[AGG_STAGES];  // [1] MMA commit
    uint64_t acc_full[2];        // [1] MMA commit: a piece's sum is in accumulator a
    uint64_t acc_empty[2];       // [4] read-out warps: accumulator a is in registers
    uint64_t fin;                // [1] tear-down: every MMA done
    uint32_t tmem_base;
    volatile int abort;
};
static_assert(sizeof(AggCtrl) <= 1024, "control block too large");

__device__ __forceinline__ bool agg_wait(uint64_t *bar, uint32_t parity, const AggParams &p, AggCtrl *cb) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t deadline = globaltimer_ns() + p.wait_limit_ns;
    if (la_wait(bar, parity, deadline, &cb->abort)) return true;
    cb->abort = 1;
    record_status(p.status, ST_TIMEOUT);
    return false;
}

__device__ __forceinline__ bool agg_warp_wait(uint64_t *bar, uint32_t parity, const AggParams &p, AggCtrl *cb) {
    return __all_sync(0xffffffffu, agg_wait(bar, parity, p, cb)) != 0;
}

__global__ void __launch_bounds__(AGG_THREADS, 1)
la_kv_aggregate_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                       const __grid_constant__ AggParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                ~static_cast<uintptr_t>(1023));
    AggCtrl *cb = reinterpret_cast<AggCtrl *>(smem + AGG_SM_CTRL);
    const int warp = __shfl_sync(0xffffffffu, (int)(threadIdx.x >> 5), 0), lane = threadIdx.x & 31;
    const uint32_t sbase = smem_u32(smem);

    if (threadIdx.x == 0) {
        for (int s = 0; s < AGG_STAGES; ++s) {
            mbar_init(&cb->full[s], 1);
            mbar_init(&cb->empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&cb->acc_full[a], 1);
            mbar_init(&cb->acc_empty[a], 4);
        }
        mbar_init(&cb->fin, 1);
        cb->abort = 0;
        fence_mbarrier_init();
        tma_prefetch_desc(&tmk);
        tma_prefetch_desc(&tmv);
    }
    if (warp == 1) {
        tmem_alloc(&cb->tmem_base, AGG_TM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = __shfl_sync(0xffffffffu, cb->tmem_base, 0);
    const long long g0 = (long long)blockIdx.x * p.per_cta;
    const long long g1 = min(g0 + p.per_cta, p.total);
    const int nblk = p.nblk;

    if (warp == 0) {
        // ===================== producer =====================
        if (lane == 0) {
            const uint64_t pol = policy_evict_first();
            uint32_t n = 0;
            int last_fill[AGG_STAGES];
            for (int s = 0; s < AGG_STAGES; ++s) last_fill[s] = -1;
            bool ok = true;
            for (long long g = g0; g < g1; ++g) {
                if (cb->abort) { ok = false; break; }
                const long long pair = g / nblk;
                const int b = (int)(g - pair * nblk);
                const int seq = (int)(pair / p.H), h = (int)(pair % p.H);
                const int s = n % AGG_STAGES;
                if (!agg_wait(&cb->empty[s], ((n / AGG_STAGES) & 1) ^ 1, p, cb)) { ok = false; break; }
                mbar_expect_tx(&cb->full[s], 2 * TILE_BYTES);
                const int row = seq * p.N + b * BLK;
                tma_load_4d(smem + AGG_SM_K + s * TILE_BYTES, &tmk, &cb->full[s], 0, h, row, 0, pol);
                tma_load_4d(smem + AGG_SM_V + s * TILE_BYTES, &tmv, &cb->full[s], 0, h, row, 0, pol);
                last_fill[s] = (int)(n / AGG_STAGES);
                ++n;
            }
            // every issued copy must land before the CTA exits
            for (int s = 0; s < AGG_STAGES; ++s)
                if (last_fill[s] >= 0) {
                    const uint64_t dl = globaltimer_ns() + p.wait_limit_ns;
                    int dummy = 0;
                    la_wait(&cb->full[s], last_fill[s] & 1, dl, &dummy);
                }
            if (!ok) cb->abort = 1;
        }
    } else if (warp == 1) {
        // ===================== MMA issuer =====================
        constexpr uint32_t ID_KV = idesc_bf16_f32(D, D, 1, 1);  // K^T (MN) x V (MN)
        uint32_t n = 0, piece_n = 0;
        bool ok = true;
        for (long long g = g0; g < g1 && ok;) {
            const long long pair = g / nblk;
            const long long pend = min(g1, (pair + 1) * nblk);
            const int acc = piece_n & 1;
            if (!agg_warp_wait(&cb->acc_empty[acc], ((piece_n >> 1) & 1) ^ 1, p, cb)) { ok = false; break; }
            tc_fence_after();
            for (long long gg = g; gg < pend; ++gg) {
                if (__any_sync(0xffffffffu, cb->abort != 0)) { ok = false; break; }
                const int s = n % AGG_STAGES;
                if (!agg_warp_wait(&cb->full[s], (n / AGG_STAGES) & 1, p, cb)) { ok = false; break; }
                const int b = (int)(gg - pair * nblk);
                const int valid = min(BLK, p.N - b * BLK);
                uint8_t *kp = smem + AGG_SM_K + s * TILE_BYTES;
                uint8_t *vp = smem + AGG_SM_V + s * TILE_BYTES;
                if (valid < BLK) {
                    // rows past the end of the sequence hold the next sequence's
                    // tokens (or TMA zero fill): zero them in K and V
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
                const uint32_t kt = sbase + AGG_SM_K + s * TILE_BYTES;
                const uint32_t vt = sbase + AGG_SM_V + s * TILE_BYTES;
#pragma unroll
                for (int kk = 0; kk < BLK / 16; ++kk)
                    mma_ss_w(tmem + acc * 128, desc_mnmajor(kt, kk), desc_mnmajor(vt, kk), ID_KV,
                             (gg > g || kk > 0) ? 1u : 0u);
                tc_commit_w(&cb->empty[s]);
                ++n;
            }
            if (!ok) break;
            tc_commit_w(&cb->acc_full[acc]);
            ++piece_n;
            g = pend;
        }
        if (!ok) cb->abort = 1;
        // tear-down: all MMAs issued by this warp must finish before TMEM is freed
        __syncwarp();
        tc_commit_w(&cb->fin);
        if (lane == 0) {
            const uint64_t dl = globaltimer_ns() + p.wait_limit_ns;
            int dummy = 0;
            la_wait(&cb->fin, 0, dl, &dummy);
        }
        __syncwarp();
    } else {
        // ===================== warps 2-5: read-out =====================
        const int q4 = warp & 3;  // TMEM lane quarter this warp may access
        const int r = q4 * 32 + lane;  // row of the d_k x d_v sum
        const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16);
        uint32_t piece_n = 0;
        for (long long g = g0; g < g1;) {
            const long long pair = g / nblk;
            const long long pend = min(g1, (pair + 1) * nblk);
            const bool whole = g == pair * nblk && pend == (pair + 1) * nblk;
            const int acc = piece_n & 1;
            if (!agg_warp_wait(&cb->acc_full[acc], (piece_n >> 1) & 1, p, cb)) break;
            tc_fence_after();
            float *dst = whole ? p.out + (size_t)pair * D * D
                               : p.partial + (size_t)(2 * blockIdx.x + (g == g0 ? 0 : 1)) * D * D;
            dst += (size_t)r * D;
#pragma unroll 1
            for (int qq = 0; qq < 4; ++qq) {
                uint32_t x[32];
                tmem_ld_wait32(trow + acc * 128 + qq * 32, x);
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<float4 *>(dst + qq * 32 + 4 * c) =
                        make_float4(__uint_as_float(x[4 * c]), __uint_as_float(x[4 * c + 1]),
                                    __uint_as_float(x[4 * c + 2]), __uint_as_float(x[4 * c + 3]));
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&cb->acc_empty[acc]);
            ++piece_n;
            g = pend;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, AGG_TM_COLS);
}

// Sum the partial pieces of every pair that a range boundary cut, in range
// order; pairs of zero-length sequences get a zero sum.  Grid: (npairs,
// AGG_RED_SLICES); each block covers D*D / AGG_RED_SLICES elements of one pair.
constexpr int AGG_RED_THREADS = 256;
constexpr int AGG_RED_SLICES = 8;

__global__ void __launch_bounds__(AGG_RED_THREADS)
la_agg_reduce_kernel(float *out, const float *partial, int nblk, long long per_cta) {
    const long long pair = blockIdx.x;
    constexpr int SLICE4 = D * D / 4 / AGG_RED_SLICES;  // float4s per block
    const size_t base4 = (size_t)pair * (D * D / 4) + (size_t)blockIdx.y * SLICE4;
    float4 *o = reinterpret_cast<float4 *>(out) + base4;
    if (nblk == 0) {
        for (int e = threadIdx.x; e < SLICE4; e += AGG_RED_THREADS) o[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        return;
    }
    const long long first = pair * nblk, last = first + nblk - 1;
    const long long c0 = first / per_cta, c1 = last / per_cta;
    if (c0 == c1) return;  // one CTA held the whole pair and wrote it directly
    const float4 *part = reinterpret_cast<const float4 *>(partial) + (size_t)blockIdx.y * SLICE4;
    for (int e = threadIdx.x; e < SLICE4; e += AGG_RED_THREADS) {
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (long long c = c0; c <= c1; ++c) {
            // the pair is the first piece of range c iff the range starts inside it
            const long long slot = 2 * c + ((c * per_cta) / nblk == pair ? 0 : 1);
            const float4 x = part[(size_t)slot * (D * D / 4) + e];
            acc.x += x.x;
            acc.y += x.y;
            acc.z += x.z;
            acc.w += x.w;
        }
        o[e] = acc;
    }
}

// out = (state_in or 0) + parts[0] + ... + parts[count-1], elementwise in that
// order; every array holds n4 float4s.  out may alias state_in.
constexpr int PREFIX_THREADS = 256;

__global__ void __launch_bounds__(PREFIX_THREADS)
la_state_prefix_kernel(const float4 *__restrict__ parts, int count, const float4 *state_in, float4 *out,
                       long long n4) {
    for (long long e = (long long)blockIdx.x * PREFIX_THREADS + threadIdx.x; e < n4;
         e += (long long)gridDim.x * PREFIX_THREADS) {
        float4 acc = state_in ? state_in[e] : make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i = 0; i < count; ++i) {
            const float4 x = parts[(size_t)i * n4 + e];
            acc.x += x.x;
            acc.y += x.y;
            acc.z += x.z;
            acc.w += x.w;
        }
        out[e] = acc;
    }
}

// out[s] = in[s]^T for nstates D x D fp32 matrices (32 x 32 tiles through
// shared memory; grid (nstates, (D/32)^2), 32 x 8 threads).
constexpr int TRANSPOSE_TILE = 32;

__global__ void __launch_bounds__(256)
la_state_transpose_kernel(const float *__restrict__ in, float *__restrict__ out) {
    __shared__ float tile[TRANSPOSE_TILE][TRANSPOSE_TILE + 1];
    constexpr int TILES = D / TRANSPOSE_TILE;
    const size_t base = (size_t)blockIdx.x * D * D;
    const int ti = blockIdx.y / TILES, tj = blockIdx.y % TILES;  // tile row / column of `in`
    const int x = threadIdx.x & 31, y0 = threadIdx.x >> 5;
    for (int y = y0; y < TRANSPOSE_TILE; y += 8)
        tile[y][x] = in[base + (size_t)(ti * TRANSPOSE_TILE + y) * D + tj * TRANSPOSE_TILE + x];
    __syncthreads();
    for (int y = y0; y < TRANSPOSE_TILE; y += 8)
        out[base + (size_t)(tj * TRANSPOSE_TILE + y) * D + ti * TRANSPOSE_TILE + x] = tile[x][y];
}

}  // namespace la
