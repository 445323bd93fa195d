// la_decode.cuh -- fused batched decode step on a persistent fp32 state.
//
// "MiniMax-01技术报告解读", §3.3 items 1-2: length-1 tokens run in a kernel of
// their own whose KV computation is fused with the update of the prefix-KV
// cache.  For every (b, h):  S <- S + k^T v  (in place),  o = q S  (inclusive);
// with a per-head decay lambda_h (the decayed recurrence, read from §3.3
// item 1's decay computation):  S <- lambda_h S + k^T v.
//
// The step is a pure stream over the state (read 64 KiB, write 64 KiB per
// (b, h) at d = 128), so the kernel is built for HBM bandwidth: one CTA of
// 256 threads per (b, h) pair; thread (row group g = tid/32, column quad
// c = tid%32) owns rows g, g+8, ..., g+120 and columns 4c..4c+3, so every warp
// instruction moves one contiguous 512-byte state row.  All 16 row loads are
// issued before any arithmetic (16 x 16 B in flight per thread), with
// streaming (evict-first) cache hints since the state is touched once per
// step.  The per-column partial sums of o are reduced across the 8 row groups
// through shared memory.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace la {

constexpr int DEC_THREADS = 256;
constexpr int DEC_ROWS_PER_THREAD = 16;  // 128 rows / 8 row groups

__device__ __forceinline__ float4 ld_stream_f4(const float *p) {
    float4 v;
    asm volatile("ld.global.cs.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
    return v;
}
__device__ __forceinline__ void st_stream_f4(float *p, float4 v) {
    asm volatile("st.global.cs.v4.f32 [%0], {%1,%2,%3,%4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z),
                 "f"(v.w) : "memory");
}

// Row b of q/k/v/out updates state b, or, with `slots`, state slots[b] of a
// pool of n_slots (sequence, H heads) states; a slot outside [0, n_slots)
// skips the row and records LA_ERR_INVALID_ARGUMENT in the status word.
__global__ void __launch_bounds__(DEC_THREADS)
la_decode_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ k,
                 const __nv_bfloat16 *__restrict__ v, float *__restrict__ state, void *__restrict__ out,
                 int out_fp32, long long npairs, int H, const int *__restrict__ slots, int n_slots,
                 const float *__restrict__ decay, int *status) {
    constexpr int Dd = 128;
    __shared__ float red[8][Dd];
    __shared__ float qs[Dd], ks[Dd];
    const int tid = threadIdx.x;
    const int g = tid >> 5, c = tid & 31;
    for (long long pair = blockIdx.x; pair < npairs; pair += gridDim.x) {
        const size_t vec = (size_t)pair * Dd;
        long long spair = pair;
        if (slots) {
            const long long b = pair / H;
            const int slot = slots[b];
            if (slot < 0 || slot >= n_slots) {  // uniform across the block
                if (tid == 0 && pair % H == 0) atomicCAS(status, 0, 1);
                continue;
            }
            spair = (long long)slot * H + (pair - b * H);
        }
        // per-head decay lambda (1 without decay): S <- lambda S + k^T v
        float lam = 1.f;
        if (decay) {
            lam = decay[pair % H];
            if (!(lam > 0.f && lam <= 1.f)) {  // uniform across the block; also rejects NaN
                if (tid == 0) atomicCAS(status, 0, 1);
                continue;
            }
        }
        float *S = state + (size_t)spair * Dd * Dd;
        float4 s[DEC_ROWS_PER_THREAD];
#pragma unroll
        for (int m = 0; m < DEC_ROWS_PER_THREAD; ++m)
            s[m] = ld_stream_f4(S + (size_t)(g + 8 * m) * Dd + 4 * c);
        if (tid < Dd) {
            qs[tid] = __bfloat162float(q[vec + tid]);
            ks[tid] = __bfloat162float(k[vec + tid]);
        }
        const __nv_bfloat162 *v2 = reinterpret_cast<const __nv_bfloat162 *>(v + vec + 4 * c);
        const float2 va = __bfloat1622float2(v2[0]), vb = __bfloat1622float2(v2[1]);
        __syncthreads();
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int m = 0; m < DEC_ROWS_PER_THREAD; ++m) {
            const int i = g + 8 * m;
            const float ki = ks[i], qi = qs[i];
            float4 x = s[m];
            x.x = fmaf(ki, va.x, lam * x.x);  // S[i][j] = lambda S[i][j] + k_i v_j
            x.y = fmaf(ki, va.y, lam * x.y);
            x.z = fmaf(ki, vb.x, lam * x.z);
            x.w = fmaf(ki, vb.y, lam * x.w);
            st_stream_f4(S + (size_t)i * Dd + 4 * c, x);
            acc.x = fmaf(qi, x.x, acc.x);  // o_j += q_i S'[i][j]
            acc.y = fmaf(qi, x.y, acc.y);
            acc.z = fmaf(qi, x.z, acc.z);
            acc.w = fmaf(qi, x.w, acc.w);
        }
        *reinterpret_cast<float4 *>(&red[g][4 * c]) = acc;
        __syncthreads();
        if (tid < Dd) {
            float o = 0.f;
#pragma unroll
            for (int gg = 0; gg < 8; ++gg) o += red[gg][tid];
            if (out_fp32)
                reinterpret_cast<float *>(out)[vec + tid] = o;
            else
                reinterpret_cast<__nv_bfloat16 *>(out)[vec + tid] = __float2bfloat16_rn(o);
        }
        __syncthreads();
    }
}

}  // namespace la
