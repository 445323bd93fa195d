// la_lib.cu -- C ABI of the Lightning Attention library (declared in
// include/lightning_attn.h): argument checks, workspace partitioning, TMA
// tensor-map encoding and kernel launches.  Everything is one translation unit
// so that the sticky device status word is a plain __device__ variable.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "lightning_attn.h"
#include "la_aggregate.cuh"
#include "la_decode.cuh"
#include "la_prefill.cuh"

namespace {

__device__ int g_la_status;  // sticky per-device status word (0 = OK)

std::atomic<unsigned long long> g_wait_limit_ns{2000000000ull};
std::atomic<int> g_seg_len_override{0};
std::atomic<int> g_inject{0};
std::atomic<int> g_last_seg_len{0};
std::atomic<unsigned long long> g_launches{0};

constexpr unsigned long long kDefaultWaitNs = 2000000000ull;

// ---------------------------------------------------------------------------
// driver entry point for cuTensorMapEncodeTiled (no link-time libcuda dependency)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// [T, H, 128] bf16 viewed as a 4-D tensor {64, H, T, 2}: dimension 0 = the
// 64 features of one half, 1 = head (256-byte stride), 2 = token (H*256-byte
// stride), 3 = which half (128-byte stride).  A box {64, 1, 128, 2} loads both
// halves of 128 tokens as two [128 x 64] blocks with the 128-byte swizzle; zero
// fill outside the tensor.
bool encode_qkv_map(CUtensorMap *map, const void *base, int T, int H) {
    EncodeTiledFn fn = get_encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {64, (cuuint64_t)H, (cuuint64_t)T, 2};
    const cuuint64_t strides[3] = {(cuuint64_t)la::D * 2, (cuuint64_t)H * la::D * 2, 128};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)la::BLK, 2};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int device_sm_count() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0)
        return 148;
    return sms;
}

inline bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Segment length of the cross-SM scan.  Depends on the problem only (not on
// the device) so that the workspace size is a pure function of the shape.
int choose_seg_len(int nseq, long long T, int H, int block = 0) {
    // with 256-token row blocks a segment holds whole blocks
    const int ov = g_seg_len_override.load();
    if (ov > 0) return (block == 256 && ov % 256) ? ov + la::BLK : ov;
    // Longer segments for few heads: each (sequence, head) scan then has fewer
    // cross-SM hand-offs in its chain (measured at H = 8, N = 1M: 6.2 / 3.3 /
    // 2.5 / 2.5 / 2.7 ms for 1024 / 2048 / 4096 / 8192 / 16384 tokens).
    int L = (H <= 16) ? 4096 : 1024;
    const long long target = 2 * 148;  // want at least ~2 items per SM of a B200
    while (L > la::BLK) {
        const long long segs = (T + L - 1) / L + 0;  // lower bound of segments over all sequences
        if (segs * (long long)H >= target) break;
        L /= 2;
    }
    (void)nseq;
    return (block == 256 && L % 256) ? L + la::BLK : L;
}

struct WsLayout {
    size_t hdr, segs, flags, incl, total;
    long long gmax;
};

WsLayout ws_layout(long long gmax, int H) {
    WsLayout w;
    w.gmax = gmax;
    w.hdr = 0;
    w.segs = la::HDR_BYTES;
    w.flags = w.segs + round_up((size_t)gmax * sizeof(int4), 256);
    w.incl = w.flags + round_up((size_t)gmax * H * sizeof(int), 256);
    w.total = w.incl + (size_t)gmax * H * la::D * la::D * sizeof(float);
    return w;
}

// Upper bound of the number of segments of a packed batch: every sequence
// boundary can add one partial segment.
long long gmax_for(int nseq, long long T, int L) { return (T + L - 1) / L + nseq; }

// Exact number of segments of B equal-length sequences of N tokens.
long long gmax_fixed(int B, long long N, int L) { return (long long)B * ((N + L - 1) / L); }

// Dynamic shared-memory limits are a property of each device's context, so the
// attribute is set once per device (and again on a device that has not seen it).
constexpr int kMaxDevices = 64;

struct SmemAttr {
    std::mutex mu;
    bool done[kMaxDevices] = {};
};

template <typename Kernel>
la_status ensure_smem_attr(SmemAttr &a, Kernel *kernel, int bytes) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return LA_ERR_CUDA;
    if (dev >= kMaxDevices) {  // not cached: set it on every call
        return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess
                   ? LA_OK : LA_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(a.mu);
    if (!a.done[dev]) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
            return LA_ERR_CUDA;
        a.done[dev] = true;
    }
    return LA_OK;
}

SmemAttr g_attr_prefill, g_attr_prefill_pair, g_attr_prefill_decay, g_attr_prefill_b64,
    g_attr_prefill_b256, g_attr_agg;

bool ranges_overlap(const void *a, size_t na, const void *b, size_t nb) {
    if (!a || !b || na == 0 || nb == 0) return false;
    const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

la_status check_common(int H, int d, int block, la_dtype out_dtype) {
    if (H <= 0 || d <= 0 || block < 0) return LA_ERR_INVALID_ARGUMENT;
    if (out_dtype != LA_BF16 && out_dtype != LA_FP32) return LA_ERR_INVALID_ARGUMENT;
    if (d != la::D) return LA_ERR_UNSUPPORTED;
    if (block != 0 && block != 64 && block != la::BLK && block != 256) return LA_ERR_UNSUPPORTED;
    return LA_OK;
}

// The prefill kernel instantiation for a row-block length (0 = 128); with
// mq2, the paired reversed sweep that also runs (q2, v, k).
template <bool DECAY>
la_status launch_prefill(int block, int grid, const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                         const la::PrefillParams &pp, cudaStream_t stream, const CUtensorMap *mq2 = nullptr);

// Shared body of la_prefill / la_prefill_varlen.
la_status prefill_impl(const void *q, const void *k, const void *v, const int *cu, int fixed_len,
                       int nseq, long long T, int max_seqlen, int H, int d, int block,
                       const float *state_in, void *out, la_dtype out_dtype, float *state_out,
                       void *workspace, size_t ws_bytes, cudaStream_t stream,
                       const int *slots = nullptr, int n_slots = 0,
                       const float *decay = nullptr, const void *q2 = nullptr, void *out2 = nullptr,
                       bool rev = false) {
    la_status st = check_common(H, d, block, out_dtype);
    if (st != LA_OK) return st;
    if (nseq < 0 || T < 0 || max_seqlen < 0) return LA_ERR_INVALID_ARGUMENT;
    if (T > 0x7fffffffLL) return LA_ERR_INVALID_ARGUMENT;
    if (nseq == 0) return T == 0 ? LA_OK : LA_ERR_INVALID_ARGUMENT;
    if (T > 0 && (!q || !k || !v || !out)) return LA_ERR_INVALID_ARGUMENT;
    const void *ptrs[6] = {q, k, v, out, state_in, state_out};
    for (const void *p : ptrs)
        if (p && !aligned(p, 16)) return LA_ERR_INVALID_ARGUMENT;
    const size_t esz = out_dtype == LA_FP32 ? 4 : 2;
    const size_t n_in = (size_t)T * H * la::D * 2, n_out = (size_t)T * H * la::D * esz;
    if (slots && (n_slots <= 0 || !aligned(slots, 4) || state_in != state_out || !state_out))
        return LA_ERR_INVALID_ARGUMENT;
    if (decay && !aligned(decay, 4)) return LA_ERR_INVALID_ARGUMENT;
    if ((block == 64 || block == 256) && decay) return LA_ERR_UNSUPPORTED;
    // paired problems (q, k, v) and (q2, v, k) in a reversed sweep
    if ((q2 != nullptr) != (out2 != nullptr) || (q2 != nullptr) != rev) return LA_ERR_INVALID_ARGUMENT;
    if (q2 && (decay || (block != 0 && block != la::BLK) || slots)) return LA_ERR_UNSUPPORTED;
    const size_t n_state = (size_t)(slots ? n_slots : nseq) * H * la::D * la::D * 4;
    if (state_out && state_out != state_in && ranges_overlap(state_out, n_state, state_in, n_state))
        return LA_ERR_INVALID_ARGUMENT;
    const void *ins[3] = {q, k, v};
    for (const void *p : ins) {
        if (ranges_overlap(out, n_out, p, n_in)) return LA_ERR_INVALID_ARGUMENT;
        if (ranges_overlap(state_out, n_state, p, n_in)) return LA_ERR_INVALID_ARGUMENT;
    }
    if (ranges_overlap(out, n_out, state_out, n_state) || ranges_overlap(out, n_out, state_in, n_state))
        return LA_ERR_INVALID_ARGUMENT;
    if (q2) {
        if (!aligned(q2, 16) || !aligned(out2, 16)) return LA_ERR_INVALID_ARGUMENT;
        if (ranges_overlap(out2, n_out, out, n_out) || ranges_overlap(out2, n_out, state_in, n_state) ||
            ranges_overlap(out2, n_out, q2, n_in) || ranges_overlap(out, n_out, q2, n_in))
            return LA_ERR_INVALID_ARGUMENT;
        for (const void *p : ins)
            if (ranges_overlap(out2, n_out, p, n_in)) return LA_ERR_INVALID_ARGUMENT;
    }

    const int L = choose_seg_len(nseq, T, H, block);
    if (L <= 0 || L % la::BLK) return LA_ERR_INVALID_ARGUMENT;
    const long long gmax = cu ? gmax_for(nseq, T, L) : gmax_fixed(nseq, fixed_len, L);
    const WsLayout w = ws_layout(gmax, H);
    if (!workspace || ws_bytes < w.total) return LA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return LA_ERR_INVALID_ARGUMENT;
    if (gmax * (long long)H > 0x7fffffffLL) return LA_ERR_UNSUPPORTED;
    if (ranges_overlap(workspace, w.total, out, n_out)) return LA_ERR_INVALID_ARGUMENT;
    g_last_seg_len = L;

    int *status = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void **>(&status), g_la_status) != cudaSuccess)
        return LA_ERR_CUDA;
    uint8_t *ws = static_cast<uint8_t *>(workspace);

    la::ScheduleParams sp;
    sp.cu = cu;
    sp.fixed_len = fixed_len;
    sp.nseq = nseq;
    sp.T = (int)T;
    sp.max_seqlen = max_seqlen;
    sp.H = H;
    sp.seg_len = L;
    sp.Gmax = (int)gmax;
    sp.hdr = reinterpret_cast<int *>(ws + w.hdr);
    sp.segs = reinterpret_cast<int4 *>(ws + w.segs);
    sp.flags = reinterpret_cast<int *>(ws + w.flags);
    sp.state_in = state_in;
    sp.state_out = state_out;
    sp.slots = slots;
    sp.n_slots = n_slots;
    sp.decay = decay;
    sp.reverse = rev ? 1 : 0;
    sp.status = status;
    la::la_schedule_kernel<<<1, la::SCHED_THREADS, 0, stream>>>(sp);
    if (cudaGetLastError() != cudaSuccess) return LA_ERR_CUDA;
    ++g_launches;
    if (T == 0) return LA_OK;

    CUtensorMap mq, mk, mv, mq2;
    if (!encode_qkv_map(&mq, q, (int)T, H) || !encode_qkv_map(&mk, k, (int)T, H) ||
        !encode_qkv_map(&mv, v, (int)T, H) || (q2 && !encode_qkv_map(&mq2, q2, (int)T, H)))
        return LA_ERR_CUDA;

    la::PrefillParams pp;
    pp.state_in = state_in;
    pp.state_out = state_out;
    pp.slots = slots;
    pp.out = out;
    pp.out2 = out2;
    pp.out_fp32 = out_dtype == LA_FP32;
    pp.out_al32 = aligned(out, 32) && (!out2 || aligned(out2, 32));
    pp.H = H;
    pp.hdr = sp.hdr;
    pp.segs = sp.segs;
    pp.flags = sp.flags;
    pp.incl = reinterpret_cast<float *>(ws + w.incl);
    pp.wait_limit_ns = g_wait_limit_ns.load();
    pp.inject = g_inject.load();
    pp.decay = decay;
    pp.seg_len = L;
    pp.status = status;

    const long long items = gmax * (long long)H;
    const int grid = (int)(items < device_sm_count() ? items : device_sm_count());
    st = decay ? launch_prefill<true>(block, grid, mq, mk, mv, pp, stream)
               : launch_prefill<false>(block, grid, mq, mk, mv, pp, stream, q2 ? &mq2 : nullptr);
    if (st != LA_OK) return st;
    ++g_launches;
    return LA_OK;
}

template <bool DECAY, int BK, bool PAIR = false, bool REV = false>
la_status launch_prefill_bk(SmemAttr &attr, int grid, const CUtensorMap &mq, const CUtensorMap &mk,
                            const CUtensorMap &mv, const la::PrefillParams &pp, cudaStream_t stream,
                            const CUtensorMap *mq2 = nullptr) {
    la_status st = ensure_smem_attr(attr, la::la_prefill_kernel<DECAY, BK, PAIR, REV>, la::PREFILL_SMEM);
    if (st != LA_OK) return st;
    // (unpaired instantiations never read the fourth map)
    la::la_prefill_kernel<DECAY, BK, PAIR, REV><<<grid, la::PREFILL_THREADS, la::PREFILL_SMEM, stream>>>(
        mq, mk, mv, mq2 ? *mq2 : mq, pp);
    return cudaGetLastError() == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

template <bool DECAY>
la_status launch_prefill(int block, int grid, const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                         const la::PrefillParams &pp, cudaStream_t stream, const CUtensorMap *mq2) {
    if (!DECAY && mq2)  // the paired reversed sweep
        return launch_prefill_bk<false, 128, true, true>(g_attr_prefill_pair, grid, mq, mk, mv, pp, stream, mq2);
    if (DECAY) return launch_prefill_bk<true, 128>(g_attr_prefill_decay, grid, mq, mk, mv, pp, stream);
    if (block == 64) return launch_prefill_bk<false, 64>(g_attr_prefill_b64, grid, mq, mk, mv, pp, stream);
    if (block == 256) return launch_prefill_bk<false, 256>(g_attr_prefill_b256, grid, mq, mk, mv, pp, stream);
    return launch_prefill_bk<false, 128>(g_attr_prefill, grid, mq, mk, mv, pp, stream);
}

// Shared body of la_decode_step / la_decode_step_slots.
la_status decode_impl(const void *q, const void *k, const void *v, float *state, const int *slots, int n_slots,
                      void *out, la_dtype out_dtype, int B, int H, int d, cudaStream_t stream,
                      const float *decay = nullptr) {
    la_status st = check_common(H, d, 0, out_dtype);
    if (st != LA_OK) return st;
    if (B < 0) return LA_ERR_INVALID_ARGUMENT;
    if (B == 0) return LA_OK;
    if (!q || !k || !v || !state || !out) return LA_ERR_INVALID_ARGUMENT;
    const void *ptrs[5] = {q, k, v, state, out};
    for (const void *p : ptrs)
        if (!aligned(p, 16)) return LA_ERR_INVALID_ARGUMENT;
    if (slots && (n_slots <= 0 || !aligned(slots, 4))) return LA_ERR_INVALID_ARGUMENT;
    if (decay && !aligned(decay, 4)) return LA_ERR_INVALID_ARGUMENT;
    const long long npairs = (long long)B * H;
    const long long nstates = (slots ? (long long)n_slots : (long long)B) * H;
    const size_t esz = out_dtype == LA_FP32 ? 4 : 2;
    if (ranges_overlap(out, npairs * la::D * esz, state, nstates * la::D * la::D * 4))
        return LA_ERR_INVALID_ARGUMENT;
    const long long grid = npairs < (1LL << 30) ? npairs : (1LL << 30);
    int *status = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void **>(&status), g_la_status) != cudaSuccess)
        return LA_ERR_CUDA;
    la::la_decode_kernel<<<(unsigned)grid, la::DEC_THREADS, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
        static_cast<const __nv_bfloat16 *>(v), state, out, out_dtype == LA_FP32, npairs, H, slots, n_slots,
        decay, status);
    if (cudaGetLastError() != cudaSuccess) return LA_ERR_CUDA;
    ++g_launches;
    return LA_OK;
}

// Cut the block list of la_kv_aggregate into equal ranges, one per CTA.
// Depends on the shape only, so the workspace size is a pure function of it.
struct AggPlan {
    long long total = 0, per_cta = 1;
    int ctas = 0;
    int nblk = 0;
};

AggPlan agg_plan(long long npairs, int N) {
    AggPlan a;
    a.nblk = (int)(((long long)N + la::BLK - 1) / la::BLK);
    a.total = npairs * a.nblk;
    if (a.total == 0) return a;
    const long long c = a.total < la::AGG_CTAS ? a.total : la::AGG_CTAS;
    a.per_cta = (a.total + c - 1) / c;
    a.ctas = (int)((a.total + a.per_cta - 1) / a.per_cta);
    return a;
}

size_t agg_ws_bytes(const AggPlan &a) { return (size_t)2 * a.ctas * la::D * la::D * sizeof(float); }

la_status launch_transpose(const float *in, float *out, long long nstates, cudaStream_t stream) {
    if (nstates <= 0) return LA_OK;
    const int tiles = (la::D / la::TRANSPOSE_TILE) * (la::D / la::TRANSPOSE_TILE);
    la::la_state_transpose_kernel<<<dim3((unsigned)nstates, tiles), 256, 0, stream>>>(in, out);
    if (cudaGetLastError() != cudaSuccess) return LA_ERR_CUDA;
    ++g_launches;
    return LA_OK;
}

// Workspace of la_prefill_backward(_varlen): one prefill workspace (reused
// by the two sweeps, which run in stream order) and one [nseq, H, D, D] fp32
// state (S_in transposed).  cu: packed sequences (segment count bounded as
// for la_prefill_varlen), else nseq sequences of fixed_len tokens.
struct BwdLayout {
    size_t prefill, st0, total;
};

BwdLayout bwd_layout(bool packed, int nseq, int fixed_len, long long T, int H) {
    BwdLayout w;
    const int L = choose_seg_len(nseq, T, H);
    const long long gmax = packed ? gmax_for(nseq, T, L) : gmax_fixed(nseq, fixed_len, L);
    const size_t pre = ws_layout(gmax, H).total;
    const size_t st = (size_t)nseq * H * la::D * la::D * sizeof(float);
    w.prefill = 0;
    w.st0 = round_up(pre, 256);
    w.total = w.st0 + st;
    return w;
}

// Shared body of la_prefill_backward and la_prefill_backward_varlen.
la_status backward_impl(const void *q, const void *k, const void *v, const void *dout, const int *cu,
                        int fixed_len, int nseq, long long T, int max_seqlen, int H, int d,
                        const float *state_in, const float *dstate_out, void *dq, void *dk, void *dv,
                        la_dtype grad_dtype, float *dstate_in, void *workspace, size_t ws_bytes,
                        cudaStream_t stream) {
    la_status st = check_common(H, d, 0, grad_dtype);
    if (st != LA_OK) return st;
    if (nseq < 0 || T < 0 || max_seqlen < 0) return LA_ERR_INVALID_ARGUMENT;
    if (nseq == 0) return T == 0 ? LA_OK : LA_ERR_INVALID_ARGUMENT;
    if (T > 0x7fffffffLL) return LA_ERR_INVALID_ARGUMENT;
    if (T > 0 && (!q || !k || !v || !dout || !dq || !dk || !dv)) return LA_ERR_INVALID_ARGUMENT;
    const void *ptrs[10] = {q, k, v, dout, dq, dk, dv, state_in, dstate_out, dstate_in};
    for (const void *p : ptrs)
        if (p && !aligned(p, 16)) return LA_ERR_INVALID_ARGUMENT;
    const size_t esz = grad_dtype == LA_FP32 ? 4 : 2;
    const size_t n_in = (size_t)T * H * la::D * 2, n_g = (size_t)T * H * la::D * esz;
    const size_t n_state = (size_t)nseq * H * la::D * la::D * 4;
    const void *ins[4] = {q, k, v, dout};
    void *gs[3] = {dq, dk, dv};
    for (int i = 0; i < 3; ++i) {
        void *g = gs[i];
        for (const void *p : ins)
            if (ranges_overlap(g, n_g, p, n_in)) return LA_ERR_INVALID_ARGUMENT;
        for (int j = i + 1; j < 3; ++j)
            if (ranges_overlap(g, n_g, gs[j], n_g)) return LA_ERR_INVALID_ARGUMENT;
        if (ranges_overlap(g, n_g, dstate_in, n_state) || ranges_overlap(g, n_g, state_in, n_state) ||
            ranges_overlap(g, n_g, dstate_out, n_state))
            return LA_ERR_INVALID_ARGUMENT;
    }
    if (ranges_overlap(dstate_in, n_state, state_in, n_state) || ranges_overlap(dstate_in, n_state, dstate_out, n_state))
        return LA_ERR_INVALID_ARGUMENT;
    const BwdLayout w = bwd_layout(cu != nullptr, nseq, fixed_len, T, H);
    if (!workspace || ws_bytes < w.total) return LA_ERR_WORKSPACE;
    if (!aligned(workspace, 256)) return LA_ERR_INVALID_ARGUMENT;
    for (const void *p : ptrs)
        if (p && ranges_overlap(workspace, w.total, p, p == q || p == k || p == v || p == dout ? n_in
                                                       : (p == dq || p == dk || p == dv ? n_g : n_state)))
            return LA_ERR_INVALID_ARGUMENT;
    if (cu && ranges_overlap(workspace, w.total, cu, (size_t)(nseq + 1) * sizeof(int))) return LA_ERR_INVALID_ARGUMENT;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    void *ws_pre = ws + w.prefill;
    const size_t pre_bytes = w.st0 - w.prefill;
    float *A = reinterpret_cast<float *>(ws + w.st0);

    // dQ: a forward sweep of (q, k, v) = (dO, V, K) from S_in^T
    //     dq_t = sum_{s <= t} (g_t . v_s) k_s + g_t S_in^T
    if (state_in && (st = launch_transpose(state_in, A, (long long)nseq * H, stream)) != LA_OK) return st;
    st = prefill_impl(dout, v, k, cu, fixed_len, nseq, T, max_seqlen, H, d, 0, state_in ? A : nullptr, dq,
                      grad_dtype, nullptr, ws_pre, pre_bytes, stream);
    if (st != LA_OK) return st;
    // dV and dK, sums over the later tokens:
    //     dv_s = sum_{t >= s} (q_t . k_s) g_t + k_s G,   dk_s = sum_{t >= s} (g_t . v_s) q_t + v_s G^T
    // one reversed sweep of the paired problems (q, k, v) = (K, Q, dO) and
    // (q2, v, k) = (V, dO, Q) from G, dK's state being dV's transposed; the
    // sweep's final state G + sum_t q_t^T g_t is dS_in.
    return prefill_impl(k, q, dout, cu, fixed_len, nseq, T, max_seqlen, H, d, 0, dstate_out, dv, grad_dtype,
                        dstate_in, ws_pre, pre_bytes, stream, nullptr, 0, nullptr, v, dk, true);
}

}  // namespace

extern "C" {

size_t la_prefill_workspace_size(int B, int N, int H, int d, int block) {
    (void)d;
    if (B <= 0 || N < 0 || H <= 0) return la::HDR_BYTES;
    const long long T = (long long)B * N;
    const int L = choose_seg_len(B, T, H, block);
    return ws_layout(gmax_fixed(B, N, L), H).total;
}

size_t la_prefill_varlen_workspace_size(int nseq, int total_tokens, int max_seqlen, int H, int d,
                                        int block) {
    (void)d;
    (void)max_seqlen;
    if (nseq <= 0 || total_tokens < 0 || H <= 0) return la::HDR_BYTES;
    const int L = choose_seg_len(nseq, total_tokens, H, block);
    return ws_layout(gmax_for(nseq, total_tokens, L), H).total;
}

la_status la_prefill(const void *q, const void *k, const void *v, int B, int N, int H, int d, int block,
                     const float *state_in, void *out, la_dtype out_dtype, float *state_out,
                     void *workspace, size_t ws_bytes, cudaStream_t stream) {
    if (B < 0 || N < 0) return LA_ERR_INVALID_ARGUMENT;
    const long long T = (long long)B * N;
    return prefill_impl(q, k, v, nullptr, N, B, T, N, H, d, block, state_in, out, out_dtype, state_out,
                        workspace, ws_bytes, stream);
}

la_status la_prefill_varlen(const void *q, const void *k, const void *v, const int *cu_seqlens,
                            int nseq, int total_tokens, int max_seqlen, int H, int d, int block,
                            const float *state_in, void *out, la_dtype out_dtype, float *state_out,
                            void *workspace, size_t ws_bytes, cudaStream_t stream) {
    if (!cu_seqlens || nseq < 0 || total_tokens < 0) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(cu_seqlens, 4)) return LA_ERR_INVALID_ARGUMENT;
    return prefill_impl(q, k, v, cu_seqlens, 0, nseq, total_tokens, max_seqlen, H, d, block, state_in,
                        out, out_dtype, state_out, workspace, ws_bytes, stream);
}

la_status la_prefill_varlen_slots(const void *q, const void *k, const void *v, const int *cu_seqlens,
                                  const int *slots, int nseq, int total_tokens, int max_seqlen, int H, int d,
                                  int block, float *state_pool, int n_slots, void *out, la_dtype out_dtype,
                                  void *workspace, size_t ws_bytes, cudaStream_t stream) {
    if (!cu_seqlens || nseq < 0 || total_tokens < 0) return LA_ERR_INVALID_ARGUMENT;
    if (nseq > 0 && (!slots || !state_pool)) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(cu_seqlens, 4)) return LA_ERR_INVALID_ARGUMENT;
    if (nseq == 0) return total_tokens == 0 ? LA_OK : LA_ERR_INVALID_ARGUMENT;
    return prefill_impl(q, k, v, cu_seqlens, 0, nseq, total_tokens, max_seqlen, H, d, block, state_pool,
                        out, out_dtype, state_pool, workspace, ws_bytes, stream, slots, n_slots);
}

la_status la_decode_step(const void *q, const void *k, const void *v, float *state, void *out,
                         la_dtype out_dtype, int B, int H, int d, cudaStream_t stream) {
    return decode_impl(q, k, v, state, nullptr, 0, out, out_dtype, B, H, d, stream);
}

la_status la_decode_step_slots(const void *q, const void *k, const void *v, float *state_pool, int n_slots,
                               const int *slots, void *out, la_dtype out_dtype, int B, int H, int d,
                               cudaStream_t stream) {
    if (B > 0 && !slots) return LA_ERR_INVALID_ARGUMENT;
    return decode_impl(q, k, v, state_pool, slots, n_slots, out, out_dtype, B, H, d, stream);
}

la_status la_prefill_decay(const void *q, const void *k, const void *v, int B, int N, int H, int d, int block,
                           const float *decay, const float *state_in, void *out, la_dtype out_dtype,
                           float *state_out, void *workspace, size_t ws_bytes, cudaStream_t stream) {
    if (B < 0 || N < 0 || !decay) return LA_ERR_INVALID_ARGUMENT;
    const long long T = (long long)B * N;
    return prefill_impl(q, k, v, nullptr, N, B, T, N, H, d, block, state_in, out, out_dtype, state_out,
                        workspace, ws_bytes, stream, nullptr, 0, decay);
}

la_status la_prefill_varlen_decay(const void *q, const void *k, const void *v, const int *cu_seqlens, int nseq,
                                  int total_tokens, int max_seqlen, int H, int d, int block, const float *decay,
                                  const float *state_in, void *out, la_dtype out_dtype, float *state_out,
                                  void *workspace, size_t ws_bytes, cudaStream_t stream) {
    if (!cu_seqlens || nseq < 0 || total_tokens < 0 || !decay) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(cu_seqlens, 4)) return LA_ERR_INVALID_ARGUMENT;
    return prefill_impl(q, k, v, cu_seqlens, 0, nseq, total_tokens, max_seqlen, H, d, block, state_in,
                        out, out_dtype, state_out, workspace, ws_bytes, stream, nullptr, 0, decay);
}

la_status la_decode_step_decay(const void *q, const void *k, const void *v, const float *decay, float *state,
                               void *out, la_dtype out_dtype, int B, int H, int d, cudaStream_t stream) {
    if (!decay) return LA_ERR_INVALID_ARGUMENT;
    return decode_impl(q, k, v, state, nullptr, 0, out, out_dtype, B, H, d, stream, decay);
}

la_status la_mixed_step(const void *q, const void *k, const void *v, const int *cu_seqlens,
                        const int *prefill_slots, int n_prefill, int prefill_tokens, int max_seqlen,
                        const int *decode_slots, int n_decode, int H, int d, float *state_pool, int n_slots,
                        void *out, la_dtype out_dtype, void *workspace, size_t ws_bytes,
                        cudaStream_t prefill_stream, cudaStream_t decode_stream) {
    la_status st = check_common(H, d, 0, out_dtype);
    if (st != LA_OK) return st;
    if (n_prefill < 0 || n_decode < 0 || prefill_tokens < 0 || n_slots <= 0 || !state_pool)
        return LA_ERR_INVALID_ARGUMENT;
    if ((long long)prefill_tokens + n_decode > 0x7fffffffLL) return LA_ERR_INVALID_ARGUMENT;
    if (n_prefill == 0 && prefill_tokens != 0) return LA_ERR_INVALID_ARGUMENT;
    if (n_decode > 0 && (!decode_slots || !q || !k || !v || !out)) return LA_ERR_INVALID_ARGUMENT;
    // rows [0, prefill_tokens): packed prefill chunks; rows [prefill_tokens, + n_decode): one
    // decode token per decode slot
    const size_t row = (size_t)H * la::D;
    const size_t esz = out_dtype == LA_FP32 ? 4 : 2;
    if (n_decode > 0) {  // the decode part's checks, before anything is queued
        const void *ptrs[5] = {q, k, v, out, state_pool};
        for (const void *p : ptrs)
            if (!aligned(p, 16)) return LA_ERR_INVALID_ARGUMENT;
        if (!aligned(decode_slots, 4)) return LA_ERR_INVALID_ARGUMENT;
        const size_t n_out = ((size_t)prefill_tokens + n_decode) * row * esz;
        if (ranges_overlap(out, n_out, state_pool, (size_t)n_slots * H * la::D * la::D * 4))
            return LA_ERR_INVALID_ARGUMENT;
    }
    if (n_prefill > 0) {
        st = la_prefill_varlen_slots(q, k, v, cu_seqlens, prefill_slots, n_prefill, prefill_tokens, max_seqlen, H,
                                     d, 0, state_pool, n_slots, out, out_dtype, workspace, ws_bytes, prefill_stream);
        if (st != LA_OK) return st;
    }
    if (n_decode > 0) {
        const size_t off = (size_t)prefill_tokens * row;
        st = decode_impl(static_cast<const uint16_t *>(q) + off, static_cast<const uint16_t *>(k) + off,
                         static_cast<const uint16_t *>(v) + off, state_pool, decode_slots, n_slots,
                         static_cast<uint8_t *>(out) + off * esz, out_dtype, n_decode, H, d, decode_stream);
        if (st != LA_OK) return st;
        if (decode_stream != prefill_stream) {
            // join: work queued on the prefill stream after this call sees both results
            static thread_local cudaEvent_t ev = nullptr;
            if (!ev && cudaEventCreateWithFlags(&ev, cudaEventDisableTiming) != cudaSuccess) return LA_ERR_CUDA;
            if (cudaEventRecord(ev, decode_stream) != cudaSuccess) return LA_ERR_CUDA;
            if (cudaStreamWaitEvent(prefill_stream, ev, 0) != cudaSuccess) return LA_ERR_CUDA;
        }
    }
    return LA_OK;
}


// ---------------------------------------------------------------------------
// Prefill of inputs in pinned host memory: chunks of tokens copied in, scanned
// from the carried state and copied out, pipelined over three streams.
// ---------------------------------------------------------------------------
namespace {

struct HostLayout {
    size_t slot_in, slot_out, slot, state, ws, total;
};

HostLayout host_layout(int B, int C, int H, size_t esz) {
    HostLayout l;
    l.slot_in = round_up((size_t)B * C * H * la::D * 2, 256);
    l.slot_out = round_up((size_t)B * C * H * la::D * esz, 256);
    l.slot = 3 * l.slot_in + l.slot_out;
    l.state = round_up((size_t)B * H * la::D * la::D * 4, 256);
    // the workspace of the longest chunk, or of a shorter last chunk (which may
    // be cut into more, shorter segments)
    size_t ws = 0;
    for (int n = 1; n <= C; ++n) {
        const size_t w = la_prefill_workspace_size(B, n, H, la::D, 0);
        ws = w > ws ? w : ws;
    }
    l.ws = round_up(ws, 256);
    l.total = 2 * l.slot + l.state + l.ws;
    return l;
}

bool pinned_host(const void *p) {
    cudaPointerAttributes a;
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return a.type == cudaMemoryTypeHost;
}

}  // namespace

size_t la_prefill_from_host_buffer_size(int B, int chunk_tokens, int H, int d, la_dtype out_dtype) {
    if (B <= 0 || chunk_tokens <= 0 || H <= 0 || d != la::D) return 0;
    return host_layout(B, chunk_tokens, H, out_dtype == LA_FP32 ? 4 : 2).total;
}

la_status la_prefill_from_host(const void *q, const void *k, const void *v, int B, int N, int H, int d,
                               int chunk_tokens, const float *state_in, void *out, la_dtype out_dtype,
                               float *state_out, void *buffers, size_t buffer_bytes, cudaStream_t copy_in,
                               cudaStream_t compute, cudaStream_t copy_out) {
    la_status st = check_common(H, d, 0, out_dtype);
    if (st != LA_OK) return st;
    if (B < 0 || N < 0 || chunk_tokens <= 0) return LA_ERR_INVALID_ARGUMENT;
    if (B == 0) return LA_OK;
    if ((long long)B * N > 0x7fffffffLL) return LA_ERR_INVALID_ARGUMENT;
    const int C = chunk_tokens < N ? chunk_tokens : (N > 0 ? N : 1);
    const size_t esz = out_dtype == LA_FP32 ? 4 : 2;
    const HostLayout l = host_layout(B, C, H, esz);
    if (!buffers || buffer_bytes < l.total) return LA_ERR_WORKSPACE;
    if (!aligned(buffers, 256)) return LA_ERR_INVALID_ARGUMENT;
    if (N > 0) {
        if (!q || !k || !v || !out) return LA_ERR_INVALID_ARGUMENT;
        const void *host[4] = {q, k, v, out};
        for (const void *p : host)
            if (!pinned_host(p)) return LA_ERR_INVALID_ARGUMENT;  // pinned host memory only
    }
    if ((state_in && !aligned(state_in, 16)) || (state_out && !aligned(state_out, 16))) return LA_ERR_INVALID_ARGUMENT;
    const size_t n_state = (size_t)B * H * la::D * la::D * 4;
    if (ranges_overlap(buffers, l.total, state_in, n_state) || ranges_overlap(buffers, l.total, state_out, n_state))
        return LA_ERR_INVALID_ARGUMENT;

    // events: per host thread and device, created once, reused by every call
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LA_ERR_CUDA;
    static thread_local cudaEvent_t events[kMaxDevices][7] = {};
    cudaEvent_t *ev = events[dev];
    if (!ev[6])  // the last one is set only once all seven exist
        for (int i = 0; i < 7; ++i)
            if (!ev[i] && cudaEventCreateWithFlags(&ev[i], cudaEventDisableTiming) != cudaSuccess) return LA_ERR_CUDA;
    cudaEvent_t *ev_in = ev, *ev_cmp = ev + 2, *ev_out = ev + 4, ev_start = ev[6];

    uint8_t *base = static_cast<uint8_t *>(buffers);
    float *state = reinterpret_cast<float *>(base + 2 * l.slot);
    void *ws = base + 2 * l.slot + l.state;
    // the copy streams start after the compute stream's earlier work
    if (cudaEventRecord(ev_start, compute) != cudaSuccess) return LA_ERR_CUDA;
    if (cudaStreamWaitEvent(copy_in, ev_start, 0) != cudaSuccess) return LA_ERR_CUDA;
    if (cudaStreamWaitEvent(copy_out, ev_start, 0) != cudaSuccess) return LA_ERR_CUDA;
    // the running state starts as state_in (or zero)
    if ((st = la_state_prefix(nullptr, 0, state_in, state, B * H, d, compute)) != LA_OK) return st;

    const size_t row_in = (size_t)H * la::D * 2, row_out = (size_t)H * la::D * esz;
    const int nchunks = N > 0 ? (N + C - 1) / C : 0;
    for (int c = 0; c < nchunks; ++c) {
        const int j = c & 1;
        const int t0 = c * C, n = (t0 + C < N ? C : N - t0);
        uint8_t *slot = base + j * l.slot;
        uint8_t *dq = slot, *dk = slot + l.slot_in, *dv = slot + 2 * l.slot_in, *dout = slot + 3 * l.slot_in;
        // copy in (slot j is free once the chunk two before it was scanned and copied out)
        if (c >= 2 && (cudaStreamWaitEvent(copy_in, ev_cmp[j], 0) != cudaSuccess ||
                       cudaStreamWaitEvent(copy_in, ev_out[j], 0) != cudaSuccess))
            return LA_ERR_CUDA;
        for (int b = 0; b < B; ++b) {
            const size_t src = ((size_t)b * N + t0) * row_in, dst = (size_t)b * n * row_in, bytes = (size_t)n * row_in;
            if (cudaMemcpyAsync(dq + dst, static_cast<const uint8_t *>(q) + src, bytes, cudaMemcpyHostToDevice, copy_in) != cudaSuccess ||
                cudaMemcpyAsync(dk + dst, static_cast<const uint8_t *>(k) + src, bytes, cudaMemcpyHostToDevice, copy_in) != cudaSuccess ||
                cudaMemcpyAsync(dv + dst, static_cast<const uint8_t *>(v) + src, bytes, cudaMemcpyHostToDevice, copy_in) != cudaSuccess)
                return LA_ERR_CUDA;
        }
        if (cudaEventRecord(ev_in[j], copy_in) != cudaSuccess) return LA_ERR_CUDA;
        // scan the chunk from the carried state, in place (the state-carry
        // identity: a prefill of chunk c from the state after chunk c-1 is the
        // prefill of the longer sequence)
        if (cudaStreamWaitEvent(compute, ev_in[j], 0) != cudaSuccess) return LA_ERR_CUDA;
        if (c >= 2 && cudaStreamWaitEvent(compute, ev_out[j], 0) != cudaSuccess) return LA_ERR_CUDA;
        st = la_prefill(dq, dk, dv, B, n, H, d, 0, state, dout, out_dtype, state, ws, l.ws, compute);
        if (st != LA_OK) return st;
        if (cudaEventRecord(ev_cmp[j], compute) != cudaSuccess) return LA_ERR_CUDA;
        // copy out
        if (cudaStreamWaitEvent(copy_out, ev_cmp[j], 0) != cudaSuccess) return LA_ERR_CUDA;
        for (int b = 0; b < B; ++b) {
            const size_t dst = ((size_t)b * N + t0) * row_out, src = (size_t)b * n * row_out, bytes = (size_t)n * row_out;
            if (cudaMemcpyAsync(static_cast<uint8_t *>(out) + dst, dout + src, bytes, cudaMemcpyDeviceToHost, copy_out) != cudaSuccess)
                return LA_ERR_CUDA;
        }
        if (cudaEventRecord(ev_out[j], copy_out) != cudaSuccess) return LA_ERR_CUDA;
    }
    if (state_out && cudaMemcpyAsync(state_out, state, n_state, cudaMemcpyDefault, compute) != cudaSuccess)
        return LA_ERR_CUDA;
    // work queued on the compute stream after this call sees every result
    if (nchunks > 0 && cudaStreamWaitEvent(compute, ev_out[(nchunks - 1) & 1], 0) != cudaSuccess) return LA_ERR_CUDA;
    return LA_OK;
}

la_status la_get_device_status(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return LA_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_la_status, sizeof(int)) != cudaSuccess) return LA_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpyToSymbol(g_la_status, &zero, sizeof(int)) != cudaSuccess) return LA_ERR_CUDA;
    }
    return static_cast<la_status>(v);
}

const char *la_status_string(la_status s) {
    switch (s) {
        case LA_OK: return "ok";
        case LA_ERR_INVALID_ARGUMENT: return "invalid argument";
        case LA_ERR_UNSUPPORTED: return "unsupported (d = 128 only; row blocks 0/64/128/256, decay at 128 only)";
        case LA_ERR_CUDA: return "CUDA error";
        case LA_ERR_TIMEOUT: return "a bounded device-side wait ran out";
        case LA_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

la_status la_set_wait_limit_ns(unsigned long long ns) {
    g_wait_limit_ns = ns ? ns : kDefaultWaitNs;
    return LA_OK;
}

la_status la_set_segment_len(int tokens) {
    if (tokens < 0 || (tokens > 0 && tokens % la::BLK)) return LA_ERR_INVALID_ARGUMENT;
    g_seg_len_override = tokens;
    return LA_OK;
}

la_status la_debug_inject(int mode) {
    if (mode != LA_INJECT_NONE && mode != LA_INJECT_SKIP_PUBLISH) return LA_ERR_INVALID_ARGUMENT;
    g_inject = mode;
    return LA_OK;
}

int la_last_segment_len(void) { return g_last_seg_len.load(); }

unsigned long long la_kernel_launches(void) { return g_launches.load(); }

size_t la_kv_aggregate_workspace_size(int B, int N, int H, int d) {
    (void)d;
    if (B <= 0 || N <= 0 || H <= 0) return 0;
    return agg_ws_bytes(agg_plan((long long)B * H, N));
}

la_status la_kv_aggregate(const void *k, const void *v, int B, int N, int H, int d, float *agg, void *workspace,
                          size_t ws_bytes, cudaStream_t stream) {
    la_status st = check_common(H, d, 0, LA_FP32);
    if (st != LA_OK) return st;
    if (B < 0 || N < 0) return LA_ERR_INVALID_ARGUMENT;
    if (B == 0) return LA_OK;
    const long long T = (long long)B * N;
    if (T > 0x7fffffffLL || (long long)B * H > 0x7fffffffLL) return LA_ERR_INVALID_ARGUMENT;
    if (!agg || !aligned(agg, 16)) return LA_ERR_INVALID_ARGUMENT;
    if (T > 0 && (!k || !v || !aligned(k, 16) || !aligned(v, 16))) return LA_ERR_INVALID_ARGUMENT;
    const size_t n_in = (size_t)T * H * la::D * 2, n_agg = (size_t)B * H * la::D * la::D * 4;
    if (ranges_overlap(agg, n_agg, k, n_in) || ranges_overlap(agg, n_agg, v, n_in)) return LA_ERR_INVALID_ARGUMENT;
    const AggPlan a = agg_plan((long long)B * H, N);
    const size_t need = agg_ws_bytes(a);
    if (need > 0) {
        if (!workspace || ws_bytes < need) return LA_ERR_WORKSPACE;
        if (!aligned(workspace, 16)) return LA_ERR_INVALID_ARGUMENT;
        if (ranges_overlap(workspace, need, agg, n_agg)) return LA_ERR_INVALID_ARGUMENT;
    }
    int *status = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void **>(&status), g_la_status) != cudaSuccess) return LA_ERR_CUDA;
    if (a.ctas > 0) {
        CUtensorMap mk, mv;
        if (!encode_qkv_map(&mk, k, (int)T, H) || !encode_qkv_map(&mv, v, (int)T, H)) return LA_ERR_CUDA;
        la::AggParams p;
        p.out = agg;
        p.partial = static_cast<float *>(workspace);
        p.N = N;
        p.H = H;
        p.nblk = a.nblk;
        p.total = a.total;
        p.per_cta = a.per_cta;
        p.wait_limit_ns = g_wait_limit_ns.load();
        p.status = status;
        st = ensure_smem_attr(g_attr_agg, la::la_kv_aggregate_kernel, la::AGG_SMEM);
        if (st != LA_OK) return st;
        la::la_kv_aggregate_kernel<<<a.ctas, la::AGG_THREADS, la::AGG_SMEM, stream>>>(mk, mv, p);
        if (cudaGetLastError() != cudaSuccess) return LA_ERR_CUDA;
        ++g_launches;
    }
    // sums of the pairs that range boundaries cut (zeros when N == 0)
    la::la_agg_reduce_kernel<<<dim3((unsigned)((long long)B * H), la::AGG_RED_SLICES), la::AGG_RED_THREADS, 0,
                               stream>>>(agg, static_cast<const float *>(workspace), a.nblk, a.per_cta);
    if (cudaGetLastError() != cudaSuccess) return LA_ERR_CUDA;
    ++g_launches;
    return LA_OK;
}

size_t la_prefill_backward_workspace_size(int B, int N, int H, int d) {
    (void)d;
    if (B <= 0 || N < 0 || H <= 0) return la::HDR_BYTES;
    return bwd_layout(false, B, N, (long long)B * N, H).total;
}

la_status la_prefill_backward(const void *q, const void *k, const void *v, const void *dout, int B, int N, int H,
                              int d, const float *state_in, const float *dstate_out, void *dq, void *dk, void *dv,
                              la_dtype grad_dtype, float *dstate_in, void *workspace, size_t ws_bytes,
                              cudaStream_t stream) {
    if (B < 0 || N < 0) return LA_ERR_INVALID_ARGUMENT;
    if (B == 0) return check_common(H, d, 0, grad_dtype);
    return backward_impl(q, k, v, dout, nullptr, N, B, (long long)B * N, N, H, d, state_in, dstate_out, dq, dk,
                         dv, grad_dtype, dstate_in, workspace, ws_bytes, stream);
}

size_t la_prefill_backward_varlen_workspace_size(int nseq, int total_tokens, int max_seqlen, int H, int d) {
    (void)d;
    (void)max_seqlen;
    if (nseq <= 0 || total_tokens < 0 || H <= 0) return la::HDR_BYTES;
    return bwd_layout(true, nseq, 0, total_tokens, H).total;
}

la_status la_prefill_backward_varlen(const void *q, const void *k, const void *v, const void *dout,
                                     const int *cu_seqlens, int nseq, int total_tokens, int max_seqlen, int H,
                                     int d, const float *state_in, const float *dstate_out, void *dq, void *dk,
                                     void *dv, la_dtype grad_dtype, float *dstate_in, void *workspace,
                                     size_t ws_bytes, cudaStream_t stream) {
    if (!cu_seqlens || nseq < 0 || total_tokens < 0) return LA_ERR_INVALID_ARGUMENT;
    if (!aligned(cu_seqlens, 4)) return LA_ERR_INVALID_ARGUMENT;
    return backward_impl(q, k, v, dout, cu_seqlens, 0, nseq, total_tokens, max_seqlen, H, d, state_in, dstate_out,
                         dq, dk, dv, grad_dtype, dstate_in, workspace, ws_bytes, stream);
}

la_status la_state_prefix(const float *parts, int count, const float *state_in, float *out, int nstates, int d,
                          cudaStream_t stream) {
    if (d <= 0 || nstates < 0 || count < 0) return LA_ERR_INVALID_ARGUMENT;
    if (d != la::D) return LA_ERR_UNSUPPORTED;
    if (nstates == 0) return LA_OK;
    if (!out || !aligned(out, 16)) return LA_ERR_INVALID_ARGUMENT;
    if (count > 0 && (!parts || !aligned(parts, 16))) return LA_ERR_INVALID_ARGUMENT;
    if (state_in && !aligned(state_in, 16)) return LA_ERR_INVALID_ARGUMENT;
    const size_t n = (size_t)nstates * la::D * la::D * 4;
    if (ranges_overlap(out, n, parts, (size_t)count * n)) return LA_ERR_INVALID_ARGUMENT;
    if (state_in && state_in != out && ranges_overlap(out, n, state_in, n)) return LA_ERR_INVALID_ARGUMENT;
    const long long n4 = (long long)nstates * (la::D * la::D / 4);
    long long blocks = (n4 + la::PREFIX_THREADS - 1) / la::PREFIX_THREADS;
    const long long cap = (long long)device_sm_count() * 8;
    if (blocks > cap) blocks = cap;
    la::la_state_prefix_kernel<<<(unsigned)blocks, la::PREFIX_THREADS, 0, stream>>>(
        reinterpret_cast<const float4 *>(parts), count, reinterpret_cast<const float4 *>(state_in),
        reinterpret_cast<float4 *>(out), n4);
    if (cudaGetLastError() != cudaSuccess) return LA_ERR_CUDA;
    ++g_launches;
    return LA_OK;
}

}  // extern "C"

// ===========================================================================
// la_prefill_noalloc -- la_prefill for callers that cannot allocate.
//
// Some callers have no way to hand us a workspace: a plugin loaded into a host
// framework that owns the device allocator and offers no allocation hook, or a
// serving process that reserves all device memory up front (for its caches)
// and forbids further cudaMalloc calls on its request path, where cudaMalloc
// would also be a slow, device-synchronising call.  For them this entry point
// takes no workspace: its scratch is the fixed-size device array below,
// reserved once in every process that loads the library, on every GPU it
// touches, until the process exits.
//
// Its scratch needs grow with the number of (segment, head) work items, so
// this variant lengthens the segments (which changes only speed and
// rounding) until the scratch fits; if even one segment per sequence does not
// fit, the call is rejected with LA_ERR_WORKSPACE before anything is launched.
// The scheduler kernel re-initialises every word of scratch that must start
// at zero (ticket counter, hand-off flags) at the start of each call, so the
// contents left by the previous call do not matter.  All calls share the one
// array: calls that can overlap on the GPU (different streams, or different
// host threads) race on it and must be serialised by the caller.
// ===========================================================================
#define LA_NOALLOC_SCRATCH_BYTES (32u << 20)  // 32 MiB per GPU
static __device__ __align__(256) unsigned char g_la_noalloc_scratch[LA_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_addr[kNoAllocMaxDevices] = {};

// Device address of the scratch array on the current device.  The host-side
// symbol is only a stand-in; the real address comes from cudaGetSymbolAddress,
// looked up once per device on the first call made with that device current.
la_status noalloc_scratch_address(void **addr) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return LA_ERR_CUDA;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return LA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_la_noalloc_scratch);
        if (e != cudaSuccess || p == nullptr) return LA_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    *addr = g_noalloc_addr[dev];
    return LA_OK;
}

}  // namespace

extern "C" la_status la_prefill_noalloc(const void *q, const void *k, const void *v, int B, int N, int H,
                                        int d, int block, const float *state_in, void *out,
                                        la_dtype out_dtype, float *state_out, cudaStream_t stream) {
    la_status st = check_common(H, d, block, out_dtype);
    if (st != LA_OK) return st;
    if (B < 0 || N < 0) return LA_ERR_INVALID_ARGUMENT;
    const long long T = (long long)B * N;
    if (T > 0x7fffffffLL) return LA_ERR_INVALID_ARGUMENT;
    if (B == 0) return LA_OK;
    if (T > 0 && (!q || !k || !v || !out)) return LA_ERR_INVALID_ARGUMENT;
    const void *ptrs[6] = {q, k, v, out, state_in, state_out};
    for (const void *p : ptrs)
        if (p && !aligned(p, 16)) return LA_ERR_INVALID_ARGUMENT;
    const size_t esz = out_dtype == LA_FP32 ? 4 : 2;
    const size_t n_in = (size_t)T * H * la::D * 2, n_out = (size_t)T * H * la::D * esz;
    const size_t n_state = (size_t)B * H * la::D * la::D * 4;
    if (state_out && state_out != state_in && ranges_overlap(state_out, n_state, state_in, n_state))
        return LA_ERR_INVALID_ARGUMENT;
    const void *ins[3] = {q, k, v};
    for (const void *p : ins) {
        if (ranges_overlap(out, n_out, p, n_in)) return LA_ERR_INVALID_ARGUMENT;
        if (ranges_overlap(state_out, n_state, p, n_in)) return LA_ERR_INVALID_ARGUMENT;
    }
    if (ranges_overlap(out, n_out, state_out, n_state) || ranges_overlap(out, n_out, state_in, n_state))
        return LA_ERR_INVALID_ARGUMENT;

    // longest useful segment: one per sequence
    const int max_len = (int)(((long long)(N > 0 ? N : 1) + la::BLK - 1) / la::BLK * la::BLK);
    int L = choose_seg_len(B, T, H, block);
    while (ws_layout(gmax_fixed(B, N, L), H).total > LA_NOALLOC_SCRATCH_BYTES && L < max_len)
        L = (2 * L < max_len) ? 2 * L : max_len;
    const long long gmax = gmax_fixed(B, N, L);
    const WsLayout w = ws_layout(gmax, H);
    if (w.total > LA_NOALLOC_SCRATCH_BYTES) return LA_ERR_WORKSPACE;  // beyond the built-in scratch

    void *scratch = nullptr;
    st = noalloc_scratch_address(&scratch);
    if (st != LA_OK) return st;
    int *status = nullptr;
    if (cudaGetSymbolAddress(reinterpret_cast<void **>(&status), g_la_status) != cudaSuccess)
        return LA_ERR_CUDA;
    uint8_t *ws = static_cast<uint8_t *>(scratch);
    g_last_seg_len = L;

    la::ScheduleParams sp;
    sp.cu = nullptr;
    sp.fixed_len = N;
    sp.nseq = B;
    sp.T = (int)T;
    sp.max_seqlen = N;
    sp.H = H;
    sp.seg_len = L;
    sp.Gmax = (int)gmax;
    sp.hdr = reinterpret_cast<int *>(ws + w.hdr);
    sp.segs = reinterpret_cast<int4 *>(ws + w.segs);
    sp.flags = reinterpret_cast<int *>(ws + w.flags);
    sp.state_in = state_in;
    sp.state_out = state_out;
    sp.slots = nullptr;
    sp.n_slots = 0;
    sp.decay = nullptr;
    sp.reverse = 0;
    sp.status = status;
    la::la_schedule_kernel<<<1, la::SCHED_THREADS, 0, stream>>>(sp);
    if (cudaGetLastError() != cudaSuccess) return LA_ERR_CUDA;
    ++g_launches;
    if (T == 0) return LA_OK;

    CUtensorMap mq, mk, mv;
    if (!encode_qkv_map(&mq, q, (int)T, H) || !encode_qkv_map(&mk, k, (int)T, H) ||
        !encode_qkv_map(&mv, v, (int)T, H))
        return LA_ERR_CUDA;
    la::PrefillParams pp;
    pp.state_in = state_in;
    pp.state_out = state_out;
    pp.slots = nullptr;
    pp.out = out;
    pp.out2 = nullptr;
    pp.out_fp32 = out_dtype == LA_FP32;
    pp.out_al32 = aligned(out, 32);
    pp.H = H;
    pp.hdr = sp.hdr;
    pp.segs = sp.segs;
    pp.flags = sp.flags;
    pp.incl = reinterpret_cast<float *>(ws + w.incl);
    pp.wait_limit_ns = g_wait_limit_ns.load();
    pp.inject = g_inject.load();
    pp.decay = nullptr;
    pp.seg_len = L;
    pp.status = status;
    const long long items = gmax * (long long)H;
    const int grid = (int)(items < device_sm_count() ? items : device_sm_count());
    st = launch_prefill<false>(block, grid, mq, mk, mv, pp, stream);
    if (st != LA_OK) return st;
    ++g_launches;
    return LA_OK;
}
