/*
 * lightning_oracle.c -- plain, slow, fp64 CPU oracle for Lightning Attention
 * (blocked causal linear attention).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may include, link,
 * load or call this file: only the test suite, the smoke check of the entry
 * module and the CPU-baseline leg of the benchmark use it.  It shares no code,
 * header, table or helper with the CUDA library; both sides only receive the
 * same seeded input bits.
 *
 * Every input value is a bf16 bit pattern (uint16) and is widened exactly to
 * double; all arithmetic is fp64 with plain loops in the order the definitions
 * state.  OpenMP splits the independent (sequence, head) pairs across threads;
 * nothing inside one pair is blocked, fused or reordered beyond the definition.
 *
 * Sources (web pages on the MiniMax-01 report):
 *   [P2] "MiniMax-01技术报告解读（一）模型架构" (blog.csdn.net), §2.2 线性注意力:
 *        the right-product kernel trick with a recursively updated KV product;
 *        intra-block left product, inter-block right product; Q/K/V split into
 *        row blocks.
 *   [P5] "MiniMax-01技术报告解读" (qingkelab.github.io), §2.2 (same text as P2),
 *        §3.2 item 3 (LASP+: local prefix KV_t, AllGather, global prefix KV_G),
 *        §3.2 item 1 (data packing: samples joined end to end),
 *        §3.3 items 1-2 (decode: length-1 tokens, KV update fused with the
 *        prefix-KV cache).
 *   Gradients: [P5] §3.2 item 3 trains the model with LASP+ but the pages
 *   give no backward formulas; lao_backward writes out the derivatives of
 *   the forward definition below, term by term.
 *   The pages print no formula; the formula used is the plainest reading of
 *   that prose: O = (Q K^T ⊙ M) V with the inclusive causal mask
 *   M[t][s] = 1 iff s <= t, no scale, feature map, normalisation or decay
 *   inside the operation, and state S[i][j] = sum_s k_s[i] v_s[j]
 *   (d_k rows x d_v columns).
 *
 * Layouts (all row-major, token-major packing as in [P5] §3.2 item 1):
 *   q, k, v     : uint16 bf16 bits [T][H][d]; sequence i owns tokens
 *                 [cu_seqlens[i], cu_seqlens[i+1]).
 *   heads       : the nh head indices to compute (NULL = all H, in order).
 *   state_in    : double [nseq][nh][d][d] or NULL (= zero state).
 *   out         : double [T][nh][d].
 *   state_out   : double [nseq][nh][d][d] or NULL.
 * Every function returns 0 on success and -1 on an invalid argument.
 *
 * Parity status: every function here is pinned by the CPU test suite against
 * closed forms, exact-integer library routines and brute force (see the
 * test files); none is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 is the upper half of an IEEE binary32; the widening is exact. */
static double widen_bf16(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static int check_common(const int32_t *cu, int nseq, int H, int d,
                        const int32_t *heads, int nh)
{
    if (!cu || nseq < 0 || H <= 0 || d <= 0 || nh <= 0) return -1;
    if (cu[0] != 0) return -1;
    for (int i = 0; i < nseq; ++i)
        if (cu[i + 1] < cu[i]) return -1;
    if (heads)
        for (int j = 0; j < nh; ++j)
            if (heads[j] < 0 || heads[j] >= H) return -1;
    if (!heads && nh != H) return -1;
    return 0;
}

/* The host's default thread count, captured before any call changes it, so
 * that a call with nthreads = 0 runs on the default again after a call that
 * asked for a specific count (omp_set_num_threads persists in the calling
 * thread). */
static int default_threads(void)
{
#ifdef _OPENMP
    static int def = 0;
    if (def <= 0) def = omp_get_max_threads();
    return def;
#else
    return 1;
#endif
}

static void set_threads(int nthreads)
{
#ifdef _OPENMP
    omp_set_num_threads(nthreads > 0 ? nthreads : default_threads());
#else
    (void)nthreads;
#endif
}

int lao_max_threads(void)
{
    return default_threads();
}

/* Pointer to the d-vector of token t, head h in a [T][H][d] array. */
#define ROW(x, t, h) ((x) + ((size_t)(t) * (size_t)H + (size_t)(h)) * (size_t)d)

/*
 * Recurrent form ([P2]/[P5] §2.2: "the KV product is updated recursively"):
 *   S_0 = S_in,  S_t = S_{t-1} + k_t^T v_t,  o_t = q_t S_t.
 * The state after token t includes token t, so o_t sees s <= t (inclusive).
 */
int lao_recurrent(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                  const int32_t *cu_seqlens, int nseq, int H, int d,
                  const int32_t *heads, int nh, const double *state_in,
                  double *out, double *state_out, int nthreads)
{
    if (!q || !k || !v || !out) return -1;
    if (check_common(cu_seqlens, nseq, H, d, heads, nh)) return -1;
    set_threads(nthreads);
    const long npairs = (long)nseq * nh;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long p = 0; p < npairs; ++p) {
        const int i = (int)(p / nh), j = (int)(p % nh);
        const int h = heads ? heads[j] : j;
        double *S = (double *)calloc((size_t)d * d, sizeof(double));
        double *kt = (double *)malloc((size_t)d * sizeof(double));
        double *vt = (double *)malloc((size_t)d * sizeof(double));
        double *qt = (double *)malloc((size_t)d * sizeof(double));
        if (!S || !kt || !vt || !qt) {
            bad = 1;
            free(S); free(kt); free(vt); free(qt);
            continue;
        }
        if (state_in)
            memcpy(S, state_in + (size_t)p * d * d, (size_t)d * d * sizeof(double));
        for (int t = cu_seqlens[i]; t < cu_seqlens[i + 1]; ++t) {
            for (int a = 0; a < d; ++a) {
                qt[a] = widen_bf16(ROW(q, t, h)[a]);
                kt[a] = widen_bf16(ROW(k, t, h)[a]);
                vt[a] = widen_bf16(ROW(v, t, h)[a]);
            }
            /* S_t = S_{t-1} + k_t^T v_t */
            for (int a = 0; a < d; ++a)
                for (int b = 0; b < d; ++b)
                    S[(size_t)a * d + b] += kt[a] * vt[b];
            /* o_t = q_t S_t */
            double *o = out + ((size_t)t * nh + j) * d;
            for (int b = 0; b < d; ++b) o[b] = 0.0;
            for (int a = 0; a < d; ++a)
                for (int b = 0; b < d; ++b)
                    o[b] += qt[a] * S[(size_t)a * d + b];
        }
        if (state_out)
            memcpy(state_out + (size_t)p * d * d, S, (size_t)d * d * sizeof(double));
        free(S); free(kt); free(vt); free(qt);
    }
    return bad ? -1 : 0;
}

/*
 * Quadratic (masked, left-product) form, spec definition
 * O = (Q K^T ⊙ M) V with M[t][s] = 1 iff s <= t; a carried-in state adds
 * q_t S_in to every row.
 *   o_t = sum_{s <= t} (q_t . k_s) v_s + q_t S_in
 */
int lao_quadratic(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                  const int32_t *cu_seqlens, int nseq, int H, int d,
                  const int32_t *heads, int nh, const double *state_in,
                  double *out, double *state_out, int nthreads)
{
    if (!q || !k || !v || !out) return -1;
    if (check_common(cu_seqlens, nseq, H, d, heads, nh)) return -1;
    set_threads(nthreads);
    const long npairs = (long)nseq * nh;
#pragma omp parallel for schedule(dynamic, 1)
    for (long p = 0; p < npairs; ++p) {
        const int i = (int)(p / nh), j = (int)(p % nh);
        const int h = heads ? heads[j] : j;
        const int t0 = cu_seqlens[i], t1 = cu_seqlens[i + 1];
        const double *Sin = state_in ? state_in + (size_t)p * d * d : NULL;
        for (int t = t0; t < t1; ++t) {
            double *o = out + ((size_t)t * nh + j) * d;
            for (int b = 0; b < d; ++b) o[b] = 0.0;
            for (int s = t0; s <= t; ++s) {
                double score = 0.0;                  /* (Q K^T)[t][s] */
                for (int a = 0; a < d; ++a)
                    score += widen_bf16(ROW(q, t, h)[a]) * widen_bf16(ROW(k, s, h)[a]);
                for (int b = 0; b < d; ++b)
                    o[b] += score * widen_bf16(ROW(v, s, h)[b]);
            }
            if (Sin)
                for (int a = 0; a < d; ++a) {
                    const double qa = widen_bf16(ROW(q, t, h)[a]);
                    for (int b = 0; b < d; ++b) o[b] += qa * Sin[(size_t)a * d + b];
                }
        }
        if (state_out) {
            /* final state: S_in + K^T V over the whole sequence */
            double *S = state_out + (size_t)p * d * d;
            for (size_t e = 0; e < (size_t)d * d; ++e) S[e] = Sin ? Sin[e] : 0.0;
            for (int s = t0; s < t1; ++s)
                for (int a = 0; a < d; ++a) {
                    const double ka = widen_bf16(ROW(k, s, h)[a]);
                    for (int b = 0; b < d; ++b)
                        S[(size_t)a * d + b] += ka * widen_bf16(ROW(v, s, h)[b]);
                }
        }
    }
    return 0;
}

/*
 * Blocked form ([P2]/[P5] §2.2): Q, K, V are split along the sequence into row
 * blocks of `block` tokens (the last block of a sequence may be shorter).
 * Within block b the left product is used, across blocks the right product:
 *   O_b     = (Q_b K_b^T ⊙ M_b) V_b + Q_b S_{<b}
 *   S_{<=b} = S_{<b} + K_b^T V_b,          S_{<0} = S_in.
 */
static void blocked_one(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        int H, int d, int h, int j, int nh, int t0, int t1,
                        int block, double *S, double *out)
{
    for (int b0 = t0; b0 < t1; b0 += block) {
        const int b1 = (b0 + block < t1) ? b0 + block : t1;
        for (int t = b0; t < b1; ++t) {
            double *o = out + ((size_t)t * nh + j) * d;
            for (int b = 0; b < d; ++b) o[b] = 0.0;
            /* intra-block left product (Q_b K_b^T ⊙ M_b) V_b */
            for (int s = b0; s <= t; ++s) {
                double score = 0.0;
                for (int a = 0; a < d; ++a)
                    score += widen_bf16(ROW(q, t, h)[a]) * widen_bf16(ROW(k, s, h)[a]);
                for (int b = 0; b < d; ++b)
                    o[b] += score * widen_bf16(ROW(v, s, h)[b]);
            }
            /* inter-block right product Q_b S_{<b} */
            for (int a = 0; a < d; ++a) {
                const double qa = widen_bf16(ROW(q, t, h)[a]);
                for (int b = 0; b < d; ++b) o[b] += qa * S[(size_t)a * d + b];
            }
        }
        /* S_{<=b} = S_{<b} + K_b^T V_b */
        for (int s = b0; s < b1; ++s)
            for (int a = 0; a < d; ++a) {
                const double ka = widen_bf16(ROW(k, s, h)[a]);
                for (int b = 0; b < d; ++b)
                    S[(size_t)a * d + b] += ka * widen_bf16(ROW(v, s, h)[b]);
            }
    }
}

int lao_blocked(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                const int32_t *cu_seqlens, int nseq, int H, int d,
                const int32_t *heads, int nh, int block, const double *state_in,
                double *out, double *state_out, int nthreads)
{
    if (!q || !k || !v || !out || block <= 0) return -1;
    if (check_common(cu_seqlens, nseq, H, d, heads, nh)) return -1;
    set_threads(nthreads);
    const long npairs = (long)nseq * nh;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long p = 0; p < npairs; ++p) {
        const int i = (int)(p / nh), j = (int)(p % nh);
        const int h = heads ? heads[j] : j;
        double *S = (double *)calloc((size_t)d * d, sizeof(double));
        if (!S) { bad = 1; continue; }
        if (state_in)
            memcpy(S, state_in + (size_t)p * d * d, (size_t)d * d * sizeof(double));
        blocked_one(q, k, v, H, d, h, j, nh, cu_seqlens[i], cu_seqlens[i + 1],
                    block, S, out);
        if (state_out)
            memcpy(state_out + (size_t)p * d * d, S, (size_t)d * d * sizeof(double));
        free(S);
    }
    return bad ? -1 : 0;
}

/*
 * Segmented form, the LASP+ recipe of [P5] §3.2 item 3 applied to the
 * segments of one sequence instead of to ranks:
 *   1. every segment r (seg_len tokens, the last one shorter) computes its
 *      local KV sum KV_r = sum_{s in r} k_s^T v_s;
 *   2. the local sums are gathered;
 *   3. segment r forms its global prefix KV_G(r) = S_in + sum_{r' < r} KV_r'
 *      and runs the blocked form over its own tokens starting from it.
 * The final state is KV_G(last) + KV_last.
 */
int lao_segmented(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                  const int32_t *cu_seqlens, int nseq, int H, int d,
                  const int32_t *heads, int nh, int seg_len, int block,
                  const double *state_in, double *out, double *state_out,
                  int nthreads)
{
    if (!q || !k || !v || !out || block <= 0 || seg_len <= 0) return -1;
    if (check_common(cu_seqlens, nseq, H, d, heads, nh)) return -1;
    set_threads(nthreads);
    const long npairs = (long)nseq * nh;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long p = 0; p < npairs; ++p) {
        const int i = (int)(p / nh), j = (int)(p % nh);
        const int h = heads ? heads[j] : j;
        const int t0 = cu_seqlens[i], t1 = cu_seqlens[i + 1];
        const int nseg = (t1 - t0 + seg_len - 1) / seg_len;
        const size_t dd = (size_t)d * d;
        /* step 1: local sums, one per segment (the "gathered" array of step 2) */
        double *local = (double *)calloc((size_t)(nseg > 0 ? nseg : 1) * dd, sizeof(double));
        double *G = (double *)malloc(dd * sizeof(double));
        if (!local || !G) { bad = 1; free(local); free(G); continue; }
        for (int r = 0; r < nseg; ++r) {
            const int s0 = t0 + r * seg_len;
            const int s1 = (s0 + seg_len < t1) ? s0 + seg_len : t1;
            double *L = local + (size_t)r * dd;
            for (int s = s0; s < s1; ++s)
                for (int a = 0; a < d; ++a) {
                    const double ka = widen_bf16(ROW(k, s, h)[a]);
                    for (int b = 0; b < d; ++b)
                        L[(size_t)a * d + b] += ka * widen_bf16(ROW(v, s, h)[b]);
                }
        }
        /* step 3: each segment's global prefix, then its blocked scan */
        for (int r = 0; r < nseg; ++r) {
            for (size_t e = 0; e < dd; ++e)
                G[e] = state_in ? state_in[(size_t)p * dd + e] : 0.0;
            for (int r2 = 0; r2 < r; ++r2)
                for (size_t e = 0; e < dd; ++e) G[e] += local[(size_t)r2 * dd + e];
            const int s0 = t0 + r * seg_len;
            const int s1 = (s0 + seg_len < t1) ? s0 + seg_len : t1;
            blocked_one(q, k, v, H, d, h, j, nh, s0, s1, block, G, out);
        }
        if (state_out) {
            double *So = state_out + (size_t)p * dd;
            for (size_t e = 0; e < dd; ++e)
                So[e] = state_in ? state_in[(size_t)p * dd + e] : 0.0;
            for (int r = 0; r < nseg; ++r)
                for (size_t e = 0; e < dd; ++e) So[e] += local[(size_t)r * dd + e];
        }
        free(local); free(G);
    }
    return bad ? -1 : 0;
}

/*
 * One decode step on a persistent state ([P5] §3.3 items 1-2: length-1 tokens
 * go to their own kernel, whose KV computation is fused with the update of
 * the prefix-KV cache).  For every (b, h):
 *   S <- S + k^T v,   o = q S          (inclusive: the new token sees itself)
 * q, k, v: bf16 bits [B][H][d]; state: double [B][H][d][d] updated in place;
 * out: double [B][H][d].
 */
int lao_decode_step(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                    int B, int H, int d, double *state, double *out, int nthreads)
{
    if (!q || !k || !v || !state || !out || B < 0 || H <= 0 || d <= 0) return -1;
    set_threads(nthreads);
    const long npairs = (long)B * H;
#pragma omp parallel for schedule(static)
    for (long p = 0; p < npairs; ++p) {
        double *S = state + (size_t)p * d * d;
        const uint16_t *qp = q + (size_t)p * d, *kp = k + (size_t)p * d, *vp = v + (size_t)p * d;
        for (int a = 0; a < d; ++a) {
            const double ka = widen_bf16(kp[a]);
            for (int b = 0; b < d; ++b) S[(size_t)a * d + b] += ka * widen_bf16(vp[b]);
        }
        double *o = out + (size_t)p * d;
        for (int b = 0; b < d; ++b) o[b] = 0.0;
        for (int a = 0; a < d; ++a) {
            const double qa = widen_bf16(qp[a]);
            for (int b = 0; b < d; ++b) o[b] += qa * S[(size_t)a * d + b];
        }
    }
    return 0;
}

/*
 * Gradients of the forward definition (lao_quadratic) for a loss L with
 * dL/do_t = g_t (dout, bf16 bits [T][H][d]) and dL/dS_out = G_S (dstate_out,
 * double [nseq][nh][d][d] or NULL = 0), where
 *   o_t   = sum_{s <= t} (q_t . k_s) v_s + q_t S_in,
 *   S_out = S_in + sum_s k_s^T v_s.
 * Differentiating term by term:
 *   dq_t = sum_{s <= t} (g_t . v_s) k_s + g_t S_in^T
 *   dk_s = sum_{t >= s} (g_t . v_s) q_t + v_s G_S^T
 *   dv_s = sum_{t >= s} (q_t . k_s) g_t + k_s G_S
 *   dS_in = sum_t q_t^T g_t + G_S
 * (row vectors; (x M^T)[a] = sum_b M[a][b] x[b]).  Plain O(n^2 d) loops per
 * (sequence, head).  dq, dk, dv: double [T][nh][d]; dstate_in: double
 * [nseq][nh][d][d] or NULL.
 */
int lao_backward(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint16_t *dout,
                 const int32_t *cu_seqlens, int nseq, int H, int d,
                 const int32_t *heads, int nh, const double *state_in,
                 const double *dstate_out, double *dq, double *dk, double *dv,
                 double *dstate_in, int nthreads)
{
    if (!q || !k || !v || !dout || !dq || !dk || !dv) return -1;
    if (check_common(cu_seqlens, nseq, H, d, heads, nh)) return -1;
    set_threads(nthreads);
    const long npairs = (long)nseq * nh;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long p = 0; p < npairs; ++p) {
        const int i = (int)(p / nh), j = (int)(p % nh);
        const int h = heads ? heads[j] : j;
        const int t0 = cu_seqlens[i], n = cu_seqlens[i + 1] - cu_seqlens[i];
        const size_t nd = (size_t)(n > 0 ? n : 1) * d;
        double *Q = (double *)malloc(nd * sizeof(double));
        double *K = (double *)malloc(nd * sizeof(double));
        double *V = (double *)malloc(nd * sizeof(double));
        double *G = (double *)malloc(nd * sizeof(double));
        if (!Q || !K || !V || !G) {
            bad = 1;
            free(Q); free(K); free(V); free(G);
            continue;
        }
        for (int t = 0; t < n; ++t)
            for (int a = 0; a < d; ++a) {
                Q[(size_t)t * d + a] = widen_bf16(ROW(q, t0 + t, h)[a]);
                K[(size_t)t * d + a] = widen_bf16(ROW(k, t0 + t, h)[a]);
                V[(size_t)t * d + a] = widen_bf16(ROW(v, t0 + t, h)[a]);
                G[(size_t)t * d + a] = widen_bf16(ROW(dout, t0 + t, h)[a]);
            }
        const double *Sin = state_in ? state_in + (size_t)p * d * d : NULL;
        const double *GS = dstate_out ? dstate_out + (size_t)p * d * d : NULL;
        for (int t = 0; t < n; ++t) {
            /* dq_t = sum_{s <= t} (g_t . v_s) k_s + g_t S_in^T */
            double *o = dq + ((size_t)(t0 + t) * nh + j) * d;
            for (int a = 0; a < d; ++a) o[a] = 0.0;
            for (int s2 = 0; s2 <= t; ++s2) {
                double w = 0.0;
                for (int b = 0; b < d; ++b) w += G[(size_t)t * d + b] * V[(size_t)s2 * d + b];
                for (int a = 0; a < d; ++a) o[a] += w * K[(size_t)s2 * d + a];
            }
            if (Sin)
                for (int a = 0; a < d; ++a)
                    for (int b = 0; b < d; ++b) o[a] += Sin[(size_t)a * d + b] * G[(size_t)t * d + b];
        }
        for (int s2 = 0; s2 < n; ++s2) {
            /* dk_s = sum_{t >= s} (g_t . v_s) q_t + v_s G_S^T
               dv_s = sum_{t >= s} (q_t . k_s) g_t + k_s G_S */
            double *ok = dk + ((size_t)(t0 + s2) * nh + j) * d;
            double *ov = dv + ((size_t)(t0 + s2) * nh + j) * d;
            for (int a = 0; a < d; ++a) ok[a] = ov[a] = 0.0;
            for (int t = s2; t < n; ++t) {
                double wk = 0.0, wv = 0.0;
                for (int b = 0; b < d; ++b) {
                    wk += G[(size_t)t * d + b] * V[(size_t)s2 * d + b];
                    wv += Q[(size_t)t * d + b] * K[(size_t)s2 * d + b];
                }
                for (int a = 0; a < d; ++a) {
                    ok[a] += wk * Q[(size_t)t * d + a];
                    ov[a] += wv * G[(size_t)t * d + a];
                }
            }
            if (GS)
                for (int a = 0; a < d; ++a)
                    for (int b = 0; b < d; ++b) {
                        ok[a] += GS[(size_t)a * d + b] * V[(size_t)s2 * d + b];
                        ov[b] += K[(size_t)s2 * d + a] * GS[(size_t)a * d + b];
                    }
        }
        if (dstate_in) {
            /* dS_in = sum_t q_t^T g_t + G_S */
            double *D = dstate_in + (size_t)p * d * d;
            for (size_t e = 0; e < (size_t)d * d; ++e) D[e] = GS ? GS[e] : 0.0;
            for (int t = 0; t < n; ++t)
                for (int a = 0; a < d; ++a)
                    for (int b = 0; b < d; ++b)
                        D[(size_t)a * d + b] += Q[(size_t)t * d + a] * G[(size_t)t * d + b];
        }
        free(Q); free(K); free(V); free(G);
    }
    return bad ? -1 : 0;
}

/* ===========================================================================
 * Per-head decay.  [P5] §3.3 item 1 names a "decay value computation" fused
 * into the prefill and [P2]/[P5] §2.3 describe the attention as the
 * "transnormer" block, but no page gives the formula.  Reading (stated, not
 * printed on the pages): the decayed recurrence of the TransNormer /
 * Lightning Attention line, one constant lambda_h in (0, 1] per head h,
 *
 *   S_t = lambda S_{t-1} + k_t^T v_t,   o_t = q_t S_t,   S_{-1} = S_in,
 *
 * with t counted from the start of the sequence, equivalently
 *
 *   o_t = sum_{s <= t} lambda^{t-s} (q_t . k_s) v_s + lambda^{t+1} q_t S_in.
 *
 * lambda = 1 is the undecayed operation above (each decayed form below then
 * reproduces its undecayed counterpart bit for bit: every extra factor is an
 * exact 1.0).  `decay` is double [H], indexed by the head number h (not by the
 * position in `heads`).  Powers lambda^n use the C library's pow().
 * ======================================================================== */
static int check_decay(const double *decay, int H)
{
    if (!decay) return -1;
    for (int h = 0; h < H; ++h)
        if (!(decay[h] >= 0.0 && decay[h] <= 1.0)) return -1;
    return 0;
}

/* Decayed recurrent form: S_t = lambda S_{t-1} + k_t^T v_t, o_t = q_t S_t. */
int lao_recurrent_decay(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        const int32_t *cu_seqlens, int nseq, int H, int d,
                        const int32_t *heads, int nh, const double *decay,
                        const double *state_in, double *out, double *state_out,
                        int nthreads)
{
    if (!q || !k || !v || !out) return -1;
    if (check_common(cu_seqlens, nseq, H, d, heads, nh) || check_decay(decay, H)) return -1;
    set_threads(nthreads);
    const long npairs = (long)nseq * nh;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long p = 0; p < npairs; ++p) {
        const int i = (int)(p / nh), j = (int)(p % nh);
        const int h = heads ? heads[j] : j;
        const double lam = decay[h];
        double *S = (double *)calloc((size_t)d * d, sizeof(double));
        double *kt = (double *)malloc((size_t)d * sizeof(double));
        double *vt = (double *)malloc((size_t)d * sizeof(double));
        double *qt = (double *)malloc((size_t)d * sizeof(double));
        if (!S || !kt || !vt || !qt) {
            bad = 1;
            free(S); free(kt); free(vt); free(qt);
            continue;
        }
        if (state_in)
            memcpy(S, state_in + (size_t)p * d * d, (size_t)d * d * sizeof(double));
        for (int t = cu_seqlens[i]; t < cu_seqlens[i + 1]; ++t) {
            for (int a = 0; a < d; ++a) {
                qt[a] = widen_bf16(ROW(q, t, h)[a]);
                kt[a] = widen_bf16(ROW(k, t, h)[a]);
                vt[a] = widen_bf16(ROW(v, t, h)[a]);
            }
            /* S_t = lambda S_{t-1} + k_t^T v_t */
            for (int a = 0; a < d; ++a)
                for (int b = 0; b < d; ++b)
                    S[(size_t)a * d + b] = lam * S[(size_t)a * d + b] + kt[a] * vt[b];
            /* o_t = q_t S_t */
            double *o = out + ((size_t)t * nh + j) * d;
            for (int b = 0; b < d; ++b) o[b] = 0.0;
            for (int a = 0; a < d; ++a)
                for (int b = 0; b < d; ++b)
                    o[b] += qt[a] * S[(size_t)a * d + b];
        }
        if (state_out)
            memcpy(state_out + (size_t)p * d * d, S, (size_t)d * d * sizeof(double));
        free(S); free(kt); free(vt); free(qt);
    }
    return bad ? -1 : 0;
}

/*
 * Decayed quadratic form, the closed form of the recurrence:
 *   o_t   = sum_{s <= t} lambda^{t-s} (q_t . k_s) v_s + lambda^{t-t0+1} q_t S_in
 *   S_out = lambda^{n} S_in + sum_s lambda^{t1-1-s} k_s^T v_s
 * (t0, t1 = the sequence's first and one-past-last token, n = t1 - t0).
 */
int lao_quadratic_decay(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        const int32_t *cu_seqlens, int nseq, int H, int d,
                        const int32_t *heads, int nh, const double *decay,
                        const double *state_in, double *out, double *state_out,
                        int nthreads)
{
    if (!q || !k || !v || !out) return -1;
    if (check_common(cu_seqlens, nseq, H, d, heads, nh) || check_decay(decay, H)) return -1;
    set_threads(nthreads);
    const long npairs = (long)nseq * nh;
#pragma omp parallel for schedule(dynamic, 1)
    for (long p = 0; p < npairs; ++p) {
        const int i = (int)(p / nh), j = (int)(p % nh);
        const int h = heads ? heads[j] : j;
        const double lam = decay[h];
        const int t0 = cu_seqlens[i], t1 = cu_seqlens[i + 1];
        const double *Sin = state_in ? state_in + (size_t)p * d * d : NULL;
        for (int t = t0; t < t1; ++t) {
            double *o = out + ((size_t)t * nh + j) * d;
            for (int b = 0; b < d; ++b) o[b] = 0.0;
            for (int s = t0; s <= t; ++s) {
                double score = 0.0;                  /* (Q K^T)[t][s] */
                for (int a = 0; a < d; ++a)
                    score += widen_bf16(ROW(q, t, h)[a]) * widen_bf16(ROW(k, s, h)[a]);
                const double w = score * pow(lam, (double)(t - s));
                for (int b = 0; b < d; ++b)
                    o[b] += w * widen_bf16(ROW(v, s, h)[b]);
            }
            if (Sin) {
                const double f = pow(lam, (double)(t - t0 + 1));
                for (int a = 0; a < d; ++a) {
                    const double qa = widen_bf16(ROW(q, t, h)[a]) * f;
                    for (int b = 0; b < d; ++b) o[b] += qa * Sin[(size_t)a * d + b];
                }
            }
        }
        if (state_out) {
            double *S = state_out + (size_t)p * d * d;
            const double f = pow(lam, (double)(t1 - t0));
            for (size_t e = 0; e < (size_t)d * d; ++e) S[e] = Sin ? f * Sin[e] : 0.0;
            for (int s = t0; s < t1; ++s) {
                const double w = pow(lam, (double)(t1 - 1 - s));
                for (int a = 0; a < d; ++a) {
                    const double ka = widen_bf16(ROW(k, s, h)[a]) * w;
                    for (int b = 0; b < d; ++b)
                        S[(size_t)a * d + b] += ka * widen_bf16(ROW(v, s, h)[b]);
                }
            }
        }
    }
    return 0;
}

/*
 * Decayed blocked form (the blocked algorithm of [P2]/[P5] §2.2 with the
 * decay of the reading above).  Rows b0 <= t < b1 of one block, local index
 * r = t - b0, block length nb = b1 - b0:
 *   O_b     = ((Q_b K_b^T) ⊙ D_b) V_b + diag(lambda^{r+1}) Q_b S_{<b},
 *             D_b[r][c] = lambda^{r-c} for c <= r, else 0
 *   S_{<=b} = lambda^{nb} S_{<b} + sum_{c} lambda^{nb-1-c} k_{b0+c}^T v_{b0+c}
 */
static void blocked_decay_one(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                              int H, int d, int h, int j, int nh, int t0, int t1,
                              int block, double lam, double *S, double *out)
{
    for (int b0 = t0; b0 < t1; b0 += block) {
        const int b1 = (b0 + block < t1) ? b0 + block : t1;
        for (int t = b0; t < b1; ++t) {
            double *o = out + ((size_t)t * nh + j) * d;
            for (int b = 0; b < d; ++b) o[b] = 0.0;
            /* intra-block left product ((Q_b K_b^T) ⊙ D_b) V_b */
            for (int s = b0; s <= t; ++s) {
                double score = 0.0;
                for (int a = 0; a < d; ++a)
                    score += widen_bf16(ROW(q, t, h)[a]) * widen_bf16(ROW(k, s, h)[a]);
                const double w = score * pow(lam, (double)(t - s));
                for (int b = 0; b < d; ++b)
                    o[b] += w * widen_bf16(ROW(v, s, h)[b]);
            }
            /* inter-block right product lambda^{r+1} q_t S_{<b} */
            const double f = pow(lam, (double)(t - b0 + 1));
            for (int a = 0; a < d; ++a) {
                const double qa = widen_bf16(ROW(q, t, h)[a]) * f;
                for (int b = 0; b < d; ++b) o[b] += qa * S[(size_t)a * d + b];
            }
        }
        /* S_{<=b} = lambda^{nb} S_{<b} + sum_c lambda^{nb-1-c} k^T v */
        const double f = pow(lam, (double)(b1 - b0));
        for (size_t e = 0; e < (size_t)d * d; ++e) S[e] *= f;
        for (int s = b0; s < b1; ++s) {
            const double w = pow(lam, (double)(b1 - 1 - s));
            for (int a = 0; a < d; ++a) {
                const double ka = widen_bf16(ROW(k, s, h)[a]) * w;
                for (int b = 0; b < d; ++b)
                    S[(size_t)a * d + b] += ka * widen_bf16(ROW(v, s, h)[b]);
            }
        }
    }
}

int lao_blocked_decay(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                      const int32_t *cu_seqlens, int nseq, int H, int d,
                      const int32_t *heads, int nh, int block, const double *decay,
                      const double *state_in, double *out, double *state_out, int nthreads)
{
    if (!q || !k || !v || !out || block <= 0) return -1;
    if (check_common(cu_seqlens, nseq, H, d, heads, nh) || check_decay(decay, H)) return -1;
    set_threads(nthreads);
    const long npairs = (long)nseq * nh;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long p = 0; p < npairs; ++p) {
        const int i = (int)(p / nh), j = (int)(p % nh);
        const int h = heads ? heads[j] : j;
        double *S = (double *)calloc((size_t)d * d, sizeof(double));
        if (!S) { bad = 1; continue; }
        if (state_in)
            memcpy(S, state_in + (size_t)p * d * d, (size_t)d * d * sizeof(double));
        blocked_decay_one(q, k, v, H, d, h, j, nh, cu_seqlens[i], cu_seqlens[i + 1],
                          block, decay[h], S, out);
        if (state_out)
            memcpy(state_out + (size_t)p * d * d, S, (size_t)d * d * sizeof(double));
        free(S);
    }
    return bad ? -1 : 0;
}

/*
 * Decayed segmented form (the LASP+ recipe of [P5] §3.2 item 3 over the
 * segments of one sequence, with the decay of the reading above):
 *   1. local sums   A_r = sum_{s in r} lambda^{e_r-1-s} k_s^T v_s
 *      (segment r = tokens [s_r, e_r));
 *   2. the local sums are gathered;
 *   3. global prefix G_r = lambda^{s_r-t0} S_in + sum_{r' < r} lambda^{s_r-e_r'} A_r',
 *      then the decayed blocked form over segment r starting from G_r.
 * The final state is lambda^{n} S_in + sum_r lambda^{t1-e_r} A_r.
 */
int lao_segmented_decay(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        const int32_t *cu_seqlens, int nseq, int H, int d,
                        const int32_t *heads, int nh, int seg_len, int block,
                        const double *decay, const double *state_in, double *out,
                        double *state_out, int nthreads)
{
    if (!q || !k || !v || !out || block <= 0 || seg_len <= 0) return -1;
    if (check_common(cu_seqlens, nseq, H, d, heads, nh) || check_decay(decay, H)) return -1;
    set_threads(nthreads);
    const long npairs = (long)nseq * nh;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (long p = 0; p < npairs; ++p) {
        const int i = (int)(p / nh), j = (int)(p % nh);
        const int h = heads ? heads[j] : j;
        const double lam = decay[h];
        const int t0 = cu_seqlens[i], t1 = cu_seqlens[i + 1];
        const int nseg = (t1 - t0 + seg_len - 1) / seg_len;
        const size_t dd = (size_t)d * d;
        double *local = (double *)calloc((size_t)(nseg > 0 ? nseg : 1) * dd, sizeof(double));
        double *G = (double *)malloc(dd * sizeof(double));
        if (!local || !G) { bad = 1; free(local); free(G); continue; }
        /* step 1: local sums */
        for (int r = 0; r < nseg; ++r) {
            const int s0 = t0 + r * seg_len;
            const int s1 = (s0 + seg_len < t1) ? s0 + seg_len : t1;
            double *L = local + (size_t)r * dd;
            for (int s = s0; s < s1; ++s) {
                const double w = pow(lam, (double)(s1 - 1 - s));
                for (int a = 0; a < d; ++a) {
                    const double ka = widen_bf16(ROW(k, s, h)[a]) * w;
                    for (int b = 0; b < d; ++b)
                        L[(size_t)a * d + b] += ka * widen_bf16(ROW(v, s, h)[b]);
                }
            }
        }
        /* step 3: global prefix of each segment, then its blocked scan */
        for (int r = 0; r < nseg; ++r) {
            const int s0 = t0 + r * seg_len;
            const int s1 = (s0 + seg_len < t1) ? s0 + seg_len : t1;
            const double fin = pow(lam, (double)(s0 - t0));
            for (size_t e = 0; e < dd; ++e)
                G[e] = state_in ? fin * state_in[(size_t)p * dd + e] : 0.0;
            for (int r2 = 0; r2 < r; ++r2) {
                const int e2 = t0 + (r2 + 1) * seg_len;     /* end of segment r2 (< t1) */
                const double f = pow(lam, (double)(s0 - e2));
                for (size_t e = 0; e < dd; ++e) G[e] += f * local[(size_t)r2 * dd + e];
            }
            blocked_decay_one(q, k, v, H, d, h, j, nh, s0, s1, block, lam, G, out);
        }
        if (state_out) {
            double *So = state_out + (size_t)p * dd;
            const double fin = pow(lam, (double)(t1 - t0));
            for (size_t e = 0; e < dd; ++e)
                So[e] = state_in ? fin * state_in[(size_t)p * dd + e] : 0.0;
            for (int r = 0; r < nseg; ++r) {
                const int e_r = (t0 + (r + 1) * seg_len < t1) ? t0 + (r + 1) * seg_len : t1;
                const double f = pow(lam, (double)(t1 - e_r));
                for (size_t e = 0; e < dd; ++e) So[e] += f * local[(size_t)r * dd + e];
            }
        }
        free(local); free(G);
    }
    return bad ? -1 : 0;
}

/*
 * One decayed decode step (the decode step of [P5] §3.3 items 1-2 under the
 * decay reading above).  For every (b, h):
 *   S <- lambda_h S + k^T v,   o = q S.
 */
int lao_decode_step_decay(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          int B, int H, int d, const double *decay, double *state,
                          double *out, int nthreads)
{
    if (!q || !k || !v || !state || !out || B < 0 || H <= 0 || d <= 0) return -1;
    if (check_decay(decay, H)) return -1;
    set_threads(nthreads);
    const long npairs = (long)B * H;
#pragma omp parallel for schedule(static)
    for (long p = 0; p < npairs; ++p) {
        const double lam = decay[p % H];
        double *S = state + (size_t)p * d * d;
        const uint16_t *qp = q + (size_t)p * d, *kp = k + (size_t)p * d, *vp = v + (size_t)p * d;
        for (int a = 0; a < d; ++a) {
            const double ka = widen_bf16(kp[a]);
            for (int b = 0; b < d; ++b)
                S[(size_t)a * d + b] = lam * S[(size_t)a * d + b] + ka * widen_bf16(vp[b]);
        }
        double *o = out + (size_t)p * d;
        for (int b = 0; b < d; ++b) o[b] = 0.0;
        for (int a = 0; a < d; ++a) {
            const double qa = widen_bf16(qp[a]);
            for (int b = 0; b < d; ++b) o[b] += qa * S[(size_t)a * d + b];
        }
    }
    return 0;
}
