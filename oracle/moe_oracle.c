/*
 * moe_oracle.c -- plain, slow, fp64 CPU oracle of the forward pass of a
 * top-k routed Mixture-of-Experts SwiGLU FFN layer.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg load this library. The product (the CUDA
 * library and its Python binding) never calls it, shares no code, header,
 * table or helper with it, and must fail loudly rather than fall back here.
 *
 * What it follows (web pages that define the layer):
 *  [MIX] "MoE Model Architectures" (architectures.md), section "Mixtral 8x7B",
 *        subsections "Sparse MoE Block" (gate -> softmax over all experts ->
 *        top-k -> divide by the top-k sum -> per-expert FFN on the routed rows
 *        -> scale by the routing weight -> index_add into token order) and
 *        "Expert FFN" (w2(silu(w1 x) * w3 x), no biases).
 *  [DSK] same page, section "DeepSeek-V3": "DeepSeekMoE Architecture" (shared
 *        experts always run and are added unweighted) and "Auxiliary-Loss-Free
 *        Load Balancing" (F.linear(x, W, b): a per-expert bias on the logits).
 *  [SWT] same page, section "Switch Transformers", "Top-1 Routing" (an expert
 *        capacity beyond which routed tokens are dropped; the printed mask is
 *        garbled: it compares per-expert totals, not per-token ranks).
 *  [CUR] "Current Bug: CuTeDSLMoERunner produces wrong output", sections "How
 *        the pipeline works" / "How the runner currently works": token counts
 *        [4,4,0] give expert offsets [4,8,8], or [0,4,8,8] with a leading 0.
 *  [MGA] "Faster writing: run only the chosen experts; uncap the large profile"
 *        (a capacity factor of 0 means uncapped).
 *
 * Readings taken where the pages are silent or garbled:
 *  R1  top-k is chosen on the fp32 logits. Softmax is strictly increasing in
 *      the logit, so this is the top-k of [MIX]'s probabilities wherever those
 *      are not rounded to equal values. Ties go to the lowest expert index;
 *      -0.0 and +0.0 compare equal. Output order is selection order.
 *  R2  the weights are [MIX]'s softmax over all E, restricted to the top-k
 *      and divided by their sum (computed literally, in fp64).
 *  R3  capacity C: an assignment (t, j) is kept iff fewer than C assignments
 *      to the same expert come before it in row-major (token, slot) order;
 *      C <= 0 is uncapped ([MGA]). Kept weights are not renormalised; a
 *      dropped assignment contributes nothing.
 *      Slot-priority variant (R3b): the same rule with the assignments in
 *      slot-major (slot, token) order, so every token's first choice is
 *      placed before any token's second choice (the priority GShard/GLaM-style
 *      top-2 dispatch gives the first expert; the page's comparison table
 *      names GLaM's capacity-factor tuning, and its Switch mask is garbled).
 *  R4  expert offsets have E+1 entries with a leading 0 ([CUR]'s GPU form);
 *      an expert's kept rows are laid out in rank order: ascending token (R3),
 *      or by slot, then ascending token (R3b).
 *  R5  the bias enters both the selection and the weights ([DSK]'s
 *      F.linear(x, W, b) feeds the softmax); a shared expert is added with
 *      weight 1.
 *  R6  the SwiGLU product h is optionally rounded to bf16 (round to nearest,
 *      ties to even) before w2, modelling the one rounding a bf16 tensor-core
 *      path must make; with h_bf16 = 0 the whole layer is pure fp64.
 *  R7  block-scaled 8-bit experts (precision mode 2): MXFP8 as defined at
 *      oracle_e4m3_decode, applied to x, to every expert weight row and to h
 *      along the contraction dimension; the router stays on bf16 weights.
 *  R8  the backward pass differentiates the fp64 layer with the routing
 *      decisions (top-k set, drops, slots) held fixed; see
 *      oracle_moe_backward.
 *
 * Inputs are bf16 bit patterns (uint16) and are widened exactly to double.
 * Error codes: 0 ok, 1 invalid argument, 5 non-finite logit, 6 bad expert id.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_OK 0
#define ORC_EINVAL 1
#define ORC_ENONFINITE 5
#define ORC_EBADEXPERT 6

/* bf16 is the upper half of an IEEE binary32; widening is exact. */
static double bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 value (8 significant bits, binary32
 * exponent range), ties to even, returned as a double. */
double oracle_round_bf16(double v)
{
    if (!isfinite(v) || v == 0.0)
        return v;
    int e;
    (void)frexp(v, &e);           /* v = m * 2^e, 0.5 <= |m| < 1 */
    int q = e - 8;                /* weight of the last kept bit */
    if (q < -133)                 /* bf16 subnormals: spacing 2^-133 */
        q = -133;
    double r = nearbyint(ldexp(v, -q));   /* default mode: ties to even */
    double out = ldexp(r, q);
    if (fabs(out) > 3.3895313892515355e38)  /* past the largest finite bf16 */
        out = copysign(INFINITY, v);
    return out;
}

/* Widen a bf16 array to double (helper for callers that want the values). */
void oracle_bf16_to_f64(int64_t n, const uint16_t *src, double *dst)
{
    for (int64_t i = 0; i < n; ++i)
        dst[i] = bf16_to_double(src[i]);
}

/* ---- MXFP8: OCP "Microscaling (MX) Formats" v1.0, element type E4M3 with
 * one shared E8M0 (power-of-two) scale per block of 32 consecutive elements
 * along the contraction dimension. The pages name block-scaled 4- and 8-bit
 * expert weights and activations ("Current Bug: CuTeDSLMoERunner produces
 * wrong output": per-expert activation and weight scale factors) without
 * fixing the encoding; reading R7 takes MXFP8 for weights and activations:
 *  - E4M3: sign, 4 exponent bits (bias 7), 3 mantissa bits, subnormals
 *    m/8 * 2^-6, largest finite 448, no infinities, S.1111.111 = NaN;
 *  - the shared scale of a block is 2^X with X = floor(log2(max|v|)) - 8,
 *    8 being the exponent of E4M3's largest normal power of two (the
 *    standard's conversion of a vector of scalars to an MX block), clamped
 *    to the E8M0 range [-127, 127]; an all-zero block takes X = -127. E8M0
 *    code X + 127;
 *  - each element is v * 2^-X rounded to the nearest E4M3 value, ties to
 *    even, saturating at 448: the block maximum lands in [256, 512), and
 *    scaled magnitudes of 464 and above clamp to 448 (the standard's
 *    saturating conversion). The sign of a zero result is the sign of v. */
double oracle_e4m3_decode(int code)
{
    const int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7)
        return NAN;
    const double v = (e == 0) ? ldexp((double)m, -9)          /* m/8 * 2^-6 */
                              : ldexp(8.0 + m, e - 10);       /* (1 + m/8) * 2^(e-7) */
    return s ? -v : v;
}

/* Nearest E4M3 value of |v| (ties to even), as in oracle_round_bf16: keep 3
 * fractional bits in the binade of |v|, or a spacing of 2^-9 below 2^-6;
 * saturate at 448. Returns the code. */
int oracle_e4m3_encode(double v)
{
    const double a = fabs(v);
    double r;
    if (a < ldexp(1.0, -6)) {
        r = ldexp(nearbyint(ldexp(a, 9)), -9);
    } else {
        int e;
        (void)frexp(a, &e);               /* a = f * 2^e, 0.5 <= f < 1 */
        const int q = e - 1 - 3;          /* weight of the last mantissa bit */
        r = ldexp(nearbyint(ldexp(a, -q)), q);
    }
    if (r > 448.0)
        r = 448.0;
    int code;
    if (r < ldexp(1.0, -6)) {
        code = (int)ldexp(r, 9);          /* subnormal (or zero): m = r / 2^-9 */
    } else {
        int e;
        const double f = frexp(r, &e);    /* r = f * 2^e = (1 + m/8) 2^(e-1) */
        const int m = (int)((2.0 * f - 1.0) * 8.0);
        code = ((e - 1 + 7) << 3) | m;
    }
    return code | (signbit(v) ? 0x80 : 0);
}

/* Shared exponent X of a block with maximum magnitude amax:
 * floor(log2(amax)) - 8, clamped to [-127, 127]; -127 for amax = 0. */
int oracle_mx_scale_exp(double amax)
{
    if (!(amax > 0.0))
        return -127;
    int e;
    (void)frexp(amax, &e);   /* amax = f * 2^e with 0.5 <= f < 1: floor(log2 amax) = e - 1 */
    int X = e - 1 - 8;
    if (X < -127)
        X = -127;
    if (X > 127)
        X = 127;
    return X;
}

/* Quantize rows x K (K a multiple of 32) of doubles to MXFP8:
 * codes [rows, K] (E4M3), scales [rows, K / 32] (E8M0). */
int oracle_mx_quantize(int64_t rows, int K, const double *in, uint8_t *codes, uint8_t *scales)
{
    if (rows < 0 || K < 32 || K % 32 != 0 || !in || !codes || !scales)
        return ORC_EINVAL;
    for (int64_t r = 0; r < rows; ++r)
        for (int b = 0; b < K / 32; ++b) {
            const double *v = in + r * K + b * 32;
            double amax = 0.0;
            for (int i = 0; i < 32; ++i)
                if (fabs(v[i]) > amax)
                    amax = fabs(v[i]);
            const int X = oracle_mx_scale_exp(amax);
            scales[r * (K / 32) + b] = (uint8_t)(X + 127);
            for (int i = 0; i < 32; ++i)
                codes[r * K + b * 32 + i] = (uint8_t)oracle_e4m3_encode(ldexp(v[i], -X));
        }
    return ORC_OK;
}

/* A row through MXFP8 and back: dst = dequantize(quantize(src)), in place
 * allowed. */
static void mx_qdq_row(int K, const double *src, double *dst)
{
    for (int b = 0; b < K / 32; ++b) {
        double amax = 0.0;
        for (int i = 0; i < 32; ++i)
            if (fabs(src[b * 32 + i]) > amax)
                amax = fabs(src[b * 32 + i]);
        const int X = oracle_mx_scale_exp(amax);
        for (int i = 0; i < 32; ++i)
            dst[b * 32 + i] = ldexp(oracle_e4m3_decode(oracle_e4m3_encode(
                                        ldexp(src[b * 32 + i], -X))), X);
    }
}

/* [MIX] "Sparse MoE Block": router_logits = gate(x), gate = Linear(d, E)
 * stored [E, d]; [DSK] adds the bias b[E]. Exact products, fp64 sums.
 * L64 [T,E] (may be NULL) receives the fp64 logits, L32 [T,E] (may be NULL)
 * the same values rounded once to fp32. */
int oracle_router_logits(int T, int d, int E, const uint16_t *x,
                         const uint16_t *wg, const float *bias,
                         double *L64, float *L32)
{
    if (T < 0 || d < 1 || E < 1 || !x || !wg)
        return ORC_EINVAL;
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        for (int e = 0; e < E; ++e) {
            double s = 0.0;
            for (int i = 0; i < d; ++i)
                s += bf16_to_double(x[(int64_t)t * d + i]) *
                     bf16_to_double(wg[(int64_t)e * d + i]);
            if (bias)
                s += (double)bias[e];
            if (L64)
                L64[(int64_t)t * E + e] = s;
            if (L32)
                L32[(int64_t)t * E + e] = (float)s;
        }
    }
    return ORC_OK;
}

/* [MIX] "Sparse MoE Block": softmax over all E, top-k, divide by the top-k
 * sum; readings R1 and R2. L [T,E] fp32 -> idx [T,k] (selection order),
 * w [T,k] fp64. A row holding a NaN, or whose maximum is not finite,
 * returns ORC_ENONFINITE. */
int oracle_route(int T, int E, int k, const float *L, int32_t *idx, double *w)
{
    if (T < 0 || E < 1 || k < 1 || k > E || !L || !idx || !w)
        return ORC_EINVAL;
    int rc = ORC_OK;
    double *p = (double *)malloc(sizeof(double) * (size_t)E);
    char *chosen = (char *)malloc((size_t)E);
    if (!p || !chosen) {
        free(p);
        free(chosen);
        return ORC_EINVAL;
    }
    for (int t = 0; t < T && rc == ORC_OK; ++t) {
        const float *l = L + (int64_t)t * E;
        /* softmax over all E, in fp64 */
        double M = -INFINITY;
        for (int e = 0; e < E; ++e) {
            if (isnan(l[e]))
                rc = ORC_ENONFINITE;
            if ((double)l[e] > M)
                M = (double)l[e];
        }
        if (rc != ORC_OK || !isfinite(M)) {
            rc = ORC_ENONFINITE;
            break;
        }
        double S = 0.0;
        for (int e = 0; e < E; ++e) {
            p[e] = exp((double)l[e] - M);
            S += p[e];
        }
        for (int e = 0; e < E; ++e)
            p[e] /= S;
        /* top-k: k rounds of "largest logit not yet taken", lowest index on ties */
        memset(chosen, 0, (size_t)E);
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (chosen[e])
                    continue;
                if (best < 0 || l[e] > l[best])
                    best = e;
            }
            chosen[best] = 1;
            idx[(int64_t)t * k + j] = best;
        }
        /* renormalise over the chosen k */
        double s = 0.0;
        for (int j = 0; j < k; ++j)
            s += p[idx[(int64_t)t * k + j]];
        for (int j = 0; j < k; ++j)
            w[(int64_t)t * k + j] = p[idx[(int64_t)t * k + j]] / s;
    }
    free(p);
    free(chosen);
    return rc;
}

/* Expert histogram, capacity, offsets and permutation: [CUR]'s counts and
 * offsets, [MIX]'s torch.where(selected_experts == e) row-major order, and
 * readings R3/R4 (R3b with slot_major = 1).
 *   counts[E]       routed assignments per expert (before capacity)
 *   offsets[E+1]    exclusive scan of the kept counts min(counts, C)
 *   slot_pos[T*k]   permuted row of (t, j), or -1 if dropped
 *   perm_token[T*k] token of each permuted row; rows >= n_kept are -1
 *   n_kept[1]       offsets[E]
 * Ids must lie in [0, E) and be distinct within a token (ORC_EBADEXPERT). */
int oracle_dispatch(int T, int E, int k, int C, int slot_major, const int32_t *idx,
                    int32_t *counts, int32_t *offsets, int32_t *slot_pos,
                    int32_t *perm_token, int32_t *n_kept)
{
    if (T < 0 || E < 1 || k < 1 || k > E || !idx || !counts || !offsets ||
        !slot_pos || !perm_token || !n_kept)
        return ORC_EINVAL;
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int32_t e = idx[(int64_t)t * k + j];
            if (e < 0 || e >= E)
                return ORC_EBADEXPERT;
            for (int jj = 0; jj < j; ++jj)
                if (idx[(int64_t)t * k + jj] == e)
                    return ORC_EBADEXPERT;
        }
    }
    const int64_t N = (int64_t)T * k;
    int32_t *rank = (int32_t *)malloc(sizeof(int32_t) * (size_t)(N > 0 ? N : 1));
    if (!rank)
        return ORC_EINVAL;
    for (int e = 0; e < E; ++e)
        counts[e] = 0;
    /* pass 1: each assignment's rank among the assignments to its expert that
     * come before it in the priority order */
    for (int64_t i = 0; i < N; ++i) {
        const int t = slot_major ? (int)(i % (T > 0 ? T : 1)) : (int)(i / k);
        const int j = slot_major ? (int)(i / (T > 0 ? T : 1)) : (int)(i % k);
        const int64_t a = (int64_t)t * k + j;
        const int32_t e = idx[a];
        rank[a] = counts[e];
        counts[e] += 1;
    }
    /* offsets: exclusive scan of kept counts */
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) {
        int32_t kept = counts[e];
        if (C > 0 && kept > C)
            kept = C;
        offsets[e + 1] = offsets[e] + kept;
    }
    *n_kept = offsets[E];
    /* pass 2: positions and the inverse map */
    for (int64_t r = 0; r < N; ++r)
        perm_token[r] = -1;
    for (int t = 0; t < T; ++t) {
        for (int j = 0; j < k; ++j) {
            int64_t a = (int64_t)t * k + j;
            int32_t e = idx[a];
            int keep = (C <= 0) || (rank[a] < C);
            if (keep) {
                slot_pos[a] = offsets[e] + rank[a];
                perm_token[slot_pos[a]] = t;
            } else {
                slot_pos[a] = -1;
            }
        }
    }
    free(rank);
    return ORC_OK;
}

/* Precision modes of the expert FFN (argument `h_bf16` of the entry points):
 *   0  pure fp64;
 *   1  h rounded once to bf16 (reading R6);
 *   2  MXFP8 (reading R7): x (by the caller), every weight row and h pass
 *      through MXFP8 along their contraction dimension; products and sums
 *      of the dequantized values in fp64. */
#define ORC_MODE_MXFP8 2

/* A weight row widened from bf16, through MXFP8 in mode 2. */
static void weight_row(int K, const uint16_t *src, int mode, double *dst)
{
    for (int i = 0; i < K; ++i)
        dst[i] = bf16_to_double(src[i]);
    if (mode == ORC_MODE_MXFP8)
        mx_qdq_row(K, dst, dst);
}

/* [MIX] "Expert FFN": y = w2(silu(w1 x) * w3 x); w1, w3 are [d_ff, d],
 * w2 is [d, d_ff] (nn.Linear [out, in]); readings R6/R7 for h. `wrow` is
 * scratch of max(d, d_ff) doubles. */
static void swiglu_ffn(int d, int d_ff, const double *xv, const uint16_t *w1,
                       const uint16_t *w3, const uint16_t *w2, int mode,
                       double *h, double *y, double *wrow)
{
    for (int c = 0; c < d_ff; ++c) {
        double g = 0.0, u = 0.0;
        weight_row(d, w1 + (int64_t)c * d, mode, wrow);
        for (int i = 0; i < d; ++i)
            g += wrow[i] * xv[i];
        weight_row(d, w3 + (int64_t)c * d, mode, wrow);
        for (int i = 0; i < d; ++i)
            u += wrow[i] * xv[i];
        double hv = g / (1.0 + exp(-g)) * u;   /* silu(g) = g * sigmoid(g) */
        h[c] = (mode == 1) ? oracle_round_bf16(hv) : hv;
    }
    if (mode == ORC_MODE_MXFP8)
        mx_qdq_row(d_ff, h, h);
    for (int r = 0; r < d; ++r) {
        double s = 0.0;
        weight_row(d_ff, w2 + (int64_t)r * d_ff, mode, wrow);
        for (int c = 0; c < d_ff; ++c)
            s += wrow[c] * h[c];
        y[r] = s;
    }
}

/* A token's input row, through MXFP8 in mode 2. */
static void input_row(int d, const uint16_t *x, int mode, double *xv)
{
    for (int i = 0; i < d; ++i)
        xv[i] = bf16_to_double(x[i]);
    if (mode == ORC_MODE_MXFP8)
        mx_qdq_row(d, xv, xv);
}

/* The layer output for a list of tokens, given the routing:
 * out[s, :] = sum over kept (t, j), in ascending expert order as [MIX]'s
 * expert loop visits them, of w[t, j] * FFN_{idx[t, j]}(x_t), plus the
 * shared expert FFN_s(x_t) ([DSK], reading R5) when d_ff_s > 0.
 * x [T,d]; W1, W3 [E,d_ff,d]; W2 [E,d,d_ff]; W1s, W3s [d_ff_s,d];
 * W2s [d,d_ff_s]; idx, slot_pos [T,k]; w [T,k] fp64;
 * tokens [n_tok] (each in [0,T)); out [n_tok, d] fp64. */
int oracle_moe_tokens(int T, int d, int d_ff, int E, int k, int d_ff_s,
                      const uint16_t *x, const uint16_t *W1, const uint16_t *W3,
                      const uint16_t *W2, const uint16_t *W1s,
                      const uint16_t *W3s, const uint16_t *W2s,
                      const int32_t *idx, const double *w,
                      const int32_t *slot_pos, int h_bf16, int n_tok,
                      const int32_t *tokens, double *out)
{
    if (T < 0 || d < 1 || d_ff < 1 || E < 1 || k < 1 || k > E || d_ff_s < 0 ||
        n_tok < 0 || !x || !W1 || !W3 || !W2 || !idx || !w || !slot_pos ||
        (n_tok > 0 && (!tokens || !out)))
        return ORC_EINVAL;
    if (d_ff_s > 0 && (!W1s || !W3s || !W2s))
        return ORC_EINVAL;
    for (int s = 0; s < n_tok; ++s)
        if (tokens[s] < 0 || tokens[s] >= T)
            return ORC_EINVAL;
    for (int s = 0; s < n_tok; ++s)
        for (int j = 0; j < k; ++j) {
            int32_t e = idx[(int64_t)tokens[s] * k + j];
            if (e < 0 || e >= E)
                return ORC_EBADEXPERT;
        }
    if (h_bf16 == ORC_MODE_MXFP8 && (d % 32 || d_ff % 32 || d_ff_s % 32))
        return ORC_EINVAL;
    const int hmax = d_ff > d_ff_s ? d_ff : d_ff_s;
    const int wmax = hmax > d ? hmax : d;
    int rc = ORC_OK;
#pragma omp parallel
    {
        double *xv = (double *)malloc(sizeof(double) * (size_t)d);
        double *h = (double *)malloc(sizeof(double) * (size_t)hmax);
        double *y = (double *)malloc(sizeof(double) * (size_t)d);
        double *wrow = (double *)malloc(sizeof(double) * (size_t)wmax);
        if (!xv || !h || !y || !wrow) {
#pragma omp atomic write
            rc = ORC_EINVAL;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int s = 0; s < n_tok; ++s) {
                const int t = tokens[s];
                double *o = out + (int64_t)s * d;
                input_row(d, x + (int64_t)t * d, h_bf16, xv);
                for (int i = 0; i < d; ++i)
                    o[i] = 0.0;
                /* routed experts, visited in ascending expert index */
                for (int e = 0; e < E; ++e) {
                    for (int j = 0; j < k; ++j) {
                        int64_t a = (int64_t)t * k + j;
                        if (idx[a] != e || slot_pos[a] < 0)
                            continue;
                        swiglu_ffn(d, d_ff, xv, W1 + (int64_t)e * d_ff * d,
                                   W3 + (int64_t)e * d_ff * d,
                                   W2 + (int64_t)e * d * d_ff, h_bf16, h, y, wrow);
                        for (int i = 0; i < d; ++i)
                            o[i] += w[a] * y[i];
                    }
                }
                /* shared expert, weight 1: shared_output + routed_output */
                if (d_ff_s > 0) {
                    swiglu_ffn(d, d_ff_s, xv, W1s, W3s, W2s, h_bf16, h, y, wrow);
                    for (int i = 0; i < d; ++i)
                        o[i] = y[i] + o[i];
                }
            }
        }
        free(xv);
        free(h);
        free(y);
        free(wrow);
    }
    return rc;
}

/* The expert FFN alone for a list of (token, expert) pairs, unweighted:
 * y[s, :] = FFN_{experts[s]}(x_{tokens[s]}). Used to check per-row expert
 * outputs (the permuted y of the unfused path). */
int oracle_expert_rows(int T, int d, int d_ff, int E, const uint16_t *x,
                       const uint16_t *W1, const uint16_t *W3,
                       const uint16_t *W2, int h_bf16, int n,
                       const int32_t *tokens, const int32_t *experts,
                       double *y_out)
{
    if (T < 0 || d < 1 || d_ff < 1 || E < 1 || n < 0 || !x || !W1 || !W3 ||
        !W2 || (n > 0 && (!tokens || !experts || !y_out)))
        return ORC_EINVAL;
    for (int s = 0; s < n; ++s) {
        if (tokens[s] < 0 || tokens[s] >= T)
            return ORC_EINVAL;
        if (experts[s] < 0 || experts[s] >= E)
            return ORC_EBADEXPERT;
    }
    if (h_bf16 == ORC_MODE_MXFP8 && (d % 32 || d_ff % 32))
        return ORC_EINVAL;
    int rc = ORC_OK;
#pragma omp parallel
    {
        double *xv = (double *)malloc(sizeof(double) * (size_t)d);
        double *h = (double *)malloc(sizeof(double) * (size_t)d_ff);
        double *wrow = (double *)malloc(sizeof(double) * (size_t)(d > d_ff ? d : d_ff));
        if (!xv || !h || !wrow) {
#pragma omp atomic write
            rc = ORC_EINVAL;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int s = 0; s < n; ++s) {
                const int t = tokens[s], e = experts[s];
                input_row(d, x + (int64_t)t * d, h_bf16, xv);
                swiglu_ffn(d, d_ff, xv, W1 + (int64_t)e * d_ff * d,
                           W3 + (int64_t)e * d_ff * d,
                           W2 + (int64_t)e * d * d_ff, h_bf16, h,
                           y_out + (int64_t)s * d, wrow);
            }
        }
        free(xv);
        free(h);
        free(wrow);
    }
    return rc;
}

/* [MIX] "Sparse MoE Block": the softmax over all E of one token's logits,
 * in fp64. S [T,E] receives the probabilities. */
int oracle_softmax_rows(int T, int E, const float *L, double *S)
{
    if (T < 0 || E < 1 || !L || !S)
        return ORC_EINVAL;
    for (int t = 0; t < T; ++t) {
        const float *l = L + (int64_t)t * E;
        double M = -INFINITY;
        for (int e = 0; e < E; ++e) {
            if (isnan(l[e]))
                return ORC_ENONFINITE;
            if ((double)l[e] > M)
                M = (double)l[e];
        }
        if (!isfinite(M))
            return ORC_ENONFINITE;
        double Z = 0.0;
        for (int e = 0; e < E; ++e)
            Z += exp((double)l[e] - M);
        for (int e = 0; e < E; ++e)
            S[(int64_t)t * E + e] = exp((double)l[e] - M) / Z;
    }
    return ORC_OK;
}

/* Expert-choice routing: "MoE Model Architectures", "Design Patterns",
 * "Pattern 3: Expert Choice Routing" (each expert selects its top tokens from
 * all tokens). Readings: the score of (t, e) is the softmax over experts
 * S[t, e] (given here in fp32, as both sides use it); expert e takes the
 * Ceff = min(C, T) tokens with the largest S[:, e], equal scores going to the
 * lower token index; its selected tokens are listed in ascending token order
 * with weight S[t, e]. tokens, w: [E, Ceff]; *ceff receives Ceff. */
int oracle_expert_choice(int T, int E, int C, const float *S, int32_t *tokens, double *w,
                         int32_t *ceff)
{
    if (T < 0 || E < 1 || C < 1 || !S || !tokens || !w || !ceff)
        return ORC_EINVAL;
    const int K = C < T ? C : T;
    *ceff = K;
    char *taken = (char *)malloc((size_t)(T > 0 ? T : 1));
    if (!taken)
        return ORC_EINVAL;
    for (int e = 0; e < E; ++e) {
        memset(taken, 0, (size_t)(T > 0 ? T : 1));
        /* K rounds of "largest score not yet taken", lowest token on ties */
        for (int i = 0; i < K; ++i) {
            int best = -1;
            for (int t = 0; t < T; ++t) {
                if (taken[t])
                    continue;
                const float v = S[(int64_t)t * E + e];
                if (isnan(v)) {
                    free(taken);
                    return ORC_ENONFINITE;
                }
                if (best < 0 || v > S[(int64_t)best * E + e])
                    best = t;
            }
            taken[best] = 1;
        }
        /* ascending token order */
        int n = 0;
        for (int t = 0; t < T; ++t)
            if (taken[t]) {
                tokens[(int64_t)e * K + n] = t;
                w[(int64_t)e * K + n] = (double)S[(int64_t)t * E + e];
                ++n;
            }
    }
    free(taken);
    return ORC_OK;
}

/* ---- Backward pass (reading R8): gradients of the fp64 layer (precision
 * mode 0) with the top-k selection, the capacity drops and the slot
 * positions held fixed (they are piecewise constant in the inputs). For a kept
 * assignment (t, j) to expert e with weight w = w[t, j] ([MIX]: softmax over
 * all E renormalised over the top-k) and dout row delta:
 *   g = W1_e x, u = W3_e x, s = silu(g), h = s * u, y = W2_e h
 *   dW2_e += w delta h^T;   dh = w W2_e^T delta
 *   du = dh * s;            dg = dh * u * silu'(g),
 *                           silu'(g) = sig(g) (1 + g (1 - sig(g)))
 *   dW1_e += dg x^T;  dW3_e += du x^T;  dx += W1_e^T dg + W3_e^T du
 *   G[t, j] = <delta, y>    (the gradient of the loss w.r.t. w[t, j])
 * A dropped assignment has G = 0. The shared expert ([DSK]) is the same with
 * weight 1 and no G. Router: w_j = exp(l_j) / sum_{i in top-k} exp(l_i), so
 *   dl[t, e_j] = w_j (G_j - sum_i w_i G_i) for the k chosen experts, 0 else;
 *   dWg += dl^T x;  dbias += sum_t dl;  dx += dl Wg.
 * Inputs as oracle_moe_tokens (bf16 patterns; wg [E, d]); dout [T, d] fp32.
 * Outputs (fp64, fully written): dx [T, d], dW1 / dW3 [E, d_ff, d],
 * dW2 [E, d, d_ff], dW1s / dW3s [d_ff_s, d], dW2s [d, d_ff_s] (when
 * d_ff_s > 0), dlogits [T, E], dWg [E, d], dbias [E], G [T, k].
 * Plain serial loops: meant for small shapes. */
int oracle_moe_backward(int T, int d, int d_ff, int E, int k, int d_ff_s,
                        const uint16_t *x, const uint16_t *W1, const uint16_t *W3,
                        const uint16_t *W2, const uint16_t *W1s, const uint16_t *W3s,
                        const uint16_t *W2s, const uint16_t *wg, const int32_t *idx,
                        const double *w, const int32_t *slot_pos, const float *dout,
                        double *dx, double *dW1, double *dW3, double *dW2, double *dW1s,
                        double *dW3s, double *dW2s, double *dlogits, double *dWg,
                        double *dbias, double *G)
{
    if (T < 0 || d < 1 || d_ff < 1 || E < 1 || k < 1 || k > E || d_ff_s < 0 || !x || !W1 ||
        !W3 || !W2 || !wg || !idx || !w || !slot_pos || !dout || !dx || !dW1 || !dW3 ||
        !dW2 || !dlogits || !dWg || !dbias || !G)
        return ORC_EINVAL;
    if (d_ff_s > 0 && (!W1s || !W3s || !W2s || !dW1s || !dW3s || !dW2s))
        return ORC_EINVAL;
    for (int64_t i = 0; i < (int64_t)T * d; ++i)
        dx[i] = 0.0;
    for (int64_t i = 0; i < (int64_t)E * d_ff * d; ++i)
        dW1[i] = dW3[i] = dW2[i] = 0.0;
    if (d_ff_s > 0)
        for (int64_t i = 0; i < (int64_t)d_ff_s * d; ++i)
            dW1s[i] = dW3s[i] = dW2s[i] = 0.0;
    for (int64_t i = 0; i < (int64_t)T * E; ++i)
        dlogits[i] = 0.0;
    for (int64_t i = 0; i < (int64_t)E * d; ++i)
        dWg[i] = 0.0;
    for (int e = 0; e < E; ++e)
        dbias[e] = 0.0;
    const int hmax = d_ff > d_ff_s ? d_ff : d_ff_s;
    double *xv = (double *)malloc(sizeof(double) * (size_t)d);
    double *dl = (double *)malloc(sizeof(double) * (size_t)d);
    double *gv = (double *)malloc(sizeof(double) * (size_t)hmax);
    double *uv = (double *)malloc(sizeof(double) * (size_t)hmax);
    double *hv = (double *)malloc(sizeof(double) * (size_t)hmax);
    double *dh = (double *)malloc(sizeof(double) * (size_t)hmax);
    if (!xv || !dl || !gv || !uv || !hv || !dh) {
        free(xv); free(dl); free(gv); free(uv); free(hv); free(dh);
        return ORC_EINVAL;
    }
    for (int t = 0; t < T; ++t) {
        for (int i = 0; i < d; ++i) {
            xv[i] = bf16_to_double(x[(int64_t)t * d + i]);
            dl[i] = (double)dout[(int64_t)t * d + i];
        }
        /* each kept slot, then the shared expert (src = k) */
        for (int j = 0; j <= k; ++j) {
            const int shared = (j == k);
            if (shared && d_ff_s == 0)
                break;
            int64_t a = (int64_t)t * k + j;
            if (!shared) {
                G[a] = 0.0;
                if (slot_pos[a] < 0)
                    continue;
            }
            const int e = shared ? 0 : idx[a];
            const int ff = shared ? d_ff_s : d_ff;
            const double wt = shared ? 1.0 : w[a];
            const uint16_t *w1 = shared ? W1s : W1 + (int64_t)e * d_ff * d;
            const uint16_t *w3 = shared ? W3s : W3 + (int64_t)e * d_ff * d;
            const uint16_t *w2 = shared ? W2s : W2 + (int64_t)e * d * d_ff;
            double *g1 = shared ? dW1s : dW1 + (int64_t)e * d_ff * d;
            double *g3 = shared ? dW3s : dW3 + (int64_t)e * d_ff * d;
            double *g2 = shared ? dW2s : dW2 + (int64_t)e * d * d_ff;
            for (int c = 0; c < ff; ++c) {
                double g = 0.0, u = 0.0;
                for (int i = 0; i < d; ++i) {
                    g += bf16_to_double(w1[(int64_t)c * d + i]) * xv[i];
                    u += bf16_to_double(w3[(int64_t)c * d + i]) * xv[i];
                }
                gv[c] = g;
                uv[c] = u;
                hv[c] = g / (1.0 + exp(-g)) * u;
            }
            /* y, G, dW2, dh */
            double Gtj = 0.0;
            for (int c = 0; c < ff; ++c)
                dh[c] = 0.0;
            for (int r = 0; r < d; ++r) {
                double y = 0.0;
                for (int c = 0; c < ff; ++c) {
                    const double w2rc = bf16_to_double(w2[(int64_t)r * ff + c]);
                    y += w2rc * hv[c];
                    g2[(int64_t)r * ff + c] += wt * dl[r] * hv[c];
                    dh[c] += wt * w2rc * dl[r];
                }
                Gtj += dl[r] * y;
            }
            if (!shared)
                G[a] = Gtj;
            /* SwiGLU backward, dW1, dW3, dx */
            for (int c = 0; c < ff; ++c) {
                const double sg = 1.0 / (1.0 + exp(-gv[c]));
                const double silu = gv[c] * sg;
                const double du = dh[c] * silu;
                const double dg = dh[c] * uv[c] * sg * (1.0 + gv[c] * (1.0 - sg));
                for (int i = 0; i < d; ++i) {
                    g1[(int64_t)c * d + i] += dg * xv[i];
                    g3[(int64_t)c * d + i] += du * xv[i];
                    dx[(int64_t)t * d + i] += bf16_to_double(w1[(int64_t)c * d + i]) * dg +
                                              bf16_to_double(w3[(int64_t)c * d + i]) * du;
                }
            }
        }
        /* router: renormalised softmax over the k chosen experts */
        double wG = 0.0;
        for (int j = 0; j < k; ++j)
            wG += w[(int64_t)t * k + j] * G[(int64_t)t * k + j];
        for (int j = 0; j < k; ++j) {
            const int64_t a = (int64_t)t * k + j;
            const int e = idx[a];
            const double g = w[a] * (G[a] - wG);
            dlogits[(int64_t)t * E + e] = g;
            dbias[e] += g;
            for (int i = 0; i < d; ++i) {
                const double wgi = bf16_to_double(wg[(int64_t)e * d + i]);
                dWg[(int64_t)e * d + i] += g * xv[i];
                dx[(int64_t)t * d + i] += g * wgi;
            }
        }
    }
    free(xv); free(dl); free(gv); free(uv); free(hv); free(dh);
    return ORC_OK;
}

/* Number of OpenMP threads a parallel region of this library uses. */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
