/*
 * moe_oracle.c -- plain, slow, fp64 CPU oracle of one DeepSeek-V3-style
 * mixture-of-experts feed-forward layer (forward pass).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the reference the CUDA library is
 * checked against.  Only the test-suite, the smoke check and the benchmark's
 * CPU-baseline leg may load it.  It shares no code, header, table or helper
 * with the CUDA path under mixture_experts_ffn_17_b200/csrc, and it never
 * calls into it.
 *
 * Every stored value (bf16, fp32, or FP8 e4m3 with a block scale) is first
 * decoded to fp64; all arithmetic after that is fp64 with no intermediate
 * rounding.  Loops are written in the order of the definitions; OpenMP only
 * splits independent tokens (or experts) across threads, it never reorders a
 * sum.
 *
 * Sources (web pages on DeepSeek-V3's MoE layer):
 *  - "DeepSeek-V3's mixture-of-experts architecture explained" (n4n.ai),
 *    section "The architecture in one diagram", simplified block pseudocode:
 *    gate = bias-free linear; top-k of the gate logits, then a softmax over
 *    the k selected values; output adds shared and routed parts.
 *  - "DeepSeek-V3.2-Exp / Mixture of experts / Shared expert" (atlas page),
 *    the five SwiGLU steps g=xW1, u=xW3, a=g*sigmoid(g), h=a*u, y=hW2, the
 *    per-instance parameter table (3 x 7168 x 2048 = 44,040,192), and the
 *    MoE forward block of its "Code" section: bincount of indices, a per-expert
 *    gather of the tokens that chose it in token order, y[idx] += expert(x)
 *    * weight in an fp32 accumulator, then y += shared_experts(x).
 *  - The group-limited sigmoid routing with a selection bias (config "group
 *    routing + FP8"): s = sigmoid(logit), sel = s + b, 8 contiguous groups of
 *    32, group score = sum of the group's top-2 sel, keep the top-4 groups,
 *    top-8 sel inside them, weights = s normalised to sum 1, times 2.5.  The
 *    pages only hint at this rule (Baidu page, "Hierarchical Dynamic
 *    Routing"; freedom251 page, "How V3 balances expert traffic").
 *
 * Readings where the pages are silent (all listed in the design notes):
 *  - ties in any top-k are broken toward the lowest index;
 *  - slots are returned in descending score order (torch.topk's default);
 *  - the softmax covers the k selected logits only;
 *  - the h -> x.dtype cast of the page's SwiGLU is not emulated (the oracle's
 *    x is fp64, so type_as(x) rounds nothing).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* Decoding stored formats to fp64.                                          */
/* ------------------------------------------------------------------------ */

/* bfloat16 is the upper half of an IEEE-754 binary32; widening is exact. */
static double bf16_to_f64(uint16_t h)
{
    uint32_t bits = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* OCP 8-bit floating point, E4M3 variant ("e4m3fn"): 1 sign bit, 4 exponent
 * bits with bias 7, 3 mantissa bits; exponent field 0 encodes subnormals
 * m/8 * 2^-6; there is no infinity and S.1111.111 is NaN.  Largest finite
 * magnitude is 1.75 * 2^8 = 448. */
static double e4m3_to_f64(uint8_t q)
{
    int sign = (q >> 7) & 1;
    int expo = (q >> 3) & 0xF;
    int mant = q & 0x7;
    double v;
    if (expo == 0xF && mant == 0x7)
        return NAN;
    if (expo == 0)
        v = ldexp((double)mant / 8.0, -6);
    else
        v = ldexp(1.0 + (double)mant / 8.0, expo - 7);
    return sign ? -v : v;
}

ORACLE_EXPORT void oracle_decode_bf16(int64_t n, const uint16_t *src, double *dst)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        dst[i] = bf16_to_f64(src[i]);
}

ORACLE_EXPORT void oracle_decode_f32(int64_t n, const float *src, double *dst)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i)
        dst[i] = (double)src[i];
}

ORACLE_EXPORT double oracle_e4m3_value(uint8_t q) { return e4m3_to_f64(q); }

/* Block-scaled FP8 weight matrix [rows, cols] (row-major e4m3 codes) with one
 * fp32 scale per (blk x blk) block, scales laid out [ceil(rows/blk),
 * ceil(cols/blk)] row-major.  Dequantised value = code * scale. */
ORACLE_EXPORT void oracle_decode_e4m3_blocks(int64_t rows, int64_t cols, int64_t blk,
                                             const uint8_t *q, const float *scale, double *dst)
{
    int64_t scols = (cols + blk - 1) / blk;
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t c = 0; c < cols; ++c)
            dst[r * cols + c] = e4m3_to_f64(q[r * cols + c]) * (double)scale[(r / blk) * scols + (c / blk)];
}

/* ------------------------------------------------------------------------ */
/* Router: gate linear (no bias) -> logits.                                  */
/* logits[t,e] = sum_j x[t,j] * Wg[e,j]   (x [T,d], Wg [E,d], row-major).     */
/* ------------------------------------------------------------------------ */
ORACLE_EXPORT void oracle_logits(int64_t T, int64_t d, int64_t E,
                                 const double *x, const double *Wg, double *logits)
{
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t)
        for (int64_t e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int64_t j = 0; j < d; ++j)
                acc += x[t * d + j] * Wg[e * d + j];
            logits[t * E + e] = acc;
        }
}

/* Key order used by every top-k below: larger score first; on equal score the
 * lower index first.  Returns nonzero when (va, ia) comes before (vb, ib). */
static int before(double va, int ia, double vb, int ib)
{
    return (va > vb) || (va == vb && ia < ib);
}

/* Sort the candidate list cand[0..n) by key (score desc, index asc) and write
 * the first m into out[] (m <= n).  Plain selection: m passes, each picks the
 * best not yet taken. */
static void select_top(const double *score, const int *cand, int n, int m, int *out, unsigned char *taken)
{
    for (int i = 0; i < n; ++i) taken[i] = 0;
    for (int s = 0; s < m; ++s) {
        int best = -1;
        for (int i = 0; i < n; ++i) {
            if (taken[i]) continue;
            if (best < 0 || before(score[cand[i]], cand[i], score[cand[best]], cand[best]))
                best = i;
        }
        taken[best] = 1;
        out[s] = cand[best];
    }
}

/* Page-1 routing: weights, indices = topk(logits, k); weights = softmax(weights).
 * idx[t, 0..k) in descending logit order; w = exp(l_j - l_0) / sum_i exp(l_i - l_0).
 * gaps[t, j] (j < k) = sorted_score[j] - sorted_score[j+1] over the k+1 best
 * experts (the margin that decides slot j); when k == E the last gap is +inf. */
ORACLE_EXPORT void oracle_route_topk_softmax(int64_t T, int E, int k, const double *logits,
                                             int32_t *idx, double *w, double *gaps)
{
    #pragma omp parallel
    {
        int *cand = (int *)malloc(sizeof(int) * E);
        int *top = (int *)malloc(sizeof(int) * (k + 1));
        unsigned char *taken = (unsigned char *)malloc(E);
        #pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            const double *l = logits + t * E;
            int m = (k < E) ? k + 1 : k;
            for (int e = 0; e < E; ++e) cand[e] = e;
            select_top(l, cand, E, m, top, taken);
            double den = 0.0;
            for (int j = 0; j < k; ++j) den += exp(l[top[j]] - l[top[0]]);
            for (int j = 0; j < k; ++j) {
                idx[t * k + j] = top[j];
                w[t * k + j] = exp(l[top[j]] - l[top[0]]) / den;
            }
            if (gaps) {
                for (int j = 0; j < k; ++j)
                    gaps[t * k + j] = (j + 1 < m) ? l[top[j]] - l[top[j + 1]] : INFINITY;
            }
        }
        free(cand); free(top); free(taken);
    }
}

/* Group-limited sigmoid routing with a selection bias.
 *   s = 1/(1+exp(-logit)); sel = s + bias
 *   expert e belongs to group e / (E/n_group) (contiguous blocks)
 *   group score = sum of the group's group_topn largest sel
 *   keep the topk_group best groups (score desc, group index asc)
 *   pick the k best sel among the kept groups' experts (sel desc, index asc)
 *   w_j = route_scale * s_j / sum_i s_i
 * gaps[t, j] = margin deciding slot j among the candidates (sel_j - sel_{j+1});
 * gscore_gap[t] = score of the last kept group minus the best dropped one
 * (+inf when every group is kept). */
ORACLE_EXPORT void oracle_route_sigmoid_group(int64_t T, int E, int k, int n_group, int topk_group,
                                              int group_topn, double route_scale,
                                              const double *logits, const double *bias,
                                              int32_t *idx, double *w, double *gaps, double *gscore_gap)
{
    int gsize = E / n_group;
    #pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * E);
        double *sel = (double *)malloc(sizeof(double) * E);
        double *gscore = (double *)malloc(sizeof(double) * n_group);
        int *cand = (int *)malloc(sizeof(int) * E);
        int *gl = (int *)malloc(sizeof(int) * n_group);
        int *gtop = (int *)malloc(sizeof(int) * n_group);
        int *inner = (int *)malloc(sizeof(int) * gsize);
        int *top = (int *)malloc(sizeof(int) * (k + 1));
        unsigned char *taken = (unsigned char *)malloc(E > n_group ? E : n_group);
        #pragma omp for schedule(static)
        for (int64_t t = 0; t < T; ++t) {
            const double *l = logits + t * E;
            for (int e = 0; e < E; ++e) {
                s[e] = 1.0 / (1.0 + exp(-l[e]));
                sel[e] = s[e] + (bias ? bias[e] : 0.0);
            }
            for (int g = 0; g < n_group; ++g) {
                for (int i = 0; i < gsize; ++i) cand[i] = g * gsize + i;
                select_top(sel, cand, gsize, group_topn, inner, taken);
                double acc = 0.0;
                for (int i = 0; i < group_topn; ++i) acc += sel[inner[i]];
                gscore[g] = acc;
            }
            int ng = (topk_group < n_group) ? topk_group + 1 : topk_group;
            for (int g = 0; g < n_group; ++g) gl[g] = g;
            select_top(gscore, gl, n_group, ng, gtop, taken);
            if (gscore_gap)
                gscore_gap[t] = (topk_group < n_group) ? gscore[gtop[topk_group - 1]] - gscore[gtop[topk_group]]
                                                       : INFINITY;
            /* candidates: experts of the kept groups, in index order */
            int nc = 0;
            for (int g = 0; g < n_group; ++g) {
                int kept = 0;
                for (int i = 0; i < topk_group; ++i) kept |= (gtop[i] == g);
                if (kept)
                    for (int i = 0; i < gsize; ++i) cand[nc++] = g * gsize + i;
            }
            int m = (k < nc) ? k + 1 : k;
            select_top(sel, cand, nc, m, top, taken);
            double den = 0.0;
            for (int j = 0; j < k; ++j) den += s[top[j]];
            for (int j = 0; j < k; ++j) {
                idx[t * k + j] = top[j];
                w[t * k + j] = route_scale * s[top[j]] / den;
            }
            if (gaps)
                for (int j = 0; j < k; ++j)
                    gaps[t * k + j] = (j + 1 < m) ? sel[top[j]] - sel[top[j + 1]] : INFINITY;
        }
        free(s); free(sel); free(gscore); free(cand); free(gl); free(gtop); free(inner); free(top); free(taken);
    }
}

/* Weights the page-1 rule gives to a caller-chosen index set (used when a
 * near-tie lets the device pick a different but equally valid set). */
ORACLE_EXPORT void oracle_weights_topk_softmax(int64_t T, int E, int k, const double *logits,
                                               const int32_t *idx, double *w)
{
    for (int64_t t = 0; t < T; ++t) {
        const double *l = logits + t * E;
        double lmax = l[idx[t * k]];
        for (int j = 1; j < k; ++j) if (l[idx[t * k + j]] > lmax) lmax = l[idx[t * k + j]];
        double den = 0.0;
        for (int j = 0; j < k; ++j) den += exp(l[idx[t * k + j]] - lmax);
        for (int j = 0; j < k; ++j) w[t * k + j] = exp(l[idx[t * k + j]] - lmax) / den;
    }
}

ORACLE_EXPORT void oracle_weights_sigmoid(int64_t T, int E, int k, double route_scale, const double *logits,
                                          const int32_t *idx, double *w)
{
    for (int64_t t = 0; t < T; ++t) {
        const double *l = logits + t * E;
        double den = 0.0;
        for (int j = 0; j < k; ++j) den += 1.0 / (1.0 + exp(-l[idx[t * k + j]]));
        for (int j = 0; j < k; ++j) w[t * k + j] = route_scale * (1.0 / (1.0 + exp(-l[idx[t * k + j]]))) / den;
    }
}

/* ------------------------------------------------------------------------ */
/* Dispatch: counts = bincount(indices, minlength=E); the tokens of expert e  */
/* are those with indices[t, j] == e, in ascending token order (the order of */
/* torch.where on a row-major [T, k] array).  The permuted order lists the   */
/* experts in ascending order; offsets is the exclusive prefix sum of counts; */
/* perm_token[r] is the token at permuted position r and row_of[t*k+j] the   */
/* permuted position of (t, j).  Returns 0, or -1 on an out-of-range index.  */
/* ------------------------------------------------------------------------ */
ORACLE_EXPORT int oracle_dispatch(int64_t T, int k, int E, const int32_t *idx,
                                  int32_t *counts, int32_t *offsets, int32_t *perm_token, int32_t *row_of)
{
    for (int e = 0; e < E; ++e) counts[e] = 0;
    for (int64_t i = 0; i < T * k; ++i) {
        if (idx[i] < 0 || idx[i] >= E) return -1;
        counts[idx[i]] += 1;
    }
    offsets[0] = 0;
    for (int e = 0; e < E; ++e) offsets[e + 1] = offsets[e] + counts[e];
    int64_t r = 0;
    for (int e = 0; e < E; ++e)
        for (int64_t t = 0; t < T; ++t)
            for (int j = 0; j < k; ++j)
                if (idx[t * k + j] == e) {
                    perm_token[r] = (int32_t)t;
                    row_of[t * k + j] = (int32_t)r;
                    ++r;
                }
    return 0;
}

/* ------------------------------------------------------------------------ */
/* SwiGLU expert on a batch of rows:                                          */
/*   g = x W1, u = x W3, a = g * sigmoid(g), h = a * u, o = h W2             */
/* x rows [n, d]; W1, W3 [d, I]; W2 [I, d] (math orientation, row-major).     */
/* ------------------------------------------------------------------------ */
ORACLE_EXPORT void oracle_swiglu_rows(int64_t n, int64_t d, int64_t I, const double *x,
                                      const double *W1, const double *W3, const double *W2, double *out)
{
    #pragma omp parallel
    {
        double *g = (double *)malloc(sizeof(double) * I);
        double *u = (double *)malloc(sizeof(double) * I);
        double *h = (double *)malloc(sizeof(double) * I);
        #pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < n; ++r) {
            const double *xr = x + r * d;
            for (int64_t i = 0; i < I; ++i) { g[i] = 0.0; u[i] = 0.0; }
            for (int64_t j = 0; j < d; ++j) {
                double xj = xr[j];
                const double *w1 = W1 + j * I, *w3 = W3 + j * I;
                for (int64_t i = 0; i < I; ++i) { g[i] += xj * w1[i]; u[i] += xj * w3[i]; }
            }
            for (int64_t i = 0; i < I; ++i) {
                double a = g[i] / (1.0 + exp(-g[i]));
                h[i] = a * u[i];
            }
            double *o = out + r * d;
            for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
            for (int64_t i = 0; i < I; ++i) {
                double hi = h[i];
                const double *w2 = W2 + i * d;
                for (int64_t c = 0; c < d; ++c) o[c] += hi * w2[c];
            }
        }
        free(g); free(u); free(h);
    }
}

/* ------------------------------------------------------------------------ */
/* Whole layer for sizes that fit in host memory (all weights fp64):          */
/*   y[t] = sum_j w[t,j] * expert_{idx[t,j]}(x[t]) + shared(x[t])             */
/* route: 0 = page-1 top-k then softmax, 1 = sigmoid group-limited.           */
/* W1, W3 [E, d, I]; W2 [E, I, d]; W1s, W3s [d, Is]; W2s [Is, d] (Is may be   */
/* 0: no shared expert).  Optional outputs idx, w, logits may be NULL.        */
/* When force_idx is non-NULL the routing uses those indices (weights from    */
/* the same rule) instead of selecting them.                                  */
/* ------------------------------------------------------------------------ */
ORACLE_EXPORT int oracle_moe_forward(int64_t T, int64_t d, int E, int k, int64_t I, int64_t Is,
                                     int route, int n_group, int topk_group, int group_topn, double route_scale,
                                     const double *x, const double *Wg, const double *bias,
                                     const double *W1, const double *W3, const double *W2,
                                     const double *W1s, const double *W3s, const double *W2s,
                                     const int32_t *force_idx,
                                     double *y, int32_t *idx_out, double *w_out, double *logits_out)
{
    double *logits = (double *)malloc(sizeof(double) * T * E);
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * T * k);
    double *w = (double *)malloc(sizeof(double) * T * k);
    if (!logits || !idx || !w) { free(logits); free(idx); free(w); return -1; }

    oracle_logits(T, d, E, x, Wg, logits);
    if (force_idx) {
        memcpy(idx, force_idx, sizeof(int32_t) * T * k);
        if (route == 0) oracle_weights_topk_softmax(T, E, k, logits, idx, w);
        else oracle_weights_sigmoid(T, E, k, route_scale, logits, idx, w);
    } else if (route == 0) {
        oracle_route_topk_softmax(T, E, k, logits, idx, w, NULL);
    } else {
        oracle_route_sigmoid_group(T, E, k, n_group, topk_group, group_topn, route_scale,
                                   logits, bias, idx, w, NULL, NULL);
    }

    for (int64_t i = 0; i < T * d; ++i) y[i] = 0.0;
    double *o = (double *)malloc(sizeof(double) * d);
    /* routed part: one token, one slot at a time */
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int e = idx[t * k + j];
            oracle_swiglu_rows(1, d, I, x + t * d, W1 + (int64_t)e * d * I, W3 + (int64_t)e * d * I,
                               W2 + (int64_t)e * I * d, o);
            for (int64_t c = 0; c < d; ++c) y[t * d + c] += w[t * k + j] * o[c];
        }
    /* shared expert on every token */
    if (Is > 0)
        for (int64_t t = 0; t < T; ++t) {
            oracle_swiglu_rows(1, d, Is, x + t * d, W1s, W3s, W2s, o);
            for (int64_t c = 0; c < d; ++c) y[t * d + c] += o[c];
        }
    free(o);

    if (idx_out) memcpy(idx_out, idx, sizeof(int32_t) * T * k);
    if (w_out) memcpy(w_out, w, sizeof(double) * T * k);
    if (logits_out) memcpy(logits_out, logits, sizeof(double) * T * E);
    free(logits); free(idx); free(w);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Combine step alone: y[t] = sum_j w[t,j] * Yp[row_of[t*k+j]] + Ys[t]        */
/* (the y[idx] += expert_out * weight accumulation of the atlas page's       */
/* "Code" section, MoE forward block, then y += shared).  Ys may be NULL.    */
/* Rows with row_of < 0 are skipped.                                          */
/* ------------------------------------------------------------------------ */
ORACLE_EXPORT void oracle_combine(int64_t T, int k, int64_t d, const double *Yp, const double *Ys,
                                  const int32_t *row_of, const double *w, double *y)
{
    #pragma omp parallel for schedule(static)
    for (int64_t t = 0; t < T; ++t) {
        double *yt = y + t * d;
        for (int64_t c = 0; c < d; ++c) yt[c] = 0.0;
        for (int j = 0; j < k; ++j) {
            int32_t r = row_of[t * k + j];
            if (r < 0) continue;
            for (int64_t c = 0; c < d; ++c) yt[c] += w[t * k + j] * Yp[(int64_t)r * d + c];
        }
        if (Ys)
            for (int64_t c = 0; c < d; ++c) yt[c] += Ys[t * d + c];
    }
}

/* ------------------------------------------------------------------------ */
/* Device-limited routing (n4n page, "Why 256 experts with top-8 routing?",   */
/* device-limited routing code): experts not on this device get a -inf mask   */
/* added to their logits before the top-k; then the page-1 rule.  allowed[e] */
/* is nonzero for the experts this device holds.                              */
/* ------------------------------------------------------------------------ */
ORACLE_EXPORT void oracle_route_topk_softmax_limited(int64_t T, int E, int k, const double *logits,
                                                     const uint8_t *allowed, int32_t *idx, double *w, double *gaps)
{
    double *masked = (double *)malloc(sizeof(double) * T * E);
    for (int64_t t = 0; t < T; ++t)
        for (int e = 0; e < E; ++e)
            masked[t * E + e] = allowed[e] ? logits[t * E + e] : -INFINITY;
    oracle_route_topk_softmax(T, E, k, masked, idx, w, gaps);
    free(masked);
}

/* ------------------------------------------------------------------------ */
/* Expert-utilisation monitor (n4n page, "Where the architecture struggles",  */
/* log_expert_utilization): utilisation = counts / sum(counts); an expert is  */
/* flagged +1 when its count exceeds 2x the mean count, -1 when it is below   */
/* 0.1x the mean, 0 otherwise.  With mean = total / E the two tests are the   */
/* integer comparisons count*E > 2*total and 10*count*E < total, decided      */
/* exactly.                                                                   */
/* ------------------------------------------------------------------------ */
ORACLE_EXPORT void oracle_expert_utilisation(int E, const int32_t *counts, double *util, int32_t *flag)
{
    int64_t total = 0;
    for (int e = 0; e < E; ++e) total += counts[e];
    for (int e = 0; e < E; ++e) {
        int64_t c = counts[e];
        util[e] = total > 0 ? (double)c / (double)total : 0.0;
        flag[e] = (c * E > 2 * total) ? 1 : ((10 * c * E < total) ? -1 : 0);
    }
}

/* ------------------------------------------------------------------------ */
/* One rank's share of the expert-parallel layer (atlas page, "Code"         */
/* section: the MoE constructor block gives rank r the experts                */
/* [r*E/size, (r+1)*E/size) and a shared-expert MLP whose W1/W3 are column-  */
/* parallel and whose W2 is row-parallel without an output reduction; the    */
/* MoE forward block adds the local experts' weighted outputs and the shared  */
/* MLP's output into y, then all-reduces y over the ranks).                   */
/*   W1l, W3l [El, d, I], W2l [El, I, d]: the rank's experts, slice 0 is     */
/*     expert e_lo;                                                          */
/*   W1sl, W3sl [d, Isl], W2sl [Isl, d]: the rank's hidden features of the   */
/*     shared expert (Isl may be 0);                                         */
/*   y[t] = sum_{j: e_lo <= idx[t,j] < e_lo+El} w[t,j] expert(x[t])           */
/*        + W2sl(silu(x[t] W1sl) * (x[t] W3sl)).                             */
/* Routing is over all E experts, as every rank routes every token.          */
/* ------------------------------------------------------------------------ */
ORACLE_EXPORT int oracle_moe_forward_ep_rank(int64_t T, int64_t d, int E, int k, int64_t I, int64_t Isl,
                                             int route, int n_group, int topk_group, int group_topn,
                                             double route_scale, const double *x, const double *Wg,
                                             const double *bias, int e_lo, int El, const double *W1l,
                                             const double *W3l, const double *W2l, const double *W1sl,
                                             const double *W3sl, const double *W2sl, double *y)
{
    double *logits = (double *)malloc(sizeof(double) * T * E);
    int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * T * k);
    double *w = (double *)malloc(sizeof(double) * T * k);
    double *o = (double *)malloc(sizeof(double) * d);
    if (!logits || !idx || !w || !o) { free(logits); free(idx); free(w); free(o); return -1; }

    oracle_logits(T, d, E, x, Wg, logits);
    if (route == 0)
        oracle_route_topk_softmax(T, E, k, logits, idx, w, NULL);
    else
        oracle_route_sigmoid_group(T, E, k, n_group, topk_group, group_topn, route_scale,
                                   logits, bias, idx, w, NULL, NULL);

    for (int64_t i = 0; i < T * d; ++i) y[i] = 0.0;
    for (int64_t t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            const int e = idx[t * k + j];
            if (e < e_lo || e >= e_lo + El) continue;  /* another rank's expert */
            const int64_t el = e - e_lo;
            const double wj = w[t * k + j];
            oracle_swiglu_rows(1, d, I, x + t * d, W1l + el * d * I, W3l + el * d * I, W2l + el * I * d, o);
            for (int64_t c = 0; c < d; ++c) y[t * d + c] += wj * o[c];
        }
    if (Isl > 0)
        for (int64_t t = 0; t < T; ++t) {
            oracle_swiglu_rows(1, d, Isl, x + t * d, W1sl, W3sl, W2sl, o);
            for (int64_t c = 0; c < d; ++c) y[t * d + c] += o[c];
        }
    free(logits); free(idx); free(w); free(o);
    return 0;
}
