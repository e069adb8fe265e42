/*
 * oracle.c -- plain, slow, fp64 CPU oracle for lookahead importance scoring.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  The product path
 * (the CUDA library behind include/speckv.h) never calls it, and the two
 * share no code: this file includes nothing from the CUDA side.
 *
 * Source of every definition: "Draft-based Approximate Inference for LLMs"
 * (paper notes, ICLR 2026), section "关键设计" (Key design):
 *   SpecKV  -- for every attention head, the queries of the last n_window
 *              input tokens and of the n_lookahead draft tokens attend to
 *              the input keys; the cross-attention they give the remaining
 *              input keys estimates each KV pair's importance; the top-C_max
 *              KV pairs plus the window are kept.
 *   SpecPC  -- draft attention A[layer][head][query][key]; a large query
 *              window with weights that fall off with distance from the end,
 *              the first l_skip layers skipped, mean first, then max.
 * and section "损失函数 / 训练策略": SpecPC smooths with local pooling.
 *
 * Readings where the pages are silent (the kernels take the same ones):
 *   - the softmax of a query row runs over the input keys it can see
 *     causally (a window row at position p sees keys 0..p; a lookahead row
 *     sees every input key); lookahead keys are not input keys;
 *   - SpecKV scores only the prefix keys [0, n_pre), n_pre = n_in - n_window;
 *     the window is kept unconditionally;
 *   - the GQA group of KV head h is query heads h*g .. h*g+g-1, and their
 *     attention is summed; rows are summed without weights;
 *   - pooling is a stride-1 max (or, as the averaging variant, the mean)
 *     over the window [j-r, j+r] clipped to the row;
 *   - a SpecPC row of weight 0 contributes nothing;
 *   - ties in the selection go to the lower index; the output lists the
 *     selected indices in ascending order, then the window.
 *
 * Every floating-point step is done in double on the exact values decoded
 * from the bf16 inputs.  Nothing is blocked, fused or reordered beyond the
 * definitions below.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 bit pattern -> double (exact: bf16 is the top half of an fp32). */
static double bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double *decode_bf16(const uint16_t *bits, size_t n) {
    double *out = (double *)malloc((n > 0 ? n : 1) * sizeof(double));
    if (out)
        for (size_t t = 0; t < n; ++t) out[t] = bf16_to_double(bits[t]);
    return out;
}

/*
 * One causal softmax row over the first c keys, accumulated with weight w
 * into acc[0..c).  z_j = scale * <q, k_j>; p_j = exp(z_j - m) / sum exp(z - m).
 * Returns the row's log-sum-exp (natural log) for callers that want it.
 */
static double softmax_row_accumulate(const double *q, const double *k, int d, int c,
                                     double scale, double w, double *acc, double *z /*[c]*/) {
    double m = -INFINITY;
    for (int j = 0; j < c; ++j) {
        const double *kj = k + (size_t)j * d;
        double dot = 0.0;
        for (int t = 0; t < d; ++t) dot += q[t] * kj[t];
        z[j] = scale * dot;
        if (z[j] > m) m = z[j];
    }
    double Z = 0.0;
    for (int j = 0; j < c; ++j) Z += exp(z[j] - m);
    for (int j = 0; j < c; ++j) acc[j] += w * (exp(z[j] - m) / Z);
    return m + log(Z);
}

/*
 * SpecKV importance of one unit (one batch element, layer and KV head).
 *
 *   q    : [g][R][d], R = n_window + n_lookahead; rows 0..n_window-1 are
 *          the window queries (positions n_in-n_window+i), the rest are the
 *          lookahead (draft) queries (positions >= n_in).
 *   k    : [n_in][d].
 *   scores      : [n_pre] out, s[j] = sum over the g heads and R rows of p_ij.
 *   window_mass : [n_window] out (may be NULL), the same sum on window keys.
 *   lse         : [g*R] out (may be NULL), natural-log LSE of each row.
 * Returns 0, or -1 on bad arguments / allocation failure.
 */
int oracle_speckv_unit_f64(const double *q, const double *k, int g, int n_window, int n_lookahead,
                       int n_in, int d, double scale, double *scores, double *window_mass,
                       double *lse) {
    if (g < 1 || n_window < 0 || n_lookahead < 0 || n_window > n_in || d < 1) return -1;
    const int R = n_window + n_lookahead;
    const int n_pre = n_in - n_window;
    double *acc = (double *)calloc((size_t)(n_in > 0 ? n_in : 1), sizeof(double));
    double *z = (double *)malloc((size_t)(n_in > 0 ? n_in : 1) * sizeof(double));
    if (!acc || !z) { free(acc); free(z); return -1; }
    for (int h = 0; h < g; ++h) {
        for (int i = 0; i < R; ++i) {
            /* position of the query row, and how many input keys it sees */
            long pos = (i < n_window) ? (long)(n_in - n_window + i) : (long)n_in + (i - n_window);
            int c = (int)((pos < n_in - 1 ? pos : n_in - 1) + 1);
            const double *qi = q + ((size_t)h * R + i) * d;
            double l = c > 0 ? softmax_row_accumulate(qi, k, d, c, scale, 1.0, acc, z) : -INFINITY;
            if (lse) lse[h * R + i] = l;
        }
    }
    for (int j = 0; j < n_pre; ++j) scores[j] = acc[j];
    if (window_mass)
        for (int j = n_pre; j < n_in; ++j) window_mass[j - n_pre] = acc[j];
    free(acc);
    free(z);
    return 0;
}

/*
 * SpecPC importance for one batch element.
 *
 *   q : [L][Hq][W][d], the last W query positions of the draft; row i
 *       sits at position n_in + n_lookahead - 1 - W + i.
 *   k : [L][Hkv][n_in][d].
 *   w : [W] row weights (oldest row first).
 *   scores : [n_in] out.
 * For each query head qh, S_qh[j] = (1/(L-l_skip)) * sum_{l>=l_skip}
 * sum_i w_i p^{l,qh}_{ij} / sum_i w_i ("mean over queries and layers"),
 * then s[j] = max_qh S_qh[j] ("then max").
 */
int oracle_specpc_batch_f64(const double *q, const double *k, const double *w, int L, int l_skip,
                        int hq, int hkv, int W, int n_lookahead, int n_in, int d, double scale,
                        double *scores) {
    if (hkv < 1 || hq % hkv != 0 || l_skip < 0 || l_skip >= L || W < 1 || n_in < 1) return -1;
    if ((long)n_in + n_lookahead - 1 - W < 0) return -1;
    const int g = hq / hkv;
    double wsum = 0.0;
    for (int i = 0; i < W; ++i) wsum += w[i];
    double *acc = (double *)calloc((size_t)hq * n_in, sizeof(double));
    double *z = (double *)malloc((size_t)n_in * sizeof(double));
    if (!acc || !z) { free(acc); free(z); return -1; }
    for (int l = l_skip; l < L; ++l) {
        for (int qh = 0; qh < hq; ++qh) {
            const int h = qh / g;
            const double *kh = k + (((size_t)l * hkv + h) * n_in) * d;
            for (int i = 0; i < W; ++i) {
                long pos = (long)n_in + n_lookahead - 1 - W + i;
                int c = (int)((pos < n_in - 1 ? pos : n_in - 1) + 1);
                const double *qi = q + ((((size_t)l * hq + qh) * W) + i) * d;
                softmax_row_accumulate(qi, kh, d, c, scale, w[i], acc + (size_t)qh * n_in, z);
            }
        }
    }
    const double norm = wsum * (double)(L - l_skip);
    for (int j = 0; j < n_in; ++j) {
        double best = -INFINITY;
        for (int qh = 0; qh < hq; ++qh) {
            double s = acc[(size_t)qh * n_in + j] / norm;
            if (s > best) best = s;
        }
        scores[j] = best;
    }
    free(acc);
    free(z);
    return 0;
}

/* bf16 entry points: decode the exact input values, then run the fp64 definition. */
int oracle_speckv_unit(const uint16_t *q, const uint16_t *k, int g, int n_window, int n_lookahead,
                       int n_in, int d, double scale, double *scores, double *window_mass,
                       double *lse) {
    const int R = n_window + n_lookahead;
    double *qd = decode_bf16(q, (size_t)g * R * d);
    double *kd = decode_bf16(k, (size_t)n_in * d);
    int rc = (qd && kd) ? oracle_speckv_unit_f64(qd, kd, g, n_window, n_lookahead, n_in, d, scale,
                                                 scores, window_mass, lse)
                        : -1;
    free(qd);
    free(kd);
    return rc;
}

int oracle_specpc_batch(const uint16_t *q, const uint16_t *k, const double *w, int L, int l_skip,
                        int hq, int hkv, int W, int n_lookahead, int n_in, int d, double scale,
                        double *scores) {
    if (hkv < 1 || L < 1) return -1;
    double *qd = decode_bf16(q, (size_t)L * hq * W * d);
    double *kd = decode_bf16(k, (size_t)L * hkv * n_in * d);
    int rc = (qd && kd) ? oracle_specpc_batch_f64(qd, kd, w, L, l_skip, hq, hkv, W, n_lookahead,
                                                  n_in, d, scale, scores)
                        : -1;
    free(qd);
    free(kd);
    return rc;
}

/* 1-D max pooling, odd kernel, stride 1, output length n, clipped edges. */
int oracle_maxpool(const double *s, int n, int kernel, double *out) {
    if (kernel < 1 || (kernel & 1) == 0 || n < 0) return -1;
    const int r = kernel / 2;
    for (int j = 0; j < n; ++j) {
        int lo = j - r < 0 ? 0 : j - r;
        int hi = j + r > n - 1 ? n - 1 : j + r;
        double m = s[lo];
        for (int t = lo + 1; t <= hi; ++t)
            if (s[t] > m) m = s[t];
        out[j] = m;
    }
    return 0;
}

/*
 * 1-D average pooling, odd kernel, stride 1, output length n: the mean of the
 * scores inside the window clipped at the row's ends (the pages name local
 * pooling without its kind; this is the averaging reading of it).
 */
int oracle_avgpool(const double *s, int n, int kernel, double *out) {
    if (kernel < 1 || (kernel & 1) == 0 || n < 0) return -1;
    const int r = kernel / 2;
    for (int j = 0; j < n; ++j) {
        int lo = j - r < 0 ? 0 : j - r;
        int hi = j + r > n - 1 ? n - 1 : j + r;
        double sum = 0.0;
        for (int t = lo; t <= hi; ++t) sum += s[t];
        out[j] = sum / (double)(hi - lo + 1);
    }
    return 0;
}

typedef struct { double v; int j; } keyed_t;

/* larger value first; equal values: lower index first */
static int by_value_desc_index_asc(const void *a, const void *b) {
    const keyed_t *x = (const keyed_t *)a, *y = (const keyed_t *)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->j > y->j) - (x->j < y->j);
}

static int int_asc(const void *a, const void *b) {
    int x = *(const int *)a, y = *(const int *)b;
    return (x > y) - (x < y);
}

/*
 * Top-k of the pooled candidate scores plus the kept tail.
 * Writes min(k, n_cand) selected indices in ascending order, then the tail
 * n_cand .. n_cand+n_tail-1.  Returns the number of indices written, or -1.
 */
int oracle_topk_with_tail(const double *pooled, int n_cand, int k, int n_tail, int32_t *idx) {
    if (n_cand < 0 || k < 0 || n_tail < 0) return -1;
    const int c = k < n_cand ? k : n_cand;
    keyed_t *order = (keyed_t *)malloc((size_t)(n_cand > 0 ? n_cand : 1) * sizeof(keyed_t));
    int *sel = (int *)malloc((size_t)(c > 0 ? c : 1) * sizeof(int));
    if (!order || !sel) { free(order); free(sel); return -1; }
    for (int j = 0; j < n_cand; ++j) { order[j].v = pooled[j]; order[j].j = j; }
    qsort(order, (size_t)n_cand, sizeof(keyed_t), by_value_desc_index_asc);
    for (int t = 0; t < c; ++t) sel[t] = order[t].j;
    qsort(sel, (size_t)c, sizeof(int), int_asc);
    for (int t = 0; t < c; ++t) idx[t] = sel[t];
    for (int t = 0; t < n_tail; ++t) idx[c + t] = n_cand + t;
    free(order);
    free(sel);
    return c + n_tail;
}

/* Compaction: dst[t] = src[idx[t]] for rows of row_bytes bytes. */
int oracle_gather_rows(const uint8_t *src, int n_src, int row_bytes, const int32_t *idx, int n_idx,
                       uint8_t *dst) {
    for (int t = 0; t < n_idx; ++t) {
        if (idx[t] < 0 || idx[t] >= n_src) return -1;
        memcpy(dst + (size_t)t * row_bytes, src + (size_t)idx[t] * row_bytes, (size_t)row_bytes);
    }
    return 0;
}

/*
 * Decode attention over a compacted cache ("Draft-based Approximate Inference
 * for LLMs", paper notes, section 整体框架: the target model runs on the
 * compressed KV cache; section 关键设计, SpecKV: that cache holds the kept
 * KV pairs).  One query row of one head against n_kv rows of its KV head:
 *   z_t = scale * <q, k_t>,  p_t = exp(z_t - max z) / sum exp(z - max z),
 *   out = sum_t p_t v_t.
 * q [d], k [n_kv][d], v [n_kv][d] as bf16 bit patterns; out [d] in double.
 */
int oracle_decode_row(const uint16_t *q, const uint16_t *k, const uint16_t *v, int n_kv, int d, double scale,
                      double *out) {
    if (n_kv < 1 || d < 1) return -1;
    double *z = (double *)malloc((size_t)n_kv * sizeof(double));
    if (!z) return -1;
    double zmax = -INFINITY;
    for (int t = 0; t < n_kv; ++t) {
        double dot = 0.0;
        for (int c = 0; c < d; ++c) dot += bf16_to_double(q[c]) * bf16_to_double(k[(size_t)t * d + c]);
        z[t] = scale * dot;
        if (z[t] > zmax) zmax = z[t];
    }
    double den = 0.0;
    for (int t = 0; t < n_kv; ++t) {
        z[t] = exp(z[t] - zmax);
        den += z[t];
    }
    for (int c = 0; c < d; ++c) out[c] = 0.0;
    for (int t = 0; t < n_kv; ++t) {
        const double pt = z[t] / den;
        for (int c = 0; c < d; ++c) out[c] += pt * bf16_to_double(v[(size_t)t * d + c]);
    }
    free(z);
    return 0;
}

/*
 * Prefill attention of one query row ("Draft-based Approximate Inference for
 * LLMs", paper notes, section 关键设计, SpecKV: the input tokens and the
 * lookahead tokens go through the target model's prefill together; the
 * importance is read from the attention of the last n_window input rows and
 * the lookahead rows).  The key/value sequence holds the n_in input tokens
 * followed by the lookahead tokens; the row attends causally to its first c
 * keys:
 *   z_j = scale <q, k_j>  (j < c),   p = softmax(z),   out = sum_j p_j v_j,
 *   lse_in = log sum_{j < min(c, n_in)} exp(z_j)   (over the INPUT keys only:
 *            the normaliser the importance scores use).
 * q [d], k [c][d], v [c][d] as bf16 bit patterns (rows >= c are not read);
 * out [d] and *lse_in in double.
 */
int oracle_prefill_row(const uint16_t *q, const uint16_t *k, const uint16_t *v, int c, int n_in, int d,
                       double scale, double *out, double *lse_in) {
    if (c < 1 || n_in < 1 || d < 1) return -1;
    double *z = (double *)malloc((size_t)c * sizeof(double));
    if (!z) return -1;
    double zmax = -INFINITY;
    for (int j = 0; j < c; ++j) {
        double dot = 0.0;
        for (int t = 0; t < d; ++t) dot += bf16_to_double(q[t]) * bf16_to_double(k[(size_t)j * d + t]);
        z[j] = scale * dot;
        if (z[j] > zmax) zmax = z[j];
    }
    /* the input keys' log-sum-exp, max-subtracted on its own maximum */
    const int c_in = c < n_in ? c : n_in;
    double mi = -INFINITY;
    for (int j = 0; j < c_in; ++j)
        if (z[j] > mi) mi = z[j];
    double si = 0.0;
    for (int j = 0; j < c_in; ++j) si += exp(z[j] - mi);
    *lse_in = mi + log(si);
    double den = 0.0;
    for (int j = 0; j < c; ++j) {
        z[j] = exp(z[j] - zmax);
        den += z[j];
    }
    for (int t = 0; t < d; ++t) out[t] = 0.0;
    for (int j = 0; j < c; ++j) {
        const double pj = z[j] / den;
        for (int t = 0; t < d; ++t) out[t] += pj * bf16_to_double(v[(size_t)j * d + t]);
    }
    free(z);
    return 0;
}

/*
 * Vertical-Slash sparse attention of one query row ("Draft-based Approximate
 * Inference for LLMs", paper notes, section 损失函数 / 训练策略: SpecKV runs the
 * target prefill with Vertical-Slash sparse attention; the pattern is the one
 * of the cited sparse-attention work: a set V of key columns every row sees
 * and a set S of diagonals, i.e. offsets o = p - j).  The row at position p
 * attends to the keys j <= p with j in V, or p - j in S, or j = p (a token
 * always sees itself, so every softmax is defined):
 *   z_j = scale <q, k_j>,  out = sum_j softmax(z)_j v_j,  lse = log sum_j exp(z_j)
 * over those keys.  vmask[j] / smask[o] (0 or 1, n entries each) mark V and S.
 * q [d], k/v [n][d] as bf16 bit patterns; out [d], *lse in double.
 */
int oracle_vs_row(const uint16_t *q, const uint16_t *k, const uint16_t *v, const uint8_t *vmask,
                  const uint8_t *smask, int n, int p, int d, double scale, double *out, double *lse) {
    if (n < 1 || p < 0 || p >= n || d < 1) return -1;
    double *z = (double *)malloc((size_t)(p + 1) * sizeof(double));
    if (!z) return -1;
    double zmax = -INFINITY;
    for (int j = 0; j <= p; ++j) {
        z[j] = -INFINITY;
        if (!(j == p || vmask[j] || smask[p - j])) continue;
        double dot = 0.0;
        for (int t = 0; t < d; ++t) dot += bf16_to_double(q[t]) * bf16_to_double(k[(size_t)j * d + t]);
        z[j] = scale * dot;
        if (z[j] > zmax) zmax = z[j];
    }
    double den = 0.0;
    for (int j = 0; j <= p; ++j) {
        z[j] = (z[j] == -INFINITY) ? 0.0 : exp(z[j] - zmax);
        den += z[j];
    }
    *lse = zmax + log(den);
    for (int t = 0; t < d; ++t) out[t] = 0.0;
    for (int j = 0; j <= p; ++j) {
        if (z[j] == 0.0) continue;
        const double pj = z[j] / den;
        for (int t = 0; t < d; ++t) out[t] += pj * bf16_to_double(v[(size_t)j * d + t]);
    }
    free(z);
    return 0;
}
