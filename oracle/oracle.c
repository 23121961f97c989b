/*
 * Plain, slow CPU oracle for block-sparse long-context attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or helper with the
 * CUDA library: it is written from the method's definition alone.
 *
 * Sources (page title, section):
 *  [M14]  "LLM Inference Systems. Module 14: Sparse attention and long
 *         context" (hermes-agent.ru course) -- §14.1 long-context economics,
 *         §14.2 StreamingLLM and the attention sink, §14.3 MoBA block gating,
 *         Exercise 14.1 (block-sparse mask and attention with additive mask).
 *  [SIA]  "Sparse long-context inference with self-indexing attention"
 *         (sarnas.ru) -- "How much memory the KV cache takes", "Importance
 *         scores and block selection", "Sliding window".
 *  [SEM]  "Semantic blocks for sparse attention" (rit.work) -- "A block groups
 *         similar keys from different parts of the request".
 *  [HYB]  "Sparse attention in hybrid LLMs" (rit.work) -- "Which parts of the
 *         context each layer reads".
 *
 * Two arithmetics live here:
 *  - fp64 for everything that is compared with a tolerance (attention
 *    outputs, log-sum-exp, reference block scores);
 *  - fp32 in one fixed, documented order for the block scores and block
 *    centroids that DECIDE the selection, so that the selected block ids
 *    can be compared bit for bit.  The order is part of the specification:
 *      centroid  c[i] = (((0 + k_0[i]) + k_1[i]) + ... ) / (float)n
 *      score     s_h  = fma chain over i = 0..D-1: acc = fmaf(q_h[i], x[i], acc)
 *                s    = ((s_0 + s_1) + s_2) + ... + s_{G-1}, then + 0.0f
 *      Quest     x[i] = q_h[i] >= 0 ? max_i : min_i   (max(q*mn, q*mx) is the
 *                product with the bound on q's side; the fma rounds it once)
 *    Compile with -ffp-contract=off so that the compiler adds no fusion.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>
#include <stdlib.h>

/* ---- element access: KV caches arrive as fp32 or as raw bf16 bit patterns.
 * bf16 -> float is exact: the 16 bits are the high half of an IEEE single. */
enum { ORC_F32 = 0, ORC_BF16 = 1 };

static float elem_f(const void *base, int dtype, int64_t idx) {
    if (dtype == ORC_F32) return ((const float *)base)[idx];
    uint32_t u = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* [SIA] "How much memory the KV cache takes": per-token bytes are
 * 2 (K and V) x layers x kv_heads x head_dim x bytes per element. */
int64_t oracle_kv_bytes_per_token(int64_t layers, int64_t kv_heads,
                                  int64_t head_dim, int64_t elem_bytes) {
    return 2 * layers * kv_heads * head_dim * elem_bytes;
}

/* [M14] §14.3 and [SEM]: per-block mean-pooled key ("block centre").
 * K is one (batch, kv-head) segment, row r at K + r*ld, D columns.
 * Block b covers rows [beg[b], end[b]).  An empty block gets a zero centre. */
void oracle_block_centroid(const void *K, int dtype, int64_t ld, int D,
                           const int64_t *beg, const int64_t *end, int nblk,
                           float *C /* [nblk][D] */) {
    for (int b = 0; b < nblk; ++b) {
        int64_t n = end[b] - beg[b];
        for (int i = 0; i < D; ++i) {
            float acc = 0.0f;
            for (int64_t r = beg[b]; r < end[b]; ++r)
                acc = acc + elem_f(K, dtype, r * ld + i);
            C[(int64_t)b * D + i] = n > 0 ? acc / (float)n : 0.0f;
        }
    }
}

/* fp32 Euclidean norm in the fixed order: fma chain over i, then sqrtf. */
static float norm_f32(const float *x, int D) {
    float acc = 0.0f;
    for (int i = 0; i < D; ++i) acc = fmaf(x[i], x[i], acc);
    return sqrtf(acc);
}

/* [SEM] "A block groups similar keys...": keys are L2-normalised and grouped
 * by spherical k-means; a block's centre is the normalised mean of its
 * normalised keys.  Each key is divided by its own norm (a zero key stays
 * zero), the unit keys are averaged in row order, and the mean is divided by
 * its norm. */
void oracle_block_centroid_normalized(const void *K, int dtype, int64_t ld, int D,
                                      const int64_t *beg, const int64_t *end,
                                      int nblk, float *C /* [nblk][D] */) {
    float *key = (float *)malloc(sizeof(float) * (size_t)D);
    float *acc = (float *)malloc(sizeof(float) * (size_t)D);
    for (int b = 0; b < nblk; ++b) {
        int64_t n = end[b] - beg[b];
        for (int i = 0; i < D; ++i) acc[i] = 0.0f;
        for (int64_t r = beg[b]; r < end[b]; ++r) {
            for (int i = 0; i < D; ++i) key[i] = elem_f(K, dtype, r * ld + i);
            float nr = norm_f32(key, D);
            for (int i = 0; i < D; ++i)
                acc[i] = acc[i] + (nr > 0.0f ? key[i] / nr : 0.0f);
        }
        float *c = C + (int64_t)b * D;
        for (int i = 0; i < D; ++i) c[i] = n > 0 ? acc[i] / (float)n : 0.0f;
        float nc = norm_f32(c, D);
        for (int i = 0; i < D; ++i) c[i] = nc > 0.0f ? c[i] / nc : 0.0f;
    }
    free(key);
    free(acc);
}

/* Quest-style page bounds ([HYB] "Which parts of the context each layer
 * reads"): elementwise min and max of the page's keys.  min/max of stored
 * values are stored values, so the bounds are exact in the cache's dtype. */
void oracle_block_minmax(const void *K, int dtype, int64_t ld, int D,
                         const int64_t *beg, const int64_t *end, int nblk,
                         float *mn /* [nblk][D] */, float *mx /* [nblk][D] */) {
    for (int b = 0; b < nblk; ++b) {
        for (int i = 0; i < D; ++i) {
            float lo = INFINITY, hi = -INFINITY;
            for (int64_t r = beg[b]; r < end[b]; ++r) {
                float v = elem_f(K, dtype, r * ld + i);
                if (v < lo) lo = v;
                if (v > hi) hi = v;
            }
            if (end[b] <= beg[b]) lo = hi = 0.0f;
            mn[(int64_t)b * D + i] = lo;
            mx[(int64_t)b * D + i] = hi;
        }
    }
}

/* Block scores for one KV head's group of G query heads, in the fixed fp32
 * order (header comment) and, independently, in fp64 straight from the
 * formulas:
 *   centroid  s = sum_h q_h . c
 *   Quest     s = sum_h sum_i max(q_h[i]*mn[i], q_h[i]*mx[i])
 * kind 0/1 = centroid (X = C), kind 2 = Quest (X = mn, X2 = mx). */
void oracle_block_scores(const float *q /* [G][D] */, int G, int D, int kind,
                         const float *X, const float *X2, int nblk,
                         float *s32 /* [nblk] */, double *s64 /* [nblk] */) {
    for (int b = 0; b < nblk; ++b) {
        const float *x = X + (int64_t)b * D;
        const float *x2 = X2 ? X2 + (int64_t)b * D : NULL;
        float tot = 0.0f;
        double tot64 = 0.0;
        for (int h = 0; h < G; ++h) {
            const float *qh = q + (int64_t)h * D;
            float acc = 0.0f;
            for (int i = 0; i < D; ++i) {
                float xi = (kind == 2) ? (qh[i] >= 0.0f ? x2[i] : x[i]) : x[i];
                acc = fmaf(qh[i], xi, acc);
                if (kind == 2) {
                    double a = (double)qh[i] * (double)x[i];
                    double c = (double)qh[i] * (double)x2[i];
                    tot64 += a > c ? a : c;
                } else {
                    tot64 += (double)qh[i] * (double)x[i];
                }
            }
            tot = (h == 0) ? acc : tot + acc;
        }
        s32[b] = tot + 0.0f;
        s64[b] = tot64;
    }
}

/* [M14] Exercise 14.1 (attention with additive mask) restricted to a token
 * set: out_h = sum_j softmax_j(scale * q_h . k_j) v_j over the listed rows of
 * one segment, in fp64, with the maximum subtracted before exponentiation.
 * lse_h = log sum_j exp(scale * q_h . k_j).  A row list that is empty gives
 * out = 0 and lse = -inf. */
void oracle_attend_rows(const float *q /* [G][D] */, int G, int D,
                        const void *K, const void *V, int dtype, int64_t ld,
                        const int64_t *rows, int64_t nrows, double scale,
                        double *out /* [G][D] */, double *lse /* [G] */) {
    double *logit = (double *)malloc(sizeof(double) * (size_t)(nrows > 0 ? nrows : 1));
    for (int h = 0; h < G; ++h) {
        const float *qh = q + (int64_t)h * D;
        double *oh = out + (int64_t)h * D;
        for (int i = 0; i < D; ++i) oh[i] = 0.0;
        if (nrows == 0) { lse[h] = -INFINITY; continue; }
        double m = -INFINITY;
        for (int64_t j = 0; j < nrows; ++j) {
            int64_t r = rows[j];
            double dot = 0.0;
            for (int i = 0; i < D; ++i)
                dot += (double)qh[i] * (double)elem_f(K, dtype, r * ld + i);
            logit[j] = dot * scale;
            if (logit[j] > m) m = logit[j];
        }
        double den = 0.0;
        for (int64_t j = 0; j < nrows; ++j) {
            double w = exp(logit[j] - m);
            den += w;
            int64_t r = rows[j];
            for (int i = 0; i < D; ++i)
                oh[i] += w * (double)elem_f(V, dtype, r * ld + i);
        }
        for (int i = 0; i < D; ++i) oh[i] /= den;
        lse[h] = m + log(den);
    }
    free(logit);
}

/* [SEM] "A block groups similar keys from different parts of the request":
 * the blocks come from spherical k-means over the L2-normalised keys; a
 * block is one cluster, its keys stored together (sorted by cluster, then by
 * original position), its centre the normalised mean of its unit keys.
 *
 * The page gives no iteration count, start or tie rule; this is the reading
 * taken (plain Lloyd iterations on the unit sphere):
 *   u_r     = k_r / ||k_r|| (a zero key stays zero), as in the centres above
 *   c_j     = u_{init[j]} to start
 *   iters rounds: every key goes to the centre with the largest u_r . c_j
 *           (fp32 fma chain over i = 0..D-1; the lowest j on equal dots);
 *           between rounds each centre becomes the normalised mean of its
 *           keys' unit vectors summed in position order (the normalised
 *           centroid arithmetic above); an empty cluster keeps its centre.
 * So `iters` assignments and iters - 1 updates: the labels returned are
 * those of the last assignment against the centres returned.
 * offsets[j] .. offsets[j+1] are cluster j's rows in the block-ordered store;
 * order[i] is the original position of block-ordered row i. */
void oracle_spherical_kmeans(const void *K, int dtype, int64_t ld, int D, int64_t L, int k,
                             int iters, const int32_t *init, float *C /* [k][D] */,
                             int32_t *labels /* [L] */, int32_t *offsets /* [k+1] */,
                             int32_t *order /* [L] */) {
    float *U = (float *)malloc(sizeof(float) * (size_t)L * (size_t)D);
    float *key = (float *)malloc(sizeof(float) * (size_t)D);
    float *acc = (float *)malloc(sizeof(float) * (size_t)D);
    int64_t *cnt = (int64_t *)calloc((size_t)k, sizeof(int64_t));
    int64_t *fill = (int64_t *)calloc((size_t)k, sizeof(int64_t));
    for (int64_t r = 0; r < L; ++r) {
        for (int i = 0; i < D; ++i) key[i] = elem_f(K, dtype, r * ld + i);
        float nr = norm_f32(key, D);
        for (int i = 0; i < D; ++i) U[r * D + i] = nr > 0.0f ? key[i] / nr : 0.0f;
    }
    for (int j = 0; j < k; ++j)
        for (int i = 0; i < D; ++i) C[(int64_t)j * D + i] = U[(int64_t)init[j] * D + i];
    for (int it = 0; it < iters; ++it) {
        /* assignment */
        for (int64_t r = 0; r < L; ++r) {
            float best = -INFINITY;
            int lab = 0;
            for (int j = 0; j < k; ++j) {
                float dot = 0.0f;
                for (int i = 0; i < D; ++i) dot = fmaf(U[r * D + i], C[(int64_t)j * D + i], dot);
                if (dot > best) { best = dot; lab = j; }
            }
            labels[r] = lab;
        }
        if (it == iters - 1) break;
        /* update: clusters summed over their keys in position order */
        for (int j = 0; j < k; ++j) {
            int64_t n = 0;
            for (int i = 0; i < D; ++i) acc[i] = 0.0f;
            for (int64_t r = 0; r < L; ++r) {
                if (labels[r] != j) continue;
                ++n;
                for (int i = 0; i < D; ++i) acc[i] = acc[i] + U[r * D + i];
            }
            if (n == 0) continue;   /* an empty cluster keeps its centre */
            float *c = C + (int64_t)j * D;
            for (int i = 0; i < D; ++i) c[i] = acc[i] / (float)n;
            float nc = norm_f32(c, D);
            for (int i = 0; i < D; ++i) c[i] = nc > 0.0f ? c[i] / nc : 0.0f;
        }
    }
    /* block-ordered store: clusters in index order, positions ascending */
    for (int64_t r = 0; r < L; ++r) ++cnt[labels[r]];
    offsets[0] = 0;
    for (int j = 0; j < k; ++j) offsets[j + 1] = offsets[j] + (int32_t)cnt[j];
    for (int64_t r = 0; r < L; ++r) {
        const int j = labels[r];
        order[offsets[j] + fill[j]++] = (int32_t)r;
    }
    free(U);
    free(key);
    free(acc);
    free(cnt);
    free(fill);
}

/* The assignment alone, for sampled keys against given centres (the same
 * arithmetic as above): labels[s] = argmax_j u_{rows[s]} . c_j. */
void oracle_kmeans_assign(const void *K, int dtype, int64_t ld, int D, const int64_t *rows,
                          int64_t n, const float *C, int k, int32_t *labels) {
    float *key = (float *)malloc(sizeof(float) * (size_t)D);
    for (int64_t s = 0; s < n; ++s) {
        const int64_t r = rows[s];
        for (int i = 0; i < D; ++i) key[i] = elem_f(K, dtype, r * ld + i);
        float nr = norm_f32(key, D);
        for (int i = 0; i < D; ++i) key[i] = nr > 0.0f ? key[i] / nr : 0.0f;
        float best = -INFINITY;
        int lab = 0;
        for (int j = 0; j < k; ++j) {
            float dot = 0.0f;
            for (int i = 0; i < D; ++i) dot = fmaf(key[i], C[(int64_t)j * D + i], dot);
            if (dot > best) { best = dot; lab = j; }
        }
        labels[s] = lab;
    }
    free(key);
}
