/*
 * Longformer self-attention forward: the fp64 CPU oracle.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg do.  It shares no code, header, table or helper with the
 * CUDA library.
 *
 * It is the plain definition of the method, written out loop by loop, with no
 * tiling, fusion or reordering:
 *
 *   - Sliding window: each token looks at w/2 neighbours on each side.
 *     ("LongFormer: The Long-Document Transformer" notes, section
 *     "Sliding Window".)
 *   - Dilation: the window has gaps of size d between its taps, and the gap
 *     size is a per-head setting.  (Same notes, "Dilated Sliding Window".)
 *   - Causal use: an autoregressive model looks only to the left.  (Same notes,
 *     section on autoregressive language models.)
 *   - Global attention: a few preselected positions attend to every position,
 *     and every position attends to them; global rows use their own
 *     projections Qg, Kg, Vg.  (Same notes, "Global Attention".)
 *   - Scaled dot-product scores QK^T / sqrt(d_head) followed by a softmax.
 *     (Same notes, abstract: the scaled dot product.)
 *   - Global-index extraction by compaction of the global mask; local rows
 *     take the softmax over their window plus the global tokens; global rows
 *     take it over the whole sequence; rows masked out by the local mask are
 *     set to zero.  (FasterTransformer Longformer Encoder guide, section
 *     "Longformer Encoder compute flow".)
 *
 * Readings taken where the pages leave a step open (each also listed in the
 * design notes):
 *   R1 non-causal window offsets k in [-w/2, w/2] (w+1 taps incl. self);
 *      causal offsets k in [0, w-1] (w taps incl. self).
 *   R2 a global key that is also inside the window is counted once (key sets
 *      are sets).
 *   R3 local rows use K, V for the global-key columns too; global rows use
 *      Qg against Kg, Vg over every valid key.
 *   R4 dilation applies to window offsets only.
 *   R5 out-of-range taps are dropped.
 *   R6 a padded key (local mask 0) is never a key; a padded query row is 0,
 *      even when it is also marked global.
 *   R7 scale = 1/sqrt(d_head).
 *   R8 causal together with global tokens is rejected.
 *   R10 the compacted index list is padded with -1.
 *
 * Parity of every function here is pinned by the test suite against full
 * attention from torch (fp64), masked attention with an explicit mask,
 * residue decomposition of dilation, truncation of padding, hand-derived key
 * sets and closed-form softmax values.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define LFO_OK 0
#define LFO_BAD_ARG (-1)
#define LFO_UNSUPPORTED (-2)
#define LFO_NOMEM (-3)

/* Compaction of the global mask of each batch into ascending positions,
 * padded with -1, and the count per batch.  (FasterTransformer Longformer
 * Encoder guide, compute flow: global-index extraction.) */
int lfo_global_index(const uint8_t *global_mask, int B, int n,
                     int32_t *global_idx, int32_t *counts)
{
    if (B < 0 || n < 0 || !global_idx || !counts) return LFO_BAD_ARG;
    for (int b = 0; b < B; ++b) {
        int cnt = 0;
        for (int p = 0; p < n; ++p) {
            if (global_mask && global_mask[(size_t)b * n + p] != 0) {
                global_idx[(size_t)b * n + cnt] = p;
                cnt += 1;
            }
        }
        for (int p = cnt; p < n; ++p) global_idx[(size_t)b * n + p] = -1;
        counts[b] = cnt;
    }
    return LFO_OK;
}

static int is_valid_key(const uint8_t *local_mask_b, int j)
{
    return local_mask_b == NULL || local_mask_b[j] != 0;
}

/* Is key j one of the window taps of query i?  Window taps are
 * i + k*dil for k in [-w/2, w/2] (non-causal) or i - k*dil for k in [0, w-1]
 * (causal), before clipping to the sequence. */
static int in_window(int i, int j, int w, int dil, int causal)
{
    int diff = j - i;
    if (causal) {
        if (diff > 0) return 0;
        int back = -diff;
        if (back % dil != 0) return 0;
        return back / dil <= w - 1;
    }
    int a = diff < 0 ? -diff : diff;
    if (a % dil != 0) return 0;
    return a / dil <= w / 2;
}

/* Key set of a local (non-global, non-padded) query row i: the window taps
 * that fall inside [0, n), then every global token that is not already a
 * window tap, all restricted to valid (unpadded) keys.  Returns the count. */
static int local_key_set(int n, const uint8_t *local_mask_b,
                         const int32_t *gidx_b, int g,
                         int w, int dil, int causal, int i, int32_t *keys)
{
    int cnt = 0;
    if (causal) {
        for (int k = w - 1; k >= 0; --k) {
            long j = (long)i - (long)k * dil;
            if (j >= 0 && j < n && is_valid_key(local_mask_b, (int)j)) keys[cnt++] = (int32_t)j;
        }
    } else {
        for (int k = -(w / 2); k <= w / 2; ++k) {
            long j = (long)i + (long)k * dil;
            if (j >= 0 && j < n && is_valid_key(local_mask_b, (int)j)) keys[cnt++] = (int32_t)j;
        }
    }
    for (int t = 0; t < g; ++t) {
        int j = gidx_b[t];
        if (!is_valid_key(local_mask_b, j)) continue;
        if (in_window(i, j, w, dil, causal)) continue;
        keys[cnt++] = j;
    }
    return cnt;
}

/* Key set of a global query row: every valid position of the sequence. */
static int global_key_set(int n, const uint8_t *local_mask_b, int32_t *keys)
{
    int cnt = 0;
    for (int j = 0; j < n; ++j)
        if (is_valid_key(local_mask_b, j)) keys[cnt++] = j;
    return cnt;
}

/* Softmax over the scaled dot products of query row qrow with the listed key
 * rows of kmat, then the weighted sum of the matching rows of vmat.
 * Probabilities are written to probs when it is non-NULL. */
static void softmax_attend(const double *qrow, const double *kmat, const double *vmat,
                           int d, double scale, const int32_t *keys, int cnt,
                           double *scores, double *out_row, double *probs)
{
    double m = -INFINITY;
    for (int t = 0; t < cnt; ++t) {
        const double *krow = kmat + (size_t)keys[t] * d;
        double dot = 0.0;
        for (int x = 0; x < d; ++x) dot += qrow[x] * krow[x];
        scores[t] = scale * dot;
        if (scores[t] > m) m = scores[t];
    }
    double denom = 0.0;
    for (int t = 0; t < cnt; ++t) {
        scores[t] = exp(scores[t] - m);
        denom += scores[t];
    }
    for (int x = 0; x < d; ++x) out_row[x] = 0.0;
    for (int t = 0; t < cnt; ++t) {
        double p = scores[t] / denom;
        if (probs) probs[t] = p;
        const double *vrow = vmat + (size_t)keys[t] * d;
        for (int x = 0; x < d; ++x) out_row[x] += p * vrow[x];
    }
}

static int check_args(int B, int H, int n, int d, int window, const int32_t *dilation,
                      int causal, const uint8_t *global_mask)
{
    if (B < 0 || H < 0 || n < 0 || d < 1) return LFO_BAD_ARG;
    if (window < 1) return LFO_BAD_ARG;
    if (!causal && (window % 2) != 0) return LFO_BAD_ARG;
    if (dilation)
        for (int h = 0; h < H; ++h)
            if (dilation[h] < 1) return LFO_BAD_ARG;
    if (causal && global_mask) {
        /* R8: the pages never combine causal windows with global tokens. */
        size_t total = (size_t)B * n;
        for (size_t p = 0; p < total; ++p)
            if (global_mask[p]) return LFO_UNSUPPORTED;
    }
    return LFO_OK;
}

/*
 * Full forward for the query rows [row_begin, row_end) of the (b, h) pairs
 * [bh_begin, bh_end) (bh = b*H + h).  All tensors are [B, H, n, d] fp64,
 * row-major; masks are [B, n] bytes (NULL: all valid / no globals); dilation
 * is [H] (NULL: all 1).  Rows outside the requested ranges are not written.
 * nthreads <= 0 uses the OpenMP default.
 */
int lfo_forward(int B, int H, int n, int d,
                const double *q, const double *k, const double *v,
                const double *qg, const double *kg, const double *vg,
                const uint8_t *local_mask, const uint8_t *global_mask,
                int window, const int32_t *dilation, int causal,
                int bh_begin, int bh_end, int row_begin, int row_end,
                double *out, int nthreads)
{
    int rc = check_args(B, H, n, d, window, dilation, causal, global_mask);
    if (rc != LFO_OK) return rc;
    if (bh_begin < 0) bh_begin = 0;
    if (bh_end > B * H) bh_end = B * H;
    if (row_begin < 0) row_begin = 0;
    if (row_end > n) row_end = n;
    if (bh_begin >= bh_end || row_begin >= row_end) return LFO_OK;

    int32_t *gidx = (int32_t *)malloc(sizeof(int32_t) * ((size_t)B * n + 1));
    int32_t *cnts = (int32_t *)malloc(sizeof(int32_t) * ((size_t)B + 1));
    if (!gidx || !cnts) { free(gidx); free(cnts); return LFO_NOMEM; }
    lfo_global_index(global_mask, B, n, gidx, cnts);

    const double scale = 1.0 / sqrt((double)d);
    const int nrows = row_end - row_begin;
    const long total = (long)(bh_end - bh_begin) * nrows;
    int failed = 0;

#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif

#pragma omp parallel reduction(| : failed)
    {
        int32_t *keys = (int32_t *)malloc(sizeof(int32_t) * ((size_t)n + (size_t)window + 2));
        double *scores = (double *)malloc(sizeof(double) * ((size_t)n + (size_t)window + 2));
        if (!keys || !scores) {
            failed = 1;
        } else {
#pragma omp for schedule(dynamic, 64)
            for (long item = 0; item < total; ++item) {
                int bh = bh_begin + (int)(item / nrows);
                int i = row_begin + (int)(item % nrows);
                int b = bh / H, h = bh % H;
                int dil = dilation ? dilation[h] : 1;
                const uint8_t *lm_b = local_mask ? local_mask + (size_t)b * n : NULL;
                const uint8_t *gm_b = global_mask ? global_mask + (size_t)b * n : NULL;
                size_t base = (size_t)bh * n * d;
                double *orow = out + base + (size_t)i * d;

                if (!is_valid_key(lm_b, i)) {                 /* R6: padded row */
                    for (int x = 0; x < d; ++x) orow[x] = 0.0;
                    continue;
                }
                if (gm_b && gm_b[i] != 0) {                    /* global row */
                    int cnt = global_key_set(n, lm_b, keys);
                    softmax_attend(qg + base + (size_t)i * d, kg + base, vg + base, d, scale,
                                   keys, cnt, scores, orow, NULL);
                } else {                                       /* local row */
                    int cnt = local_key_set(n, lm_b, gidx + (size_t)b * n, cnts[b],
                                            window, dil, causal, i, keys);
                    softmax_attend(q + base + (size_t)i * d, k + base, v + base, d, scale,
                                   keys, cnt, scores, orow, NULL);
                }
            }
        }
        free(keys);
        free(scores);
    }
    free(gidx);
    free(cnts);
    return failed ? LFO_NOMEM : LFO_OK;
}

/*
 * The key set and softmax probabilities of one query row (b, h, i), for
 * tests: writes the keys (ascending window taps, then the extra global
 * tokens; or every valid key for a global row) and their probabilities, and
 * returns the count (0 for a padded row), or a negative error code.
 * keys and probs must hold n + window + 1 entries.
 */
int lfo_row_probs(int B, int H, int n, int d,
                  const double *q, const double *k,
                  const double *qg, const double *kg,
                  const uint8_t *local_mask, const uint8_t *global_mask,
                  int window, const int32_t *dilation, int causal,
                  int b, int h, int i, int32_t *keys, double *probs)
{
    int rc = check_args(B, H, n, d, window, dilation, causal, global_mask);
    if (rc != LFO_OK) return rc;
    if (b < 0 || b >= B || h < 0 || h >= H || i < 0 || i >= n) return LFO_BAD_ARG;
    const uint8_t *lm_b = local_mask ? local_mask + (size_t)b * n : NULL;
    const uint8_t *gm_b = global_mask ? global_mask + (size_t)b * n : NULL;
    if (!is_valid_key(lm_b, i)) return 0;

    int32_t *gidx = (int32_t *)malloc(sizeof(int32_t) * ((size_t)B * n + 1));
    int32_t *cnts = (int32_t *)malloc(sizeof(int32_t) * ((size_t)B + 1));
    double *scores = (double *)malloc(sizeof(double) * ((size_t)n + (size_t)window + 2));
    double *tmp = (double *)malloc(sizeof(double) * (size_t)d);
    if (!gidx || !cnts || !scores || !tmp) {
        free(gidx); free(cnts); free(scores); free(tmp);
        return LFO_NOMEM;
    }
    lfo_global_index(global_mask, B, n, gidx, cnts);
    size_t base = ((size_t)b * H + h) * n * d;
    int dil = dilation ? dilation[h] : 1;
    int cnt;
    /* The value rows do not affect the probabilities; the key rows stand in. */
    if (gm_b && gm_b[i] != 0) {
        cnt = global_key_set(n, lm_b, keys);
        softmax_attend(qg + base + (size_t)i * d, kg + base, kg + base, d,
                       1.0 / sqrt((double)d), keys, cnt, scores, tmp, probs);
    } else {
        cnt = local_key_set(n, lm_b, gidx + (size_t)b * n, cnts[b], window, dil, causal, i, keys);
        softmax_attend(q + base + (size_t)i * d, k + base, k + base, d,
                       1.0 / sqrt((double)d), keys, cnt, scores, tmp, probs);
    }
    free(gidx); free(cnts); free(scores); free(tmp);
    return cnt;
}

int lfo_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
