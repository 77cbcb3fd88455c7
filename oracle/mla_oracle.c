/*
 * fp64 CPU oracle for MLA decoding over a paged latent KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load this file's library.  It shares no code with the
 * CUDA path, and the CUDA path never calls it.
 *
 * What it computes is the plain definition of the method, with no blocking,
 * splitting or online rescaling:
 *
 *   Attention(Q, K, V) = softmax(scale * Q K^T) V
 *     ("FlashMLA: Revolutionizing Efficient Decoding...", section 4.1.1,
 *      "Mathematical Formulation"; the printed formula is garbled, and the
 *      scale here is the runtime argument `scale`).
 *
 *   One latent row per cached token serves every query head, "somewhat like
 *   multi-query attention" ("OpenSourceWeek Day 1: FlashMLA", "Brief About
 *   Multi-head Latent Attention" and "How MLA Optimizes Memory Usage": only c_t
 *   is cached, and K and V are both derived from it).  Here K_t is the whole
 *   576-dim row and V_t is its first 512 dims.
 *
 *   The cache is paged with 64 tokens per page ("OpenSourceWeek Day 1:
 *   FlashMLA", "Key Highlights"; "FlashMLA: Revolutionizing...", section
 *   4.3.2): token t of sequence i is row t % 64 of physical page
 *   block_table[i][t / 64].
 *
 * Readings taken where the pages are silent:
 *   - causal with s_q > 1 is bottom-right aligned: query j of a sequence with
 *     L cached tokens sees tokens t <= L - s_q + j;
 *   - lse is the natural log of sum_t exp(s_t) over the visible tokens;
 *   - an empty visible set gives out = 0 and lse = -inf.
 *
 * Inputs are bf16 bit patterns; each is widened exactly to double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_PAGE 64
#define ORACLE_DQK 576
#define ORACLE_DV 512

static double bf16_to_double(uint16_t bits) {
    uint32_t w = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/* Address of the cached row of token t of sequence i. */
static const uint16_t *cache_row(const uint16_t *kcache, const int32_t *block_table,
                                 int64_t bt_stride, int i, int64_t t) {
    int64_t page = block_table[(int64_t)i * bt_stride + t / ORACLE_PAGE];
    return kcache + (page * ORACLE_PAGE + t % ORACLE_PAGE) * ORACLE_DQK;
}

/* Number of tokens query j of sequence i may attend to. */
static int64_t visible_tokens(int64_t L, int s_q, int j, int causal) {
    int64_t n = causal ? L - s_q + j + 1 : L;
    if (n < 0) n = 0;
    if (n > L) n = L;
    return n;
}

/*
 * One output row (sequence i, query position j, head h) over the visible tokens
 * that fall in [t_begin, t_end).  out_row: 512 doubles.  Returns lse.
 * `s` is scratch of at least L doubles.
 */
static double attend_range(const uint16_t *q, const uint16_t *kcache, const int32_t *block_table,
                           int64_t bt_stride, const int32_t *seqlens, int s_q, int h_q,
                           double scale, int causal, int i, int j, int h,
                           int64_t t_begin, int64_t t_end, double *s, double *out_row) {
    int64_t L = seqlens[i];
    int64_t n = visible_tokens(L, s_q, j, causal);
    if (t_begin < 0) t_begin = 0;
    if (t_end > n) t_end = n;
    const uint16_t *qrow = q + (((int64_t)i * s_q + j) * h_q + h) * ORACLE_DQK;
    double qd[ORACLE_DQK];
    for (int c = 0; c < ORACLE_DQK; ++c) qd[c] = bf16_to_double(qrow[c]);
    for (int c = 0; c < ORACLE_DV; ++c) out_row[c] = 0.0;
    if (t_end <= t_begin) return -INFINITY;

    /* logits s_t = scale * <q, K_t> over all 576 dims */
    double m = -INFINITY;
    for (int64_t t = t_begin; t < t_end; ++t) {
        const uint16_t *k = cache_row(kcache, block_table, bt_stride, i, t);
        double dot = 0.0;
        for (int c = 0; c < ORACLE_DQK; ++c) dot += qd[c] * bf16_to_double(k[c]);
        s[t] = scale * dot;
        if (s[t] > m) m = s[t];
    }
    /* two-pass softmax: weights exp(s_t - m), their sum l */
    double l = 0.0;
    for (int64_t t = t_begin; t < t_end; ++t) {
        double w = exp(s[t] - m);
        l += w;
        const uint16_t *v = cache_row(kcache, block_table, bt_stride, i, t);
        for (int c = 0; c < ORACLE_DV; ++c) out_row[c] += w * bf16_to_double(v[c]);
    }
    for (int c = 0; c < ORACLE_DV; ++c) out_row[c] /= l;
    return m + log(l);
}

/*
 * Full decode.
 *   out: [batch, s_q, h_q, 512] doubles; lse: [batch, h_q, s_q] doubles.
 *   nthreads <= 0 uses the OpenMP default.
 */
int mla_oracle_decode(const uint16_t *q, const uint16_t *kcache, const int32_t *block_table,
                      int64_t bt_stride, const int32_t *seqlens, int batch, int s_q, int h_q,
                      double scale, int causal, double *out, double *lse, int nthreads) {
    int64_t rows = (int64_t)batch * s_q * h_q;
    int64_t maxL = 0;
    for (int i = 0; i < batch; ++i)
        if (seqlens[i] > maxL) maxL = seqlens[i];
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    int err = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(maxL > 0 ? maxL : 1));
        if (!s) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < rows; ++r) {
                int h = (int)(r % h_q);
                int j = (int)((r / h_q) % s_q);
                int i = (int)(r / ((int64_t)h_q * s_q));
                double v = attend_range(q, kcache, block_table, bt_stride, seqlens, s_q, h_q,
                                        scale, causal, i, j, h, 0, seqlens[i], s,
                                        out + r * ORACLE_DV);
                lse[((int64_t)i * h_q + h) * s_q + j] = v;
            }
            free(s);
        }
    }
    return err;
}

/*
 * Selected rows only: rows (i, j, h, t_begin, t_end) in `sel` ([n_sel, 5] int32).
 * Each row attends over its visible tokens inside [t_begin, t_end); pass
 * t_begin = 0, t_end = seqlen for the ordinary result.  The output of a
 * sub-range is that range's own softmax (normalised over the range) and its lse.
 *   out: [n_sel, 512] doubles; lse: [n_sel] doubles.
 */
int mla_oracle_decode_rows(const uint16_t *q, const uint16_t *kcache, const int32_t *block_table,
                           int64_t bt_stride, const int32_t *seqlens, int batch, int s_q, int h_q,
                           double scale, int causal, const int32_t *sel, int64_t n_sel,
                           double *out, double *lse, int nthreads) {
    int64_t maxL = 0;
    for (int i = 0; i < batch; ++i)
        if (seqlens[i] > maxL) maxL = seqlens[i];
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#endif
    int err = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(maxL > 0 ? maxL : 1));
        if (!s) {
#pragma omp atomic write
            err = 1;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < n_sel; ++r) {
                int i = sel[5 * r], j = sel[5 * r + 1], h = sel[5 * r + 2];
                int64_t t0 = sel[5 * r + 3], t1 = sel[5 * r + 4];
                if (i < 0 || i >= batch || j < 0 || j >= s_q || h < 0 || h >= h_q) {
#pragma omp atomic write
                    err = 2;
                    continue;
                }
                lse[r] = attend_range(q, kcache, block_table, bt_stride, seqlens, s_q, h_q, scale,
                                      causal, i, j, h, t0, t1, s, out + r * ORACLE_DV);
            }
            free(s);
        }
    }
    return err;
}

/* Threads an OpenMP parallel region would use (1 without OpenMP). */
int mla_oracle_threads(void) {
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}
