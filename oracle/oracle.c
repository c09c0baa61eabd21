/*
 * oracle.c -- plain fp64 CPU oracle for varlen grouped-query attention
 * (decode and short-query regime, packed THD layout, tail-aligned causal).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously correct
 * definition that the CUDA path is checked against.  Only the tests, the
 * package smoke check and the CPU-baseline leg of the benchmark may load it.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * What it computes (the plain definition that split-KV flash-decoding reaches
 * up to floating-point rounding order):
 *
 *   For every sequence b, query token qi < Lq_b and query head h:
 *     hk  = h / G                       (G = Hq / Hkv; contiguous head groups)
 *     n   = clamp(Lk_b - Lq_b + qi + 1, 0, Lk_b)   visible keys (tail-aligned
 *           causal; equal to Lk_b when Lq_b = 1)
 *     s_j = scale * sum_d q[cu_q[b]+qi, h, d] * k[cu_k[b]+j, hk, d],  j < n
 *     m   = max_j s_j,   l = sum_j exp(s_j - m)
 *     out = sum_j exp(s_j - m) * v[cu_k[b]+j, hk, :] / l
 *     lse = m + ln(l)                   (natural log, scaled scores)
 *   n = 0 gives out = 0 and lse = -inf.  Rows outside cu_q are not touched.
 *
 * Sources for each part:
 *  - lengths read from cumulative offsets, seqlens = cu[1:B+1] - cu[:B], with
 *    cu buffers allowed to be longer than B+1: TransformerEngine PR #24
 *    "Build the attention padding mask without host syncs", sections
 *    Description and Changes.
 *  - per-KV-head loop with the G query heads of a group sharing one K/V head:
 *    kernbench2 docs/adr-proposed commit log, the GQA entry ("G folded into
 *    matmul M dim").
 *  - (O, m, l) partials and their log-sum-exp merge: AstrAI commit log for
 *    csrc/kernels/gqa_decode_attn.cu (split-KV commit) and the magik.net post
 *    "Wiring Split-K Dispatch into a Custom CUDA Attention Kernel", section
 *    "The Message: A Read That Reveals the Architecture".
 *  - the plain readings where the pages are silent (head mapping, LSE base,
 *    causal alignment, zero-length output) are listed in the design notes.
 *
 * Inputs are bf16 bit patterns (uint16); each is widened exactly to double.
 * All arithmetic is fp64 with plain loops: no blocking, no reordering.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* exact widening of a bf16 bit pattern (the upper half of an IEEE fp32) */
static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t w = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

/* number of keys query qi of a sequence may see (tail-aligned causal) */
static int64_t visible_keys(int64_t Lq, int64_t Lk, int64_t qi, int causal)
{
    if (!causal)
        return Lk;
    int64_t n = Lk - Lq + qi + 1;
    if (n < 0)
        n = 0;
    if (n > Lk)
        n = Lk;
    return n;
}

/*
 * One output row: (b, qi, h).  Writes out_row[D] and *lse_row.  When p_out is
 * not NULL it receives the n softmax weights exp(s_j - m) / l.
 * Scores are kept in a caller-provided buffer s[n] so that the max, the sum
 * and the weighted sum are three separate plain passes.
 */
static void attend_row(int D, int Hq, int Hkv, double scale, int causal,
                       const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       int64_t q_tok, int64_t k_tok0, int64_t Lq, int64_t Lk,
                       int64_t qi, int h, double *s, double *out_row,
                       double *lse_row, double *p_out)
{
    const int G = Hq / Hkv;
    const int hk = h / G;
    const int64_t n = visible_keys(Lq, Lk, qi, causal);

    for (int d = 0; d < D; ++d)
        out_row[d] = 0.0;
    if (n == 0) {
        *lse_row = -INFINITY;
        return;
    }

    const uint16_t *qrow = q + (q_tok * Hq + h) * (int64_t)D;
    for (int64_t j = 0; j < n; ++j) {
        const uint16_t *krow = k + ((k_tok0 + j) * Hkv + hk) * (int64_t)D;
        double acc = 0.0;
        for (int d = 0; d < D; ++d)
            acc += bf16_bits_to_double(qrow[d]) * bf16_bits_to_double(krow[d]);
        s[j] = scale * acc;
    }

    double m = s[0];
    for (int64_t j = 1; j < n; ++j)
        if (s[j] > m)
            m = s[j];

    double l = 0.0;
    for (int64_t j = 0; j < n; ++j)
        l += exp(s[j] - m);

    for (int64_t j = 0; j < n; ++j) {
        const double w = exp(s[j] - m);
        const uint16_t *vrow = v + ((k_tok0 + j) * Hkv + hk) * (int64_t)D;
        for (int d = 0; d < D; ++d)
            out_row[d] += w * bf16_bits_to_double(vrow[d]);
        if (p_out)
            p_out[j] = w / l;
    }
    for (int d = 0; d < D; ++d)
        out_row[d] /= l;
    *lse_row = m + log(l);
}

static int check_shapes(int B, int Hq, int Hkv, int D, const int32_t *cu_q,
                        const int32_t *cu_k)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || Hq % Hkv != 0)
        return -1;
    for (int b = 0; b < B; ++b) {
        if (cu_q[b + 1] < cu_q[b] || cu_k[b + 1] < cu_k[b])
            return -2;
        if (cu_q[b] < 0 || cu_k[b] < 0)
            return -2;
    }
    return 0;
}

/*
 * Whole batch.  cu_q / cu_k hold at least B+1 entries; entries past B+1 are
 * never read.  out is [T_q, Hq, D] and lse is [T_q, Hq] (token-major, like the
 * packed query); the caller pre-fills them, and rows outside cu_q keep that
 * content.  Returns 0, or a negative code for invalid shapes or decreasing
 * offsets (then nothing is written).
 */
int oracle_attention(int B, int Hq, int Hkv, int D, double scale, int causal,
                     const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     const int32_t *cu_q, const int32_t *cu_k, double *out,
                     double *lse)
{
    int rc = check_shapes(B, Hq, Hkv, D, cu_q, cu_k);
    if (rc)
        return rc;

    int64_t maxLk = 0;
    for (int b = 0; b < B; ++b)
        if (cu_k[b + 1] - cu_k[b] > maxLk)
            maxLk = cu_k[b + 1] - cu_k[b];

    /* enumerate the rows (b, qi, h) so that one parallel loop covers them */
    int64_t nrows = 0;
    for (int b = 0; b < B; ++b)
        nrows += (int64_t)(cu_q[b + 1] - cu_q[b]) * Hq;

    int failed = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(maxLk > 0 ? maxLk : 1));
        if (!s) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < nrows; ++r) {
            if (!s)
                continue;
            /* r -> (b, qi, h): walk the sequences (plain, not fast) */
            int64_t rem = r;
            int b = 0;
            while (rem >= (int64_t)(cu_q[b + 1] - cu_q[b]) * Hq) {
                rem -= (int64_t)(cu_q[b + 1] - cu_q[b]) * Hq;
                ++b;
            }
            const int64_t qi = rem / Hq;
            const int h = (int)(rem % Hq);
            const int64_t Lq = cu_q[b + 1] - cu_q[b];
            const int64_t Lk = cu_k[b + 1] - cu_k[b];
            const int64_t tok = cu_q[b] + qi;
            attend_row(D, Hq, Hkv, scale, causal, q, k, v, tok, cu_k[b], Lq, Lk,
                       qi, h, s, out + (tok * Hq + h) * (int64_t)D,
                       lse + tok * Hq + h, NULL);
        }
        free(s);
    }
    return failed ? -3 : 0;
}

/*
 * Selected rows only, for checks at sizes where the whole batch is too slow.
 * rows[3*i .. 3*i+2] = (b, qi, h).  out_rows is [nsel, D], lse_rows [nsel].
 * A row with qi >= Lq_b is rejected (-4).
 */
int oracle_attention_rows(int B, int Hq, int Hkv, int D, double scale,
                          int causal, const uint16_t *q, const uint16_t *k,
                          const uint16_t *v, const int32_t *cu_q,
                          const int32_t *cu_k, int64_t nsel, const int64_t *rows,
                          double *out_rows, double *lse_rows)
{
    int rc = check_shapes(B, Hq, Hkv, D, cu_q, cu_k);
    if (rc)
        return rc;
    for (int64_t i = 0; i < nsel; ++i) {
        const int64_t b = rows[3 * i], qi = rows[3 * i + 1], h = rows[3 * i + 2];
        if (b < 0 || b >= B || h < 0 || h >= Hq || qi < 0 ||
            qi >= cu_q[b + 1] - cu_q[b])
            return -4;
    }
    int failed = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nsel; ++i) {
        const int64_t b = rows[3 * i], qi = rows[3 * i + 1];
        const int h = (int)rows[3 * i + 2];
        const int64_t Lq = cu_q[b + 1] - cu_q[b];
        const int64_t Lk = cu_k[b + 1] - cu_k[b];
        double *s = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
        if (!s) {
#pragma omp atomic write
            failed = 1;
            continue;
        }
        attend_row(D, Hq, Hkv, scale, causal, q, k, v, cu_q[b] + qi, cu_k[b], Lq,
                   Lk, qi, h, s, out_rows + i * (int64_t)D, lse_rows + i, NULL);
        free(s);
    }
    return failed ? -3 : 0;
}

/*
 * Softmax weights of one row (b, qi, h): p[0 .. n) with n the visible count.
 * Returns n (>= 0) or a negative code.  p must hold Lk_b entries.
 */
int64_t oracle_row_weights(int B, int Hq, int Hkv, int D, double scale,
                           int causal, const uint16_t *q, const uint16_t *k,
                           const uint16_t *v, const int32_t *cu_q,
                           const int32_t *cu_k, int64_t b, int64_t qi, int h,
                           double *p, double *out_row, double *lse_row)
{
    int rc = check_shapes(B, Hq, Hkv, D, cu_q, cu_k);
    if (rc)
        return rc;
    if (b < 0 || b >= B || h < 0 || h >= Hq || qi < 0 ||
        qi >= cu_q[b + 1] - cu_q[b])
        return -4;
    const int64_t Lq = cu_q[b + 1] - cu_q[b];
    const int64_t Lk = cu_k[b + 1] - cu_k[b];
    double *s = (double *)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
    if (!s)
        return -3;
    attend_row(D, Hq, Hkv, scale, causal, q, k, v, cu_q[b] + qi, cu_k[b], Lq, Lk,
               qi, h, s, out_row, lse_row, p);
    free(s);
    return visible_keys(Lq, Lk, qi, causal);
}

/*
 * Partial state of one query row over the key range [j0, j1) of one KV head:
 *   m = max s_j,  l = sum exp(s_j - m),  o = sum exp(s_j - m) v_j  (not
 *   divided by l).  An empty range gives m = -inf, l = 0, o = 0.
 * qrow: D bf16 values.  krows / vrows: row j at krows + j * ld (elements).
 * This is the (O, m, l) triple a split-KV block emits, in natural-log units.
 */
void oracle_partial(int D, double scale, const uint16_t *qrow,
                    const uint16_t *krows, const uint16_t *vrows, int64_t ld,
                    int64_t j0, int64_t j1, double *o, double *m_out,
                    double *l_out)
{
    for (int d = 0; d < D; ++d)
        o[d] = 0.0;
    if (j1 <= j0) {
        *m_out = -INFINITY;
        *l_out = 0.0;
        return;
    }
    double m = -INFINITY;
    for (int64_t j = j0; j < j1; ++j) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d)
            acc += bf16_bits_to_double(qrow[d]) *
                   bf16_bits_to_double(krows[j * ld + d]);
        if (scale * acc > m)
            m = scale * acc;
    }
    double l = 0.0;
    for (int64_t j = j0; j < j1; ++j) {
        double acc = 0.0;
        for (int d = 0; d < D; ++d)
            acc += bf16_bits_to_double(qrow[d]) *
                   bf16_bits_to_double(krows[j * ld + d]);
        const double w = exp(scale * acc - m);
        l += w;
        for (int d = 0; d < D; ++d)
            o[d] += w * bf16_bits_to_double(vrows[j * ld + d]);
    }
    *m_out = m;
    *l_out = l;
}

/*
 * Log-sum-exp merge of S partial states (o_s[D], m_s, l_s) of one row:
 *   M = max over s with l_s > 0 of m_s,  L = sum l_s exp(m_s - M),
 *   out = sum o_s exp(m_s - M) / L,      lse = M + ln L.
 * No live partial (all l_s = 0) gives out = 0, lse = -inf.
 * o is [S, D] row-major.
 */
void oracle_merge(int D, int S, const double *o, const double *m,
                  const double *l, double *out, double *lse)
{
    double M = -INFINITY;
    for (int s = 0; s < S; ++s)
        if (l[s] > 0.0 && m[s] > M)
            M = m[s];
    for (int d = 0; d < D; ++d)
        out[d] = 0.0;
    if (M == -INFINITY) {
        *lse = -INFINITY;
        return;
    }
    double L = 0.0;
    for (int s = 0; s < S; ++s) {
        if (!(l[s] > 0.0))
            continue;
        const double w = exp(m[s] - M);
        L += l[s] * w;
        for (int d = 0; d < D; ++d)
            out[d] += o[(int64_t)s * D + d] * w;
    }
    for (int d = 0; d < D; ++d)
        out[d] /= L;
    *lse = M + log(L);
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
