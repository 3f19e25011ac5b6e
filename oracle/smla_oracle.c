/*
 * smla_oracle.c -- plain fp64 CPU oracle for split-K sparse MLA decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header or helper with the CUDA
 * library, and it is deliberately slow: every loop follows the definition in
 * the order it is written, with no blocking, fusion or reordering.
 *
 * What it computes (sources):
 *  - "The Moment of Truth: Validating Split-K Parallelization for Blackwell MLA
 *    Decode", section "The Split-K Imperative": the decode kernel attends over
 *    the top-k candidate tokens retrieved from the KV cache; split-K partitions
 *    that top-k axis across blocks, each block writes a partial attention
 *    output, and a log-sum-exp (LSE) combine kernel merges the partials.
 *  - "The Occupancy Hypothesis: How One Kernel Parameter Unlocked 1.8x Decode
 *    Speedup on Blackwell", section "The Occupancy Insight": NSPLIT is the
 *    number of chunks one query's work is cut into.
 *  - The pages print no formula, dimension or index convention.  The readings
 *    used here are the standard absorbed-MLA decode definition:
 *      row r of the latent cache = [ c_r (dc values) | k_pe_r (dr values) ]
 *      q_h = [ q_nope_h (dc) | q_pe_h (dr) ]
 *      s_j = scale * ( q_nope_h . c_r + q_pe_h . k_pe_r ),  r = row of idx[j]
 *      p_j = exp(s_j - M) / L,  M = max_j s_j,  L = sum_j exp(s_j - M)
 *      o_h = sum_j p_j c_r,     lse_h = M + ln L   (natural log)
 *    An index is a logical token position of sequence b; it maps to the
 *    physical row page_table[b][i / page_size] * page_size + i % page_size.
 *    Index -1 is padding and contributes nothing.  Any other index outside
 *    [0, pt_stride * page_size), or one whose page entry lies outside
 *    [0, num_pages), is treated like -1 and counted (the return value).
 *    No valid index: o = 0, lse = -inf.  Duplicate indices each count once
 *    per occurrence (a sum over the list).
 *
 * Inputs are bf16 bit patterns (uint16), widened exactly to double.
 * Parity pins: tests/test_oracle_pins.py.  No function here is unpinned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 -> double: bf16 is the top half of an IEEE binary32. Exact. */
static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Logical index -> physical cache row, or -1 when the entry is masked.
 * *bad is set to 1 when the entry is neither -1 nor in range. */
static int64_t resolve_row(int32_t i, const int32_t *pt_row, int pt_stride,
                           int page_size, int64_t num_pages, int *bad)
{
    *bad = 0;
    if (i == -1)
        return -1;
    if (i < 0 || (int64_t)i >= (int64_t)pt_stride * page_size) {
        *bad = 1;
        return -1;
    }
    int32_t page = pt_row[i / page_size];
    if (page < 0 || (int64_t)page >= num_pages) {
        *bad = 1;
        return -1;
    }
    return (int64_t)page * page_size + (i % page_size);
}

/* Score of one head against one cache row: scale * (q_nope.c + q_pe.k_pe). */
static double score(const uint16_t *qh, const uint16_t *row, int dc, int dr,
                    double scale)
{
    double dot_nope = 0.0, dot_pe = 0.0;
    for (int d = 0; d < dc; ++d)
        dot_nope += bf16_bits_to_double(qh[d]) * bf16_bits_to_double(row[d]);
    for (int d = 0; d < dr; ++d)
        dot_pe += bf16_bits_to_double(qh[dc + d]) * bf16_bits_to_double(row[dc + d]);
    return scale * (dot_nope + dot_pe);
}

/*
 * Softmax attention of one head over the index positions [j0, j1) of one
 * query token.  Writes the UNNORMALISED output sum_j exp(s_j - m) c_j, the
 * max m and l = sum_j exp(s_j - m).  With no valid entry: out = 0, m = -inf,
 * l = 0.  Returns the number of out-of-range entries seen.
 */
static long attend_range(const uint16_t *qh, const uint16_t *cache,
                         const int32_t *pt_row, int pt_stride, int64_t num_pages,
                         const int32_t *idx_bt, int j0, int j1, int dc, int dr,
                         int page_size, double scale, double *s_buf,
                         int64_t *row_buf, double *out, double *m_out,
                         double *l_out)
{
    const int D = dc + dr;
    long n_bad = 0;
    int n_valid = 0;
    double m = -INFINITY;

    /* 1. scores of the valid entries, and their max */
    for (int j = j0; j < j1; ++j) {
        int bad;
        int64_t r = resolve_row(idx_bt[j], pt_row, pt_stride, page_size,
                                num_pages, &bad);
        n_bad += bad;
        if (r < 0)
            continue;
        double s = score(qh, cache + r * D, dc, dr, scale);
        s_buf[n_valid] = s;
        row_buf[n_valid] = r;
        ++n_valid;
        if (s > m)
            m = s;
    }

    for (int d = 0; d < dc; ++d)
        out[d] = 0.0;
    if (n_valid == 0) {
        *m_out = -INFINITY;
        *l_out = 0.0;
        return n_bad;
    }

    /* 2. l = sum exp(s - m);  out = sum exp(s - m) c */
    double l = 0.0;
    for (int v = 0; v < n_valid; ++v) {
        double w = exp(s_buf[v] - m);
        l += w;
        const uint16_t *c = cache + row_buf[v] * D;
        for (int d = 0; d < dc; ++d)
            out[d] += w * bf16_bits_to_double(c[d]);
    }
    *m_out = m;
    *l_out = l;
    return n_bad;
}

int smla_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void smla_oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Unsplit decode.  Layouts (row-major, contiguous):
 *   q          [B, T, H, dc+dr]  bf16 bits
 *   cache      [num_pages * page_size, dc+dr] bf16 bits
 *   page_table [B, pt_stride] int32
 *   idx        [B, T, K] int32, -1 = padding
 *   o          [B, T, H, dc] double (normalised output)
 *   lse        [B, T, H] double
 * Returns the number of out-of-range entries (counted once per head).
 */
long smla_oracle_decode(const uint16_t *q, const uint16_t *cache,
                        const int32_t *page_table, int pt_stride,
                        int64_t num_pages, const int32_t *idx, int B, int T,
                        int H, int K, int dc, int dr, int page_size,
                        double scale, double *o, double *lse)
{
    const int D = dc + dr;
    long n_bad = 0;
    const long n_units = (long)B * T * H;
#pragma omp parallel reduction(+ : n_bad)
    {
        double *s_buf = (double *)malloc(sizeof(double) * (K > 0 ? K : 1));
        int64_t *row_buf = (int64_t *)malloc(sizeof(int64_t) * (K > 0 ? K : 1));
#pragma omp for schedule(dynamic, 1)
        for (long u = 0; u < n_units; ++u) {
            const int h = (int)(u % H);
            const int t = (int)((u / H) % T);
            const int b = (int)(u / ((long)H * T));
            const uint16_t *qh = q + u * D;
            const int32_t *idx_bt = idx + ((long)b * T + t) * K;
            const int32_t *pt_row = page_table + (long)b * pt_stride;
            double *oh = o + u * dc;
            double m, l;
            n_bad += attend_range(qh, cache, pt_row, pt_stride, num_pages,
                                  idx_bt, 0, K, dc, dr, page_size, scale,
                                  s_buf, row_buf, oh, &m, &l);
            if (l == 0.0) {
                lse[u] = -INFINITY;
                continue;
            }
            for (int d = 0; d < dc; ++d)
                oh[d] /= l;
            lse[u] = m + log(l);
        }
        free(s_buf);
        free(row_buf);
    }
    return n_bad;
}

/*
 * Split-K partial pass.  Split s covers index positions
 * [s*Kc, min(K, (s+1)*Kc)) with Kc = ceil(K / nsplit); trailing splits may be
 * short or empty.  For each (b, t, h, s):
 *   part_o   = sum_j exp(s_j - m_s) c_j        (unnormalised, dc values)
 *   part_m   = m_s = max_j s_j                 (-inf when empty)
 *   part_lse = m_s + ln sum_j exp(s_j - m_s)   (-inf when empty)
 * Layouts: part_o [B, T, H, nsplit, dc]; part_m, part_lse [B, T, H, nsplit].
 */
long smla_oracle_partial(const uint16_t *q, const uint16_t *cache,
                         const int32_t *page_table, int pt_stride,
                         int64_t num_pages, const int32_t *idx, int B, int T,
                         int H, int K, int dc, int dr, int page_size,
                         double scale, int nsplit, double *part_o,
                         double *part_m, double *part_lse)
{
    const int D = dc + dr;
    const int Kc = (K + nsplit - 1) / nsplit;
    long n_bad = 0;
    const long n_units = (long)B * T * H * nsplit;
#pragma omp parallel reduction(+ : n_bad)
    {
        double *s_buf = (double *)malloc(sizeof(double) * (K > 0 ? K : 1));
        int64_t *row_buf = (int64_t *)malloc(sizeof(int64_t) * (K > 0 ? K : 1));
#pragma omp for schedule(dynamic, 1)
        for (long u = 0; u < n_units; ++u) {
            const int s = (int)(u % nsplit);
            const long bth = u / nsplit;
            const int h = (int)(bth % H);
            const int t = (int)((bth / H) % T);
            const int b = (int)(bth / ((long)H * T));
            int j0 = s * Kc;
            int j1 = j0 + Kc;
            if (j0 > K)
                j0 = K;
            if (j1 > K)
                j1 = K;
            const uint16_t *qh = q + bth * D;
            const int32_t *idx_bt = idx + ((long)b * T + t) * K;
            const int32_t *pt_row = page_table + (long)b * pt_stride;
            double m, l;
            n_bad += attend_range(qh, cache, pt_row, pt_stride, num_pages,
                                  idx_bt, j0, j1, dc, dr, page_size, scale,
                                  s_buf, row_buf, part_o + u * dc, &m, &l);
            part_m[u] = m;
            part_lse[u] = (l == 0.0) ? -INFINITY : m + log(l);
        }
        free(s_buf);
        free(row_buf);
    }
    return n_bad;
}

/*
 * LSE combine of nsplit partials per (b, t, h):
 *   M   = max_s m_s
 *   L   = sum_s exp(lse_s - M)
 *   o   = sum_s exp(m_s - M) O_s / L
 *   lse = M + ln L
 * All splits empty (M = -inf): o = 0, lse = -inf.
 * n_units = B * T * H; part_o [n_units, nsplit, dc]; o [n_units, dc].
 */
void smla_oracle_combine(const double *part_o, const double *part_m,
                         const double *part_lse, long n_units, int nsplit,
                         int dc, double *o, double *lse)
{
#pragma omp parallel for schedule(static)
    for (long u = 0; u < n_units; ++u) {
        const double *m_u = part_m + u * nsplit;
        const double *lse_u = part_lse + u * nsplit;
        double *ou = o + u * dc;
        double M = -INFINITY;
        for (int s = 0; s < nsplit; ++s)
            if (m_u[s] > M)
                M = m_u[s];
        for (int d = 0; d < dc; ++d)
            ou[d] = 0.0;
        if (M == -INFINITY) {
            lse[u] = -INFINITY;
            continue;
        }
        double L = 0.0;
        for (int s = 0; s < nsplit; ++s)
            if (lse_u[s] != -INFINITY)
                L += exp(lse_u[s] - M);
        for (int s = 0; s < nsplit; ++s) {
            if (m_u[s] == -INFINITY)
                continue;
            const double w = exp(m_u[s] - M);
            const double *Os = part_o + (u * nsplit + s) * dc;
            for (int d = 0; d < dc; ++d)
                ou[d] += w * Os[d];
        }
        for (int d = 0; d < dc; ++d)
            ou[d] /= L;
        lse[u] = M + log(L);
    }
}
