/*
 * smla_indexer_oracle.c -- plain fp64 CPU oracle for the top-k indexer, the
 * step that produces the sparse decode's index lists.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests and the benchmark's CPU legs use it.  It
 * shares no code, header or helper with the CUDA library (nor with the decode
 * oracle), and every loop follows the definition in the order it is written.
 *
 * What it computes (sources):
 *  - "The Negative Result That Refined the Hunt: Disabling the MMA FlashMLA
 *    Kernel", section "The Context: A Systematic Bisection Campaign": the
 *    deployment runs an indexer kernel and a bf16 index-key path ahead of the
 *    sparse MLA decode kernel.
 *  - "The Moment of Truth: Validating Split-K Parallelization for Blackwell MLA
 *    Decode", section "The Split-K Imperative": the decode kernel attends
 *    over the top-k candidate tokens retrieved from the KV cache.
 *  - The pages print no formula.  The reading used here is the published
 *    DeepSeek sparse-attention indexer: per query token t and cached position
 *    s of its sequence,
 *      logit[j, s] = qI[t, j, :] . kI[row(s), :]            (dI bf16 values)
 *      I[s]        = sum_j w[t, j] * max(0, logit[j, s])     (HI index heads)
 *    and the selection is the min(K, n) visible positions s in [0, n) with the
 *    largest I; equal scores are ordered by the smaller position first.  The
 *    output lists the selected positions in ascending order, then -1 up to
 *    width K.  A position maps to the physical index-key row
 *      page_table[b][s / page_size] * page_size + s % page_size
 *    (the latent cache's page table).  A visible position whose page entry
 *    lies outside [0, num_pages), or beyond pt_stride * page_size, is not a
 *    candidate and is counted (the return value).
 *
 * smla_ix_oracle_select applies the same selection to scores given from
 * outside (positions with a NaN score are not candidates), so that a
 * selection made from another implementation's scores can be checked with
 * that implementation's own rounding.
 *
 * Inputs: qI and kI are bf16 bit patterns (uint16), widened exactly to
 * double; w is fp32, widened exactly.  Parity pins:
 * tests/test_indexer_oracle.py.  No function here is unpinned.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double ix_bf16(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Physical index-key row of position s of a sequence, or -1 (not a candidate). */
static int64_t ix_row(int64_t s, const int32_t *pt_row, int pt_stride, int page_size,
                      int64_t num_pages)
{
    if (s < 0 || s >= (int64_t)pt_stride * page_size)
        return -1;
    int32_t page = pt_row[s / page_size];
    if (page < 0 || (int64_t)page >= num_pages)
        return -1;
    return (int64_t)page * page_size + s % page_size;
}

/* Index score of one query token against one index-key row. */
static double ix_score(const uint16_t *q_t, const float *w_t, const uint16_t *k_row, int HI,
                       int DI)
{
    double total = 0.0;
    for (int j = 0; j < HI; ++j) {
        double logit = 0.0;
        for (int d = 0; d < DI; ++d)
            logit += ix_bf16(q_t[(int64_t)j * DI + d]) * ix_bf16(k_row[d]);
        double relu = logit > 0.0 ? logit : 0.0;
        total += (double)w_t[j] * relu;
    }
    return total;
}

typedef struct {
    double score;
    int64_t pos;
} ix_cand;

/* Order of the selection: larger score first, then the smaller position. */
static int ix_by_score(const void *a, const void *b)
{
    const ix_cand *x = (const ix_cand *)a, *y = (const ix_cand *)b;
    if (x->score > y->score)
        return -1;
    if (x->score < y->score)
        return 1;
    return (x->pos < y->pos) ? -1 : (x->pos > y->pos);
}

static int ix_by_pos(const void *a, const void *b)
{
    const int32_t x = *(const int32_t *)a, y = *(const int32_t *)b;
    return (x > y) - (x < y);
}

/* The selection from m candidates: the first min(K, m) in selection order,
 * written as ascending positions, then -1 up to width K. */
static void ix_finish(ix_cand *cand, int64_t m, int K, int32_t *o)
{
    qsort(cand, (size_t)m, sizeof(ix_cand), ix_by_score);
    const int64_t take = m < K ? m : K;
    for (int64_t i = 0; i < take; ++i)
        o[i] = (int32_t)cand[i].pos;
    qsort(o, (size_t)take, sizeof(int32_t), ix_by_pos);
    for (int64_t i = take; i < K; ++i)
        o[i] = -1;
}

/*
 * Scores of every visible position of every query token.
 *   qI  bf16 bits [B, T, HI, DI]     w  fp32 [B, T, HI]
 *   kI  bf16 bits [num_pages * page_size, DI]
 *   page_table int32 [B, pt_stride]  n_vis int32 [B, T]
 * scores [B, T, n_max]: I for s < n_vis[b, t] that are candidates, -inf
 * elsewhere.  Returns the number of visible positions that are not candidates.
 */
long smla_ix_oracle_scores(const uint16_t *qI, const float *w, const uint16_t *kI,
                           const int32_t *page_table, int pt_stride, int64_t num_pages,
                           const int32_t *n_vis, int B, int T, int HI, int DI,
                           int page_size, int n_max, double *scores)
{
    long n_bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : n_bad)
    for (int u = 0; u < B * T; ++u) {
        const int b = u / T;
        const int32_t *pt_row = page_table + (int64_t)b * pt_stride;
        double *out = scores + (int64_t)u * n_max;
        for (int s = 0; s < n_max; ++s)
            out[s] = -INFINITY;
        for (int64_t s = 0; s < n_vis[u] && s < n_max; ++s) {
            int64_t r = ix_row(s, pt_row, pt_stride, page_size, num_pages);
            if (r < 0) {
                ++n_bad;
                continue;
            }
            out[s] = ix_score(qI + (int64_t)u * HI * DI, w + (int64_t)u * HI,
                              kI + r * DI, HI, DI);
        }
    }
    return n_bad;
}

/*
 * Top-k selection: out [B, T, K] int32 as described in the header.
 * Returns the number of visible positions that are not candidates.
 */
long smla_ix_oracle_topk(const uint16_t *qI, const float *w, const uint16_t *kI,
                         const int32_t *page_table, int pt_stride, int64_t num_pages,
                         const int32_t *n_vis, int B, int T, int HI, int DI, int page_size,
                         int K, int32_t *out)
{
    long n_bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : n_bad)
    for (int u = 0; u < B * T; ++u) {
        const int b = u / T;
        const int32_t *pt_row = page_table + (int64_t)b * pt_stride;
        const int64_t n = n_vis[u] > 0 ? n_vis[u] : 0;
        ix_cand *cand = (ix_cand *)malloc(sizeof(ix_cand) * (size_t)(n > 0 ? n : 1));
        int64_t m = 0;
        /* 1. every visible candidate with its score */
        for (int64_t s = 0; s < n; ++s) {
            int64_t r = ix_row(s, pt_row, pt_stride, page_size, num_pages);
            if (r < 0) {
                ++n_bad;
                continue;
            }
            cand[m].score = ix_score(qI + (int64_t)u * HI * DI, w + (int64_t)u * HI,
                                     kI + r * DI, HI, DI);
            cand[m].pos = s;
            ++m;
        }
        ix_finish(cand, m, K, out + (int64_t)u * K);
        free(cand);
    }
    return n_bad;
}

/*
 * Selection from given scores [B*T, n_max] (double; NaN = not a candidate)
 * for positions s < n_vis[u]: out [B*T, K] as smla_ix_oracle_topk writes it.
 */
void smla_ix_oracle_select(const double *scores, const int32_t *n_vis, int BT, int n_max, int K,
                           int32_t *out)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int u = 0; u < BT; ++u) {
        const int64_t n = n_vis[u] < 0 ? 0 : (n_vis[u] > n_max ? n_max : n_vis[u]);
        ix_cand *cand = (ix_cand *)malloc(sizeof(ix_cand) * (size_t)(n > 0 ? n : 1));
        int64_t m = 0;
        for (int64_t s = 0; s < n; ++s) {
            const double v = scores[(int64_t)u * n_max + s];
            if (isnan(v))
                continue;
            cand[m].score = v;
            cand[m].pos = s;
            ++m;
        }
        ix_finish(cand, m, K, out + (int64_t)u * K);
        free(cand);
    }
}
