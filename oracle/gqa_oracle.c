/*
 * gqa_oracle.c -- plain float64 CPU oracle for grouped-query attention (GQA)
 * decode over a contiguous or paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the checker, not the product: only
 * the test suite, the smoke check and the benchmark's CPU-baseline leg load it.
 * It shares no code, header, table or helper with the CUDA library, and it
 * never calls it.  It is deliberately slow and written for reading, not speed.
 *
 * What it computes (for every sequence s and query head i of H):
 *
 *   r     = H / G                       query heads per KV group
 *   g(i)  = i / r                       (integer division)
 *   l_j   = scale * sum_k q[s,i,k] * K[s,g(i),j,k]      for j < len_s
 *   w_j   = exp(l_j - max_j l_j) / sum_j exp(l_j - max_j l_j)
 *   out[s,i,:] = sum_j w_j * V[s,g(i),j,:]
 *   lse[s,i]   = ln sum_j exp(l_j)            (oracle_gqa_decode_lse only)
 *
 * oracle_gqa_decode_multi generalises this to nq query tokens per sequence
 * (speculative-decoding verification): q and out are [b, nq, H, d], and query
 * token t (0 .. nq-1) of sequence s attends the cached positions
 * j < len_s - (nq - 1 - t), i.e. every cached token before it and itself,
 * not the drafts after it (the mask of a causal decoder, aligned to the end
 * of the cache).  nq = 1 is the decode above.
 *
 * oracle_gqa_decode_mapped takes the KV group of every query head from a table,
 * g(i) = group_of_head[i] (any values in [0, G), groups of unequal size or
 * with no head allowed), instead of g(i) = i / (H/G); H need not be a multiple
 * of G.  The table i -> i / (H/G) is the decode above.
 *
 * Sources, by page and section:
 *  - "Grouped-Query Attention" (aiwiki), the PyTorch module: keys and values are
 *    broadcast to the query heads of their group by repeat_interleave(h // g,
 *    dim=1), so group g serves the contiguous query heads g*r .. g*r+r-1, and
 *    scaled_dot_product_attention supplies softmax(q k^T * scale) v with the
 *    default scale 1/sqrt(d_k).
 *  - "GQA and MQA: Mathematical Foundations, KV-Cache Bandwidth Reduction ..."
 *    (llms.blog), "Multi-Query Attention / Mathematical Formulation": logits =
 *    einsum(bhnk,bmk->bhnm), weights = softmax(logits + mask), O =
 *    einsum(bhnm,bmv->bhnv); "Grouped-Query Attention / Mathematical
 *    Formulation": the cache has shape [b, G, m, d_k] and each group's key and
 *    value heads are broadcast to its H/G query heads.
 *  - same page, "PagedAttention": the cache is managed in fixed-size blocks of
 *    tokens (a page-table indirection); "Grouped-Query Attention" (aiwiki),
 *    "Interaction with the cache": a page is shared by the h/g query heads.
 *
 * Readings taken where the pages leave a step open:
 *  - decode: one new query token per sequence attends every cached position
 *    j < len_s (the mask only removes positions at or beyond len_s);
 *  - paged layout: pools K and V of shape [num_pages, G, P, d]; logical token t
 *    of sequence s lives in page page_table[s * max_pages_per_seq + t / P] at
 *    row t % P.  A NULL page table means the contiguous cache [b, G, m, d],
 *    i.e. page_size = m and sequence s is "page" s;
 *  - invalid data: len_s < 1 or len_s > capacity sets bit 1 of *status and a
 *    page id outside [0, num_pages) sets bit 2; such a row is written as zeros
 *    (and its lse as -infinity).
 *  - lse is the logarithm of the softmax's normaliser, sum_j exp(l_j), the
 *    quantity that lets softmax results over disjoint parts of a sequence be
 *    combined (a reading: the pages' softmax defines it but does not name it).
 *
 * Inputs are bf16 bit patterns (uint16), expanded exactly to double; every sum
 * is accumulated in double in the logical token order j = 0, 1, ..., len_s - 1.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_STATUS_BAD_SEQLEN 1
#define ORACLE_STATUS_BAD_PAGE 2

/* Exact widening of a bf16 bit pattern: bf16 is the top half of an IEEE fp32. */
static double bf16_to_f64(uint16_t bits)
{
    uint32_t word = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &word, sizeof f);
    return (double)f;
}

/*
 * Element offset of row (token) t of KV group g for sequence s, or -1 when the
 * page id found in the table is outside the pool.
 */
static long long kv_row_offset(const int32_t *page_table, int32_t s, int32_t t,
                               int32_t g, int32_t G, int32_t d, int32_t page_size,
                               int32_t num_pages, int32_t max_pages_per_seq)
{
    long long page;
    long long row_in_page;
    if (page_table == NULL) {
        page = s;                 /* contiguous [b, G, m, d]: m = page_size */
        row_in_page = t;
    } else {
        page = page_table[(long long)s * max_pages_per_seq + t / page_size];
        row_in_page = t % page_size;
    }
    if (page < 0 || page >= num_pages)
        return -1;
    return ((page * G + g) * (long long)page_size + row_in_page) * d;
}

/*
 * Decode attention for the listed rows; `lse` (may be NULL) receives
 * ln sum_j exp(l_j) per row.
 *
 * q        [b, H, d] bf16 bits
 * k_cache  [num_pages, G, page_size, d] bf16 bits (contiguous: [b, G, m, d])
 * v_cache  same layout as k_cache
 * seqlens  [b] cached length of each sequence (the new token included)
 * page_table [b, max_pages_per_seq] int32, or NULL for the contiguous cache
 * rows     list of flat row ids s * H + i, or NULL for all b * H rows
 * out      [nrows, d] float64 (row order of `rows`)
 * status   receives the OR of the status bits of every computed row
 * nthreads number of OpenMP threads (<= 0: library default)
 *
 * Returns 0, or -1 on bad arguments (nothing is written then).
 */
static int decode_rows(const uint16_t *q, const uint16_t *k_cache,
                       const uint16_t *v_cache, const int32_t *seqlens,
                       const int32_t *page_table, int32_t b, int32_t nq, int32_t H, int32_t G,
                       int32_t d, int32_t page_size, int32_t num_pages,
                       int32_t max_pages_per_seq, double scale,
                       const int64_t *rows, int64_t nrows, double *out, double *lse,
                       int32_t *status, int32_t nthreads, const int32_t *group_of_head)
{
    if (!q || !k_cache || !v_cache || !seqlens || !out || !status)
        return -1;
    if (b < 1 || nq < 1 || H < 1 || G < 1 || d < 1 || page_size < 1 || num_pages < 1)
        return -1;
    if (group_of_head == NULL && H % G != 0)
        return -1;
    if (group_of_head != NULL)
        for (int32_t i = 0; i < H; ++i)
            if (group_of_head[i] < 0 || group_of_head[i] >= G)
                return -1;
    if (page_table != NULL && max_pages_per_seq < 1)
        return -1;
    if (rows == NULL)
        nrows = (int64_t)b * nq * H;

    const int32_t r = H / G;
    const long long capacity =
        page_table ? (long long)max_pages_per_seq * page_size : (long long)page_size;
    int32_t status_all = 0;

#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads > 0 ? nthreads : omp_get_max_threads()) reduction(| : status_all)
#endif
    for (int64_t n = 0; n < nrows; ++n) {
        const int64_t row = rows ? rows[n] : n;
        double *o = out + n * (int64_t)d;
        for (int32_t k = 0; k < d; ++k)
            o[k] = 0.0;
        if (lse)
            lse[n] = -INFINITY;
        if (row < 0 || row >= (int64_t)b * nq * H) {
            status_all |= ORACLE_STATUS_BAD_SEQLEN;
            continue;
        }
        const int32_t s = (int32_t)(row / ((int64_t)nq * H));   /* row = (s * nq + tq) * H + i */
        const int32_t tq = (int32_t)((row / H) % nq);
        const int32_t i = (int32_t)(row % H);
        const int32_t g = group_of_head ? group_of_head[i] : i / r;
        const int32_t len_s = seqlens[s];
        if (len_s < nq || len_s > capacity) {
            status_all |= ORACLE_STATUS_BAD_SEQLEN;
            continue;
        }
        /* positions this query token sees: the cache up to and including itself */
        const int32_t len = len_s - (nq - 1 - tq);

        /* Every page this row touches must lie in the pool. */
        int bad_page = 0;
        for (int32_t t = 0; t < len; ++t) {
            if (kv_row_offset(page_table, s, t, g, G, d, page_size, num_pages,
                              max_pages_per_seq) < 0) {
                bad_page = 1;
                break;
            }
        }
        if (bad_page) {
            status_all |= ORACLE_STATUS_BAD_PAGE;
            continue;
        }

        double *logits = (double *)malloc(sizeof(double) * (size_t)len);
        if (logits == NULL) {
            status_all |= ORACLE_STATUS_BAD_SEQLEN;
            continue;
        }
        const uint16_t *qi = q + row * (int64_t)d;

        /* logits l_j = scale * q_i . k_j */
        for (int32_t t = 0; t < len; ++t) {
            const long long off = kv_row_offset(page_table, s, t, g, G, d, page_size,
                                                num_pages, max_pages_per_seq);
            double dot = 0.0;
            for (int32_t k = 0; k < d; ++k)
                dot += bf16_to_f64(qi[k]) * bf16_to_f64(k_cache[off + k]);
            logits[t] = scale * dot;
        }

        /* softmax with the maximum subtracted (the result is the same for any
         * constant; the maximum keeps exp() finite) */
        double mx = logits[0];
        for (int32_t t = 1; t < len; ++t)
            if (logits[t] > mx)
                mx = logits[t];
        double denom = 0.0;
        for (int32_t t = 0; t < len; ++t) {
            logits[t] = exp(logits[t] - mx);
            denom += logits[t];
        }
        /* ln sum_j exp(l_j) = mx + ln sum_j exp(l_j - mx) */
        if (lse)
            lse[n] = mx + log(denom);

        /* out = sum_j w_j v_j */
        for (int32_t t = 0; t < len; ++t) {
            const long long off = kv_row_offset(page_table, s, t, g, G, d, page_size,
                                                num_pages, max_pages_per_seq);
            const double w = logits[t] / denom;
            for (int32_t k = 0; k < d; ++k)
                o[k] += w * bf16_to_f64(v_cache[off + k]);
        }
        free(logits);
    }
    *status = status_all;
    return 0;
}

/*
 * Arguments:
 * q        [b, H, d] bf16 bits
 * k_cache  [num_pages, G, page_size, d] bf16 bits (contiguous: [b, G, m, d])
 * v_cache  same layout as k_cache
 * seqlens  [b] cached length of each sequence (the new token included)
 * page_table [b, max_pages_per_seq] int32, or NULL for the contiguous cache
 * rows     list of flat row ids s * H + i, or NULL for all b * H rows
 * out      [nrows, d] float64 (row order of `rows`)
 * status   receives the OR of the status bits of every computed row
 * nthreads number of OpenMP threads (<= 0: library default)
 * Returns 0, or -1 on bad arguments (nothing is written then).
 */
int oracle_gqa_decode(const uint16_t *q, const uint16_t *k_cache,
                      const uint16_t *v_cache, const int32_t *seqlens,
                      const int32_t *page_table, int32_t b, int32_t H, int32_t G,
                      int32_t d, int32_t page_size, int32_t num_pages,
                      int32_t max_pages_per_seq, double scale,
                      const int64_t *rows, int64_t nrows, double *out,
                      int32_t *status, int32_t nthreads)
{
    return decode_rows(q, k_cache, v_cache, seqlens, page_table, b, 1, H, G, d,
                       page_size, num_pages, max_pages_per_seq, scale, rows, nrows,
                       out, NULL, status, nthreads, NULL);
}

/* The same, plus lse [nrows] = ln sum_j exp(l_j) of each row (-inf for a row
 * with a status bit). */
int oracle_gqa_decode_lse(const uint16_t *q, const uint16_t *k_cache,
                          const uint16_t *v_cache, const int32_t *seqlens,
                          const int32_t *page_table, int32_t b, int32_t H, int32_t G,
                          int32_t d, int32_t page_size, int32_t num_pages,
                          int32_t max_pages_per_seq, double scale,
                          const int64_t *rows, int64_t nrows, double *out, double *lse,
                          int32_t *status, int32_t nthreads)
{
    if (!lse)
        return -1;
    return decode_rows(q, k_cache, v_cache, seqlens, page_table, b, 1, H, G, d,
                       page_size, num_pages, max_pages_per_seq, scale, rows, nrows,
                       out, lse, status, nthreads, NULL);
}

/* nq query tokens per sequence: q, out [b, nq, H, d] (rows (s * nq + t) * H + i),
 * lse [nrows] or NULL; a length below nq is invalid (status bit 1). */
int oracle_gqa_decode_multi(const uint16_t *q, const uint16_t *k_cache,
                            const uint16_t *v_cache, const int32_t *seqlens,
                            const int32_t *page_table, int32_t b, int32_t nq, int32_t H,
                            int32_t G, int32_t d, int32_t page_size, int32_t num_pages,
                            int32_t max_pages_per_seq, double scale,
                            const int64_t *rows, int64_t nrows, double *out, double *lse,
                            int32_t *status, int32_t nthreads)
{
    return decode_rows(q, k_cache, v_cache, seqlens, page_table, b, nq, H, G, d,
                       page_size, num_pages, max_pages_per_seq, scale, rows, nrows,
                       out, lse, status, nthreads, NULL);
}

/* Any group map: group_of_head[H] with values in [0, G); lse [nrows] or NULL. */
int oracle_gqa_decode_mapped(const uint16_t *q, const uint16_t *k_cache,
                             const uint16_t *v_cache, const int32_t *seqlens,
                             const int32_t *page_table, int32_t b, int32_t H, int32_t G,
                             int32_t d, int32_t page_size, int32_t num_pages,
                             int32_t max_pages_per_seq, double scale,
                             const int64_t *rows, int64_t nrows, double *out, double *lse,
                             int32_t *status, int32_t nthreads, const int32_t *group_of_head)
{
    if (!group_of_head)
        return -1;
    return decode_rows(q, k_cache, v_cache, seqlens, page_table, b, 1, H, G, d,
                       page_size, num_pages, max_pages_per_seq, scale, rows, nrows,
                       out, lse, status, nthreads, group_of_head);
}

/* Number of OpenMP threads a parallel region would use by default. */
int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
