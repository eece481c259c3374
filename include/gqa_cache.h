/*
 * gqa_cache.h -- the KV-cache append step that precedes every decode step, and
 * a host-side pool of page ids for paged caches.
 *
 * Decode reads a cache that grows by one token per sequence and step; the
 * cache lives in fixed-size blocks of tokens reached through a per-sequence
 * table ("GQA and MQA: Mathematical Foundations, KV-Cache Bandwidth Reduction
 * ..." (llms.blog), section "PagedAttention"; "Grouped-Query Attention"
 * (aiwiki), "Interaction with the cache": one page holds a KV group's tokens
 * for all h/g query heads of the group).  The layouts are those of gqa.h.
 *
 * The split of work follows serving practice: the host keeps every sequence's
 * length and owns the page ids (gqa_page_pool_*), so it knows, without
 * reading the GPU, which sequences start a new page this step
 * (seqlens[s] % page_size == 0); it takes ids from the pool, writes them into
 * the page table, and launches gqa_kv_append, which writes the tokens on the
 * GPU.  Decode then reads them like any other cached token.
 */
#ifndef GQA_CACHE_H
#define GQA_CACHE_H

#include "gqa.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * gqa_kv_append -- for every sequence s, with t = seqlens[s] on entry:
 *     paged (page_table != NULL): page = page_table[s * max_pages_per_seq + t / page_size],
 *                                 row = t % page_size
 *     contiguous:                 page = s, row = t   (the cache is [b, G, m, d])
 *     k_cache[page, g, row, :] = k_new[s, g, :] and v_cache likewise, for all g < G;
 *     seqlens[s] = t + 1.
 *
 * k_new, v_new: bf16 [b, G, d] device memory, 16-byte aligned.  k_cache,
 * v_cache: the pools of gqa.h, 16-byte aligned, written in place.  seqlens:
 * int32 [b] device memory, read and incremented.  page_table: int32
 * [b, max_pages_per_seq] device memory, read only (the entry for position t
 * must already hold a page of the pool), or NULL for the contiguous cache.
 * dims: as for decode (num_heads must be a multiple of num_kv_heads; only G,
 * d, page_size, num_pages, max_pages_per_seq and batch are used).
 * A position t outside [0, capacity) ORs GQA_STATUS_BAD_SEQLEN into *status,
 * a page id outside [0, num_pages) ORs GQA_STATUS_BAD_PAGE; such a sequence is
 * left untouched (nothing written, length unchanged).  Asynchronous on
 * `stream`; every sequence's row is written by one thread block, the length
 * after the block's writes.  Returns GQA_OK or a GQA_ERR_* code (nothing
 * launched on error).
 */
int gqa_kv_append(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                  int32_t *seqlens, const int32_t *page_table, const gqa_dims *dims,
                  uint32_t *status, void *stream);

/*
 * gqa_append_decode_split -- one decode step of a growing cache in one call:
 * gqa_kv_append(k_new, v_new, ...) followed by gqa_decode_split over the
 * cache with the new token (seqlens as incremented by the append; max_seqlen
 * bounds the lengths after it).  The decode kernel is launched as a
 * programmatic dependent of the append, so its blocks are dispatched while
 * the append runs and wait for it on the GPU before reading the cache.  Every
 * argument of both steps is checked before anything is launched; the results
 * equal the two calls made one after the other, bit for bit.
 */
int gqa_append_decode_split(const void *k_new, const void *v_new, const void *q, void *k_cache,
                            void *v_cache, int32_t *seqlens, const int32_t *page_table, float *out,
                            const gqa_dims *dims, float scale, uint32_t *status, int32_t split_tokens,
                            int32_t max_seqlen, void *workspace, size_t workspace_bytes, void *stream);

/*
 * A pool of page ids 0 .. num_pages-1 (host memory only; no GPU call).  Ids
 * are handed out lowest first from a fresh pool and most recently freed first
 * afterwards, so a sequence of calls always gives the same ids.  All calls on
 * one pool are serialised by a lock inside it.
 *
 * gqa_page_pool_create: NULL if num_pages < 1 or memory is short.
 * gqa_page_pool_alloc: writes n ids to ids[0 .. n-1]; GQA_ERR_NO_PAGES (and
 *   nothing taken) when fewer than n are free; GQA_ERR_DIMS for n < 0.
 * gqa_page_pool_free: returns n ids; GQA_ERR_DIMS (and nothing returned) if
 *   any id is outside the pool, not currently allocated, or listed twice.
 * gqa_page_pool_available: free ids, or GQA_ERR_NULL_POINTER.
 */
typedef struct gqa_page_pool gqa_page_pool;

gqa_page_pool *gqa_page_pool_create(int32_t num_pages);
void gqa_page_pool_destroy(gqa_page_pool *pool);
int32_t gqa_page_pool_available(const gqa_page_pool *pool);
int gqa_page_pool_alloc(gqa_page_pool *pool, int32_t n, int32_t *ids);
int gqa_page_pool_free(gqa_page_pool *pool, const int32_t *ids, int32_t n);

#ifdef __cplusplus
}
#endif

#endif /* GQA_CACHE_H */
