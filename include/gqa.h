/*
 * gqa.h -- C ABI of libgqa: grouped-query attention (GQA) decode over a
 * contiguous or paged bf16 KV cache, written for NVIDIA B200 (sm_100a).
 *
 * The operation.  For every sequence s (one new query token each) and every
 * query head i of H, with r = H / G query heads per KV group and
 * g(i) = i / r:
 *
 *     out[s, i, :] = softmax_j( scale * q[s, i, :] . K[s, g(i), j, :] ) V[s, g(i), j, :]
 *
 * over the cached positions j < seqlens[s].  This is the attention of the
 * PyTorch module in "Grouped-Query Attention" (aiwiki), where keys and values
 * are broadcast to the query heads of their group with repeat_interleave(h // g,
 * dim=1) and fed to scaled_dot_product_attention; the same page's closing note
 * says the version that matters computes the KV-head index from the query-head
 * index inside the kernel and reads the cache once.  For G = 1 it is the
 * incremental multi-query attention of "GQA and MQA: Mathematical Foundations,
 * KV-Cache Bandwidth Reduction ..." (llms.blog, "Multi-Query Attention /
 * Mathematical Formulation": logits, softmax(logits + mask), weights . V); its
 * "Grouped-Query Attention / Mathematical Formulation" gives the [b, G, m, d_k]
 * cache.  The kernels read each KV group's keys and values from HBM once per
 * decode step and share them among the group's r query heads on chip; nothing
 * is expanded with repeat_interleave.
 *
 * Readings where the pages are silent: decode attends every cached position
 * j < seqlens[s] (the new token's K/V is already in the cache); there is no
 * causal mask beyond the length.  Paged pools follow the block-managed cache of
 * the llms.blog page's "PagedAttention" section with the layout below.
 *
 * Layouts (all row-major, all device memory owned by the caller):
 *   q          bf16  [b, H, d]
 *   k_cache    bf16  paged: [num_pages, G, page_size, d]   (pool of pages)
 *                    contiguous (page_table == NULL): [b, G, m, d] with
 *                    m = dims->page_size (the capacity of every sequence)
 *   v_cache    bf16  same layout as k_cache
 *   seqlens    int32 [b]  cached tokens of each sequence, 1 <= len <= capacity
 *   page_table int32 [b, max_pages_per_seq]: logical page t / page_size of
 *              sequence s is pool page page_table[s * max_pages_per_seq + t / page_size];
 *              entries past a sequence's length are never read (may be -1)
 *   out        fp32  [b, H, d]  fully overwritten
 *   status     uint32 (device), optional (may be NULL): the kernels OR
 *              GQA_STATUS_* bits into it; the caller zeroes it
 *
 * Capacity: contiguous m = page_size; paged max_pages_per_seq * page_size.
 *
 * Errors.  Every argument check happens on the host before anything is
 * launched; a failing call returns a negative GQA_ERR_* code and launches
 * nothing.  Data-dependent problems found on the device (a length outside
 * [1, capacity], a page id outside [0, num_pages)) never fault: the affected
 * output rows are written as zeros and the matching GQA_STATUS_* bit is ORed
 * into *status.  Page ids of the table are only turned into TMA coordinates,
 * which the copy engine bounds-checks (an id outside the pool reads zeros and
 * is flagged), so a corrupt table cannot make the kernel read outside the pool.
 *
 * Concurrency.  Calls are asynchronous on `stream` (a cudaStream_t passed as
 * void*; NULL = the legacy default stream).  The library allocates no device
 * memory and keeps no state between calls apart from per-device attribute
 * caches; calls on different streams are independent if their output and
 * workspace buffers are.
 */
#ifndef GQA_H
#define GQA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes of the host entry points. */
#define GQA_OK 0
#define GQA_ERR_NULL_POINTER (-1)  /* a required pointer is NULL */
#define GQA_ERR_MISALIGNED (-2)    /* q/k/v/out/workspace not 16-byte aligned */
#define GQA_ERR_HEADS (-3)         /* H % G != 0, or H/G above GQA_MAX_GROUP_RATIO */
#define GQA_ERR_HEAD_DIM (-4)      /* head_dim not in {64, 128} */
#define GQA_ERR_PAGE_SIZE (-5)     /* paged: page_size not a power of two in [8, 2^20] */
#define GQA_ERR_DIMS (-6)          /* a size is < 1 or too large */
#define GQA_ERR_SPLIT (-7)         /* split_tokens not a positive multiple of 128 */
#define GQA_ERR_WORKSPACE (-8)     /* workspace NULL or smaller than required */
#define GQA_ERR_CUDA (-9)          /* a CUDA runtime/driver call failed */
#define GQA_ERR_DEVICE (-10)       /* current device is not sm_100 (B200) */
#define GQA_ERR_NO_PAGES (-11)     /* page pool (gqa_cache.h): not enough free pages */

/* Bits the kernels OR into *status. */
#define GQA_STATUS_BAD_SEQLEN 1u   /* a length outside [1, capacity]: row zeroed */
#define GQA_STATUS_BAD_PAGE 2u     /* a page id outside [0, num_pages): row zeroed */
#define GQA_STATUS_TIMEOUT 4u      /* an on-chip pipeline wait gave up: output undefined; before replaying a
                                      captured graph whose call reported it, zero its workspace (a unit's
                                      arrival count may have been left part-way) */

/* Largest supported group ratio r = H / G. */
#define GQA_MAX_GROUP_RATIO 64

/* gqa_dims.flags: choice of the q.k / p.v contraction (default: automatic). */
#define GQA_FLAG_CONTRACT_MMA 1u   /* tensor cores (mma.sync m16n8k16 bf16) */
#define GQA_FLAG_CONTRACT_FMA 2u   /* fp32 FMA on CUDA cores; r = H/G <= 2 only (else GQA_ERR_HEADS) */
#define GQA_FLAG_CONTRACT_TCGEN05 4u /* 5th-gen tensor cores (tcgen05, accumulators in tensor memory): one block
                                        takes all rows of a group (r times the query tokens): <= 128 at
                                        d = 128, <= 64 at d = 64 (else GQA_ERR_HEADS); split entry points
                                        (fixed splits) only.  flags == 0 picks it by itself for more than
                                        GQA_TC_AUTO_ROWS rows per group */
/* Above this many rows per group the mma.sync kernel would need a second 16-row slice. */
#define GQA_TC_AUTO_ROWS 16

typedef struct gqa_dims {
    int32_t batch;             /* b: sequences, one query token each */
    int32_t num_heads;         /* H: query heads */
    int32_t num_kv_heads;      /* G: KV groups (heads of the cache) */
    int32_t head_dim;          /* d = d_k = d_v: 64 or 128 */
    int32_t page_size;         /* paged: tokens per page; contiguous: capacity m */
    int32_t num_pages;         /* paged: pages in each pool; contiguous: ignored (the pool is b sequences) */
    int32_t max_pages_per_seq; /* paged: row stride of page_table; contiguous: 0 */
    uint32_t flags;            /* GQA_FLAG_*; 0 = automatic */
} gqa_dims;

/*
 * gqa_decode -- one decode step without a workspace.
 *
 * Computes `out` as described above.  When the (sequence, group) units are
 * enough to occupy every SM, a persistent grid streams one unit after another
 * through a single TMA pipeline per block; otherwise each unit is handled by a
 * thread-block cluster (up to 16 blocks) whose blocks split the unit's tokens
 * and merge their partial softmax states through distributed shared memory.
 * Either way no global scratch memory is used.
 *
 * scale: the softmax scale (1/sqrt(d) is scaled_dot_product_attention's default).
 * Returns GQA_OK or a GQA_ERR_* code (nothing launched on error).
 */
int gqa_decode(const void *q, const void *k_cache, const void *v_cache,
               const int32_t *seqlens, const int32_t *page_table, float *out,
               const gqa_dims *dims, float scale, uint32_t *status, void *stream);

/*
 * Split-KV decode.  The tokens of every sequence are cut into consecutive
 * splits of `split_tokens`; one thread block per (sequence, group, split)
 * item yields an unnormalised partial softmax state, and the splits of each
 * (sequence, head) are merged exactly: with m_k the split's running maximum
 * and l_k its sum of exponentials,
 *     M = max_k m_k,  L = sum_k l_k 2^(m_k - M),  out = sum_k o_k 2^(m_k - M) / L.
 * With at most GQA_MERGE_IN_KERNEL_MAX_SPLITS splits the decode kernel merges
 * them itself (one launch): each block publishes its state and counts its
 * arrival in a per-unit word of the workspace, and the block that completes a
 * unit merges the unit's rows.  With more splits a second kernel merges them,
 * one block per row.  The merge is an exact re-association of the softmax of
 * the pages' formula (the pages do not describe split-KV; it is how a long
 * cache fills the GPU).
 *
 * split_tokens: a positive multiple of 128 (fixed splits as above), or 0 to
 *               let the library cut the work from the dims, max_seqlen and
 *               the SM count.  Paged dims (max_pages_per_seq > 0), the layout
 *               of choice for unequal lengths, get equal-work ranges
 *               (stream-K) for up to 1024 sequences: the tiles of all
 *               (sequence, group) units, in order, are cut into one contiguous
 *               range per resident thread block; a block finishes the units
 *               that lie wholly in its range and leaves partial states for the
 *               (at most two) units it shares with its neighbours, which the
 *               second kernel merges (longer paged batches: splits of 4096).
 *               Contiguous dims (max_pages_per_seq == 0) get fixed splits:
 *               one per unit when the units fill at least three quarters of
 *               the GPU's resident blocks (no combine); with too few units
 *               for that, gqa_decode_split (and its lse, verification and
 *               group-map forms, on the mma.sync contraction) runs
 *               thread-block clusters when they fill the GPU (see
 *               gqa_plan_decomposition_ex); otherwise as many splits
 *               per unit as still fit one wave of resident blocks.  With
 *               max_seqlen <= 256 no unit is split (one split of 256).
 * max_seqlen:   an upper bound of every seqlens[s] (sizes the grid and the
 *               workspace); a length above it is treated as invalid
 *               (GQA_STATUS_BAD_SEQLEN, row zeroed).
 * workspace:    device memory of at least gqa_decode_split_workspace_size()
 *               bytes for the same dims, max_seqlen and split_tokens, 16-byte
 *               aligned; its contents need no initialisation and are scratch
 *               after the call.  Each call tags the arrival words with its
 *               own number, so a word left by another call, or any other
 *               contents, counts as no arrival; a call captured in a CUDA
 *               graph keeps its number and every replay leaves the words
 *               ready for the next.  Calls that overlap on the GPU must use
 *               different workspaces.
 */
#define GQA_MERGE_IN_KERNEL_MAX_SPLITS 8
size_t gqa_decode_split_workspace_size(const gqa_dims *dims, int32_t max_seqlen,
                                       int32_t split_tokens);

int gqa_decode_split(const void *q, const void *k_cache, const void *v_cache,
                     const int32_t *seqlens, const int32_t *page_table, float *out,
                     const gqa_dims *dims, float scale, uint32_t *status,
                     int32_t split_tokens, int32_t max_seqlen, void *workspace,
                     size_t workspace_bytes, void *stream);

/*
 * The two kernels of gqa_decode_split as separate calls (same arguments and
 * workspace): gqa_split_partials writes the per-split partial states into the
 * workspace; gqa_split_combine merges them into `out`.  Running the first and
 * then the second on one stream gives exactly (bit for bit) the result of
 * gqa_decode_split, which merges in-kernel with the same arithmetic.  The combine is
 * also the merge step for partial states produced elsewhere (e.g. gathered
 * from other GPUs into this workspace).  Both calls must get the same dims,
 * split_tokens and max_seqlen, on the same device.  When split_tokens == 0
 * selects equal-work ranges, the workspace starts with a 256-byte header and
 * one record per (sequence, group) unit, written by gqa_split_partials and
 * read by gqa_split_combine, and `out` must be given to gqa_split_partials
 * (units that one block covers whole are written there directly).
 *
 * out (gqa_split_partials, may be NULL): a sequence that fits in one split is
 * finished by the partials kernel itself, which writes its rows to `out` and
 * marks split 0 so that the combine leaves them alone.  With out == NULL every
 * row goes through the workspace and the combine.
 *
 * Workspace layout for fixed splits (fp32, each array 256-byte aligned,
 * S = ceil(max_seqlen / split_tokens)): o [b, H, S, d] unnormalised sum_j 2^(x_j - m) v_j;
 * m [b, H, S] the base of the split's exponentials (at most 8 below the
 * maximum of x_j = scale * log2(e) * q.k_j, never above it);
 * l [b, H, S] sum_j 2^(x_j - m), or a marker: -1 the split met an invalid page
 * id; -2 (split 0) the length is outside [1, capacity]; -3 (split 0) the row
 * is already final in `out`.
 * Then one 64-bit arrival word per (sequence, group, 16-head slice) unit,
 * {call number: 40 bits, arrivals: 24 bits}, used by gqa_decode_split's
 * in-kernel merge only (gqa_split_partials leaves it alone).
 * Split k of sequence s covers tokens [k * split_tokens, min(len, (k+1) * split_tokens));
 * the combine reads the splits k < ceil(len / split_tokens).
 */
int gqa_split_partials(const void *q, const void *k_cache, const void *v_cache,
                       const int32_t *seqlens, const int32_t *page_table, float *out,
                       const gqa_dims *dims, float scale, uint32_t *status,
                       int32_t split_tokens, int32_t max_seqlen, void *workspace,
                       size_t workspace_bytes, void *stream);

int gqa_split_combine(const int32_t *seqlens, float *out, const gqa_dims *dims,
                      uint32_t *status, int32_t split_tokens, int32_t max_seqlen,
                      const void *workspace, size_t workspace_bytes, void *stream);

/*
 * gqa_decode_split_lse -- gqa_decode_split that also returns, for every output
 * row (s, i), the natural-log sum of the row's exponentials,
 *     lse[s*H + i] = ln sum_{j < len_s} exp(scale * q[s,i] . K[s,g(i),j]),
 * and accepts seqlens[s] == 0 as an empty sequence (its rows are zero with
 * lse = -inf, and no status bit is set).  This is the per-shard half of
 * sequence-parallel decode: when the tokens of each sequence are spread over
 * several GPUs (each holding its own pool, page table and lengths for its
 * share), every GPU runs this call on its share, the (out, lse) pairs are
 * gathered, and gqa_merge_lse combines them.  The result equals attention over
 * the whole sequence (an exact re-association of the softmax of the pages'
 * formula).  lse: fp32 [b, H] device memory, 4-byte aligned, not NULL.
 * Everything else as gqa_decode_split.
 */
int gqa_decode_split_lse(const void *q, const void *k_cache, const void *v_cache,
                         const int32_t *seqlens, const int32_t *page_table, float *out, float *lse,
                         const gqa_dims *dims, float scale, uint32_t *status,
                         int32_t split_tokens, int32_t max_seqlen, void *workspace,
                         size_t workspace_bytes, void *stream);

/*
 * gqa_decode_verify -- decode of n_query new tokens per sequence at once, as
 * when a target model verifies the draft tokens of speculative decoding.  The
 * drafts are already in the cache (seqlens[s] counts them); query token t of
 * sequence s attends the cached positions before it and itself,
 *     j < seqlens[s] - (n_query - 1 - t),
 * the end-aligned mask of a causal decoder.  For each KV group, the n_query * r
 * (token, head) pairs form the group's rows and share each K/V tile read from
 * HBM: with up to 16 rows per group (the mma.sync kernel), or up to 128 at
 * d = 128 and 64 at d = 64 (the tcgen05 kernel, taken by itself above
 * GQA_TC_AUTO_ROWS rows), the cache is read once per step for all drafts;
 * with more rows, the mma.sync kernel reads it once per 16-row slice.
 *
 * q: bf16 [b, n_query, H, d]; out: fp32 [b, n_query, H, d]; lse: fp32
 * [b, n_query, H] or NULL (the natural-log normaliser of each row, as in
 * gqa_decode_split_lse).  1 <= n_query <= 64.  A length below n_query is
 * invalid (GQA_STATUS_BAD_SEQLEN, rows zeroed).  The workspace comes from
 * gqa_decode_verify_workspace_size for the same dims, n_query, max_seqlen
 * and split_tokens; everything else as gqa_decode_split (the CUDA-core
 * contraction flag needs n_query == 1).  n_query == 1 is gqa_decode_split.
 */
size_t gqa_decode_verify_workspace_size(const gqa_dims *dims, int32_t n_query, int32_t max_seqlen,
                                        int32_t split_tokens);

int gqa_decode_verify(const void *q, const void *k_cache, const void *v_cache,
                      const int32_t *seqlens, const int32_t *page_table, float *out, float *lse,
                      const gqa_dims *dims, int32_t n_query, float scale, uint32_t *status,
                      int32_t split_tokens, int32_t max_seqlen, void *workspace,
                      size_t workspace_bytes, void *stream);

/*
 * gqa_decode_split_mapped -- gqa_decode_split with the KV group of every query
 * head taken from a table, g(i) = group_of_head[i], instead of i / (H/G):
 * groups may have unequal sizes or no head at all, and num_heads need not be
 * a multiple of num_kv_heads (the non-uniform grouping of "Beyond Uniform
 * Query Distribution: Key-Driven Grouped Query Attention", Figure 1, with the
 * map given at inference).  Each group's K/V is still read once and shared by
 * its heads on chip.
 *
 * group_of_head: HOST memory, num_heads int32 entries in [0, num_kv_heads)
 * (else GQA_ERR_HEADS); num_heads <= 256, num_kv_heads <= 256.  The map is
 * read during the call only.  lse: fp32 [b, H] or NULL, as in
 * gqa_decode_split_lse.  split_tokens = 0: the library picks the
 * decomposition as for gqa_decode_split (gqa_plan_decomposition_ex with the
 * same map tells which); the workspace comes from
 * gqa_decode_split_mapped_workspace_size with the same arguments.  The
 * CUDA-core contraction flag is not available with a map.  A map
 * g(i) = i / (H/G) gives exactly gqa_decode_split's result.
 */
size_t gqa_decode_split_mapped_workspace_size(const gqa_dims *dims, const int32_t *group_of_head,
                                              int32_t max_seqlen, int32_t split_tokens);

int gqa_decode_split_mapped(const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *seqlens, const int32_t *page_table, float *out, float *lse,
                            const gqa_dims *dims, const int32_t *group_of_head, float scale,
                            uint32_t *status, int32_t split_tokens, int32_t max_seqlen, void *workspace,
                            size_t workspace_bytes, void *stream);

/*
 * gqa_merge_lse -- merges n_parts normalised partial results of the same rows,
 * each weighted by its log-sum-exp:
 *     LSE = ln sum_k exp(lse_k),   out = sum_k exp(lse_k - LSE) o_k.
 * o_parts: fp32 [n_parts][rows][head_dim], 16-byte aligned (part-major, the
 * layout an all-gather of [rows][head_dim] per part produces); lse_parts: fp32
 * [n_parts][rows]; out: fp32 [rows][head_dim], 16-byte aligned; lse_out: fp32
 * [rows] or NULL.  Parts with lse = -inf contribute nothing; a row with no
 * non-empty part is zero with LSE -inf.  head_dim: 64 or 128.  The parts are
 * taken in ascending order, so the result is deterministic.  Asynchronous on
 * `stream`; GQA_OK or a GQA_ERR_* code (nothing launched on error).
 */
int gqa_merge_lse(const float *o_parts, const float *lse_parts, int32_t n_parts, int64_t rows,
                  int32_t head_dim, float *out, float *lse_out, void *stream);

/*
 * The decomposition the pair gqa_split_partials / gqa_split_combine uses
 * when split_tokens == 0 (and gqa_decode_split, unless gqa_plan_decomposition
 * says GQA_PLAN_CLUSTERS): 0 for equal-work ranges, or the fixed split length
 * (a positive multiple of 128) it falls back to.  num_sms <= 0 queries the
 * current device.  A negative value is a GQA_ERR_* code.
 */
int32_t gqa_plan_split_tokens(const gqa_dims *dims, int32_t max_seqlen, int32_t num_sms);

/*
 * The decomposition gqa_decode_split (and gqa_decode_split_lse) runs with
 * split_tokens == 0, one query token per sequence and no group table
 * (gqa_plan_decomposition_ex: with them):
 *   GQA_PLAN_EQUAL_WORK    equal-work ranges + combine kernel (paged dims);
 *   GQA_PLAN_FIXED_SPLITS  fixed splits of *split_tokens_out tokens, merged in
 *                          the decode kernel (<= 8 splits) or by the combine;
 *   GQA_PLAN_CLUSTERS      a contiguous cache with too few (sequence, group)
 *                          units to fill the GPU one block each: the cluster
 *                          decomposition of gqa_decode, *cluster_out blocks per
 *                          thread-block cluster (<= 8) sharing each unit's
 *                          tokens and merging through distributed shared
 *                          memory, one kernel and no workspace (the workspace
 *                          passed is not touched); taken only when every
 *                          cluster of the grid is resident at once on the
 *                          device (clusters sit inside one GPC), else the
 *                          fixed splits.
 * split_tokens_out / cluster_out may be NULL.  num_sms <= 0 queries the
 * current device (its cluster occupancy included); num_sms > 0 plans for a
 * device of that many SMs without asking it.  A negative value is a GQA_ERR_*
 * code.
 */
#define GQA_PLAN_EQUAL_WORK 0
#define GQA_PLAN_FIXED_SPLITS 1
#define GQA_PLAN_CLUSTERS 2
int32_t gqa_plan_decomposition(const gqa_dims *dims, int32_t max_seqlen, int32_t num_sms,
                               int32_t *split_tokens_out, int32_t *cluster_out);

/*
 * gqa_plan_decomposition for a call with num_query_tokens query tokens per
 * sequence (gqa_decode_verify; >= 1, else GQA_ERR_DIMS) and, with one query
 * token, an optional HOST group table (gqa_decode_split_mapped, NULL for the
 * uniform grouping; checked as there).  Clusters are planned for the mma.sync
 * contraction only: with more than GQA_TC_AUTO_ROWS rows per group (or the
 * tcgen05 or CUDA-core flag in dims->flags) the plan is fixed splits or
 * equal-work ranges.  The same results and errors otherwise.
 */
int32_t gqa_plan_decomposition_ex(const gqa_dims *dims, int32_t max_seqlen, int32_t num_query_tokens,
                                  const int32_t *group_of_head, int32_t num_sms, int32_t *split_tokens_out,
                                  int32_t *cluster_out);

/*
 * gqa_decode_split_static -- gqa_decode_split without a caller-provided
 * workspace, for callers that may not allocate device memory while they
 * decode (a process whose HBM is handed out by another memory manager, or a
 * latency-critical loop that must stay out of the CUDA allocator).  The pages
 * this library follows have no counterpart of it: it only moves the scratch.
 *
 * Same arguments and results as gqa_decode_split, minus workspace and
 * workspace_bytes.  The scratch is a fixed array of GQA_STATIC_WORKSPACE_BYTES
 * in the library's device module; each GPU that loads the library holds it
 * until the process exits.  Problems whose gqa_decode_split_workspace_size()
 * exceeds that size are rejected with GQA_ERR_WORKSPACE before anything runs.
 * Argument errors take precedence over GQA_ERR_WORKSPACE, in the order
 * gqa_decode_split checks them.  The first call on a device looks up the
 * array's device address (a CUDA runtime call, no allocation) and caches it
 * for the life of the process; make that first call before any stream
 * capture, and do not use the library across cudaDeviceReset (the cached
 * address would be stale).  All calls share the array: calls whose kernels
 * overlap on the GPU (different streams or host threads) race on it.  Nothing
 * in it needs to start at zero.  No cudaMalloc, cudaFree or other allocating
 * routine is called.
 */
#define GQA_STATIC_WORKSPACE_BYTES (8u << 20)

int gqa_decode_split_static(const void *q, const void *k_cache, const void *v_cache,
                            const int32_t *seqlens, const int32_t *page_table, float *out,
                            const gqa_dims *dims, float scale, uint32_t *status,
                            int32_t split_tokens, int32_t max_seqlen, void *stream);

/* A static, human-readable name for a GQA_OK / GQA_ERR_* code. */
const char *gqa_status_string(int code);

/* ABI version of this header: (major << 16) | minor. */
int32_t gqa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GQA_H */
