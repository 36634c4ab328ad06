/*
 * attn.h - C ABI of the B200 (sm_100a) masked attention forward.
 *
 * Computes, for every sequence b of a ragged batch, every query head h and every
 * query row i,
 *
 *     out[i, h, :] = softmax_j( scale * q[i, h, :] . k[j, h / g, :]  +  mask[i, j] ) . v[j, h / g, :]
 *     lse[i, h]    = ln sum_{j visible} exp( scale * q[i, h, :] . k[j, h / g, :] )
 *
 * with g = hq / hkv (grouped-query attention) and mask[i, j] in {0, -inf}. A row
 * that sees no key gets out = 0 and lse = -inf. The masks are the kinds defined on:
 *   - "feat: support custom mask for flash attention" (sglang-jax PR #20), Highlights:
 *     ragged, paged attention with an optional custom mask or a causal flag;
 *   - "[Attention] feat: support PrefixLM" (aphrodite-engine #1526), Highlights:
 *     PrefixLM mask (bidirectional prefix, causal suffix) and prefix_len;
 *   - "Custom mask slows down attention." (flashinfer #724): bit-packed custom masks;
 *   - "Feature request: chunk-causal mask type for Flex Flash Attention" (MagiAttention
 *     #316), Current pattern / Desired representation / Proposed API: q/k range lists,
 *     attn_type_map, chunk-causal ranges with a chunk size;
 *   - "feat: add Gemma2 sliding-window (local/global) attention" (mlxcel PR #555),
 *     Summary: local mask = causal AND within the window.
 *
 * Coordinates. L_q and L_k are the query and key lengths of one sequence. Query row i
 * (0-based inside its sequence) sits at key position pos(i) = i + L_k - L_q, i.e. the
 * queries are the last L_q tokens of the sequence. All ranges are half-open.
 *
 * Usage. attn_plan() validates the problem and the mask descriptor, classifies every
 * 128 x 128 (query, key) tile as empty, full or partial, writes the tile-transposed
 * masks of the partial tiles and a balanced work list into a device workspace that the
 * plan owns. attn_masked_fwd() then runs the forward on a stream; it allocates nothing
 * and may be called any number of times with the same plan (e.g. the same lengths and
 * mask for every layer). attn_plan_destroy() frees the plan. Beyond that:
 *   - split-KV (attn_problem_t.kv_splits): few long work items are cut into key ranges
 *     whose partial results a second kernel merges;
 *   - query-row shards (attn_problem_t.q_begin / q_end): one long sequence over several
 *     GPUs, each computing its rows against all (all-gathered) keys;
 *   - attn_plan_bwd() + attn_masked_bwd(): dq, dk, dv;
 *   - attn_fp8_transpose_v() + attn_masked_fwd_fp8(): the forward on e4m3 inputs;
 *   - attn_plan_dry_run() / attn_plan_bwd_dry_run(): the forward / backward plan
 *     statistics on the host, without a GPU;
 *   - attn_masked_fwd_noalloc(): plan + forward without any device allocation.
 *
 * Errors. Every call returns an attn_status_t; nothing is thrown across the ABI and
 * nothing exits the process. attn_status_string() names a status.
 */
#ifndef MASKED_ATTN_B200_ATTN_H
#define MASKED_ATTN_B200_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t. NULL is the legacy default stream. */
typedef struct CUstream_st* attn_stream_t;

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,    /* a null pointer, a negative or inconsistent size, a bad range */
  ATTN_ERR_UNSUPPORTED = 2,    /* head_dim not in {64, 128, 256}, page_size not in {16, 32, 64, 128} */
  ATTN_ERR_MASK_TOO_SMALL = 3, /* CUSTOM: the packed mask holds fewer words than the lengths need */
  ATTN_ERR_OOM = 4,            /* cudaMalloc of the plan workspace failed */
  ATTN_ERR_CUDA = 5,           /* any other CUDA runtime error (launch, copy, no device) */
  ATTN_ERR_TIMEOUT = 6,        /* a bounded wait inside the kernel expired (see attn_plan_check_status) */
  ATTN_ERR_TOO_LARGE = 7       /* attn_masked_fwd_noalloc: the work list and masks exceed its fixed scratch */
} attn_status_t;

typedef enum {
  ATTN_MASK_FULL = 0,           /* every key */
  ATTN_MASK_CAUSAL = 1,         /* j <= pos(i) */
  ATTN_MASK_SLIDING_WINDOW = 2, /* j <= pos(i) and pos(i) - j < window */
  ATTN_MASK_PREFIX_LM = 3,      /* j < prefix_len  or  j <= pos(i) */
  ATTN_MASK_CHUNK_CAUSAL = 4,   /* CAUSAL range over [0, chunk.q_start) plus the chunk-causal range `chunk` */
  ATTN_MASK_RANGES = 5,         /* union of typed (q_range, k_range) pairs, per sequence */
  ATTN_MASK_CUSTOM = 6,         /* bit-packed boolean mask, per sequence, shared by all heads */
  ATTN_MASK_BLOCK_SPARSE = 7    /* block-sparse (BSR) mask: listed (block_q x block_k) blocks are visible */
} attn_mask_kind_t;

/* Range types. 0-3 are the attn_type_map values FULL, CAUSAL, INV_CAUSAL and BI_CAUSAL
 * printed on the chunk-causal feature request (Why existing mask types are not enough:
 * BI_CAUSAL is an "aligned band/intersection"); 4 is this library's code for CHUNK_CAUSAL. */
typedef enum {
  ATTN_RANGE_FULL = 0,          /* every (i, j) in q_range x k_range */
  ATTN_RANGE_CAUSAL = 1,        /* and j <= i, both in sequence-local coordinates */
  ATTN_RANGE_INV_CAUSAL = 2,    /* and j - k_start >= i - q_start (triangle aligned to the top-left corner) */
  ATTN_RANGE_BI_CAUSAL = 3,     /* INV_CAUSAL and j - k_end <= i - q_end (the band between the
                                   top-left and bottom-right aligned diagonals) */
  ATTN_RANGE_CHUNK_CAUSAL = 4   /* query chunk c = (i - q_start) / chunk_size sees keys
                                   [k_start, min(q_start + (c+1)*chunk_size, q_end)) within k_range */
} attn_range_type_t;

/* One (q_range, k_range) pair in sequence-local coordinates, half-open.
 * 0 <= q_start <= q_end <= L_q, 0 <= k_start <= k_end <= L_k; chunk_size >= 1 for
 * CHUNK_CAUSAL (ignored otherwise). Overlapping pairs are OR-ed. */
typedef struct {
  int32_t q_start, q_end, k_start, k_end, type, chunk_size;
} attn_range_t;

/* Mask descriptor. Only the fields of `kind` are read. */
typedef struct {
  int32_t kind;                     /* attn_mask_kind_t */
  int32_t window;                   /* SLIDING_WINDOW: >= 1 (keys including the query's own position) */
  int32_t prefix_len;               /* PREFIX_LM when prefix_lens is NULL: >= 0 */
  const int32_t* prefix_lens;       /* PREFIX_LM: host [batch] per-sequence prefix lengths, or NULL */
  attn_range_t chunk;               /* CHUNK_CAUSAL: the chunk-causal range, the same for every
                                       sequence; rows and keys past a sequence's end are dropped,
                                       the chunk arithmetic uses the values as given */
  const attn_range_t* ranges;       /* RANGES: host, all sequences' ranges concatenated */
  const int32_t* cu_ranges;         /* RANGES: host [batch+1]; sequence b owns ranges[cu_ranges[b] .. cu_ranges[b+1]) */
  const uint32_t* mask_bits;        /* CUSTOM: DEVICE pointer. Sequence b's mask starts at word
                                       mask_word_offsets[b] and is row-major [L_q][W], W = ceil(L_k/32);
                                       key j of row i is bit (j % 32) of word i*W + j/32, least
                                       significant bit first. Bits past L_k are ignored. */
  const int64_t* mask_word_offsets; /* CUSTOM: host [batch+1] word offsets (non-decreasing) */
  int64_t mask_words_total;         /* CUSTOM: number of readable words at mask_bits */
  int32_t block_q, block_k;         /* BLOCK_SPARSE: block height (query rows) and width (keys), >= 1 */
  const int32_t* bsr_row_ptr;       /* BLOCK_SPARSE: host CSR row pointer over the block rows of all
                                       sequences in order (sequence b has ceil(L_q / block_q) block
                                       rows); length = total block rows + 1, starting at 0 */
  const int32_t* bsr_col_idx;       /* BLOCK_SPARSE: host block-column indices (sequence-local, in
                                       [0, ceil(L_k / block_k))); query i, key j is visible iff
                                       block (i / block_q, j / block_k) is listed ("Custom mask slows
                                       down attention.": the sparse API, equivalent to a custom mask) */
} attn_mask_desc_t;

/* Problem shape. Host arrays are read during attn_plan() only. */
typedef struct {
  int32_t batch;                    /* number of sequences, >= 0 */
  int32_t hq, hkv;                  /* query / key-value heads, hq % hkv == 0 */
  int32_t head_dim;                 /* 64, 128 or 256 (the value head dim is the same) */
  float scale;                      /* softmax scale; <= 0 selects 1/sqrt(head_dim) */
  const int32_t* cu_seqlens_q;      /* host [batch+1] query token offsets (non-decreasing, from 0) */
  const int32_t* cu_seqlens_k;      /* host [batch+1] key token offsets; contiguous K/V only, else NULL */
  const int32_t* kv_lens;           /* host [batch] key lengths; paged K/V only, else NULL */
  const int32_t* page_table;        /* DEVICE int32 [batch][max_pages_per_seq]; paged only. Entry p of
                                       row b holds the cache page of keys [p*page_size, (p+1)*page_size).
                                       Entries outside [0, num_pages) read as zeros. Must stay valid
                                       while forwards that use the plan run. */
  int32_t page_size;                /* paged: 16, 32, 64 or 128 */
  int32_t max_pages_per_seq;        /* paged: row length of page_table */
  int32_t num_pages;                /* paged: pages in the K and V caches */
  int32_t kv_splits;                /* split-KV: 0 = automatic, 1 = never split, N >= 2 = split a work
                                       item's key tiles into at most N ranges. A split item writes
                                       fp32 partial results (out / l and lse per range) into the plan
                                       workspace and a second kernel merges them by their lse:
                                       lse = ln sum_r exp(lse_r), out = sum_r exp(lse_r - lse) out_r.
                                       Automatic splits only when the longest item exceeds 1.5x the
                                       per-CTA share of the work (few long items: short queries over
                                       long keys, the tree-verify case of "Custom mask slows down
                                       attention."). Must be >= 0. */
  int32_t q_begin, q_end;           /* query-row shard: this plan computes only the 128 / heads_per_tile row
                                       blocks of every sequence that overlap sequence-local rows
                                       [q_begin, q_end) (q_end <= 0: to the end). Rows of those blocks are
                                       written in full; other rows are left untouched. Masks keep their
                                       sequence-local row indices. For one long sequence split over GPUs:
                                       every rank holds all K/V (one all-gather) and its query rows.
                                       0 / 0 = all rows. */
} attn_problem_t;

typedef struct attn_plan attn_plan_t; /* opaque */

typedef struct {
  int64_t unmasked_pairs;           /* visible (i, j) pairs summed over sequences, for ONE head */
  int64_t tiles_empty, tiles_full, tiles_partial; /* 128 x 128 tile classes over valid rectangles */
  int64_t mask_tiles;               /* 2 KiB tile-transposed mask tiles the forward reads */
  int64_t work_items, jobs;         /* forward work list: items and (item, key tile) jobs */
  int64_t mask_tile_reads;          /* 2 KiB mask tiles one forward reads (per query tile and job) */
  int32_t ctas;                     /* persistent CTAs the forward launches */
  int32_t heads_per_tile;           /* query heads packed into one 128-row tile (short queries) */
  int32_t tiles_per_cta;            /* 128-row query tiles one CTA works on at once (1 or 2) */
  int32_t cluster_size;             /* CTAs that cooperate on one work item (2: a pair of SMs) */
  int32_t kv_splits_max;            /* largest number of key ranges any query tile was split into (1: none) */
  int32_t merge_tiles;              /* 128-row query tiles whose partial results the merge kernel combines */
  int64_t vt_keys;                  /* contiguous K/V: columns of the transposed V that attn_fp8_transpose_v
                                       writes (each sequence starts at a multiple of 128); 0 if paged */
  int64_t workspace_bytes;          /* device workspace of the forward plan: work list, mask tiles, split-KV
                                       slots (attn_plan_bwd allocates the backward's on top) */
} attn_plan_stats_t;

/* Validate and plan. `stream` orders the plan's device work (the CUSTOM mask scan and
 * the uploads); attn_plan returns after that work has finished. On success *out_plan
 * owns a device workspace. Errors: INVALID_ARG, UNSUPPORTED, MASK_TOO_SMALL, OOM, CUDA.
 * Defined by the pages listed at the top of this file; the validation rules follow the
 * custom_mask review comments of "feat: support custom mask for flash attention"
 * (conflicting options rejected; a custom mask shorter than the lengths need rejected). */
attn_status_t attn_plan(const attn_problem_t* problem, const attn_mask_desc_t* mask,
                        attn_stream_t stream, attn_plan_t** out_plan);

/* Run the forward asynchronously on `stream`. All pointers are DEVICE pointers,
 * 16-byte aligned, and must stay valid until the stream work completes:
 *   q   bf16 [total_q][hq][head_dim]             (total_q = cu_seqlens_q[batch])
 *   k,v bf16 [total_k][hkv][head_dim]            contiguous (total_k = cu_seqlens_k[batch]), or
 *       bf16 [num_pages][page_size][hkv][head_dim] paged caches
 *   out bf16 [total_q][hq][head_dim]             written for every valid row
 *   lse fp32 [total_q][hq]                       natural log, scale included; may be NULL
 * Runs on the device the plan was made on, which must be the current device.
 * Allocates nothing. Errors: INVALID_ARG (null/misaligned pointer, or another current
 * device), CUDA (launch).
 * Concurrency: the forward only reads the plan, except that a split plan (stats
 * kv_splits_max > 1) keeps the partial results of its key ranges in the plan's workspace.
 * Unsplit plans may therefore serve forwards on several streams at once; forwards of a
 * split plan, and backwards (attn_masked_bwd keeps its per-row dout . out there too), must
 * be ordered one after another (one stream, or events between the streams). */
attn_status_t attn_masked_fwd(const attn_plan_t* plan, const void* q, const void* k, const void* v,
                              void* out, float* lse, attn_stream_t stream);

/* Plan the forward AND the backward pass (gradients of out with respect to q, k, v).
 * Same arguments and errors as attn_plan(); the plan serves attn_masked_fwd() and
 * attn_masked_bwd(). Backward support: head_dim 64, 128 or 256, contiguous K/V, or a paged
 * cache when no cache page is read by two sequences (its gradient would be the sum of both;
 * the page table is copied to the host to check, else UNSUPPORTED). It adds a second device workspace: the dQ and dK/dV work lists over
 * 128 x 128 tiles of one head, the partial-tile masks in query-major and key-major form,
 * and an fp32 [total_q][hq] buffer for the row terms dout . out. */
attn_status_t attn_plan_bwd(const attn_problem_t* problem, const attn_mask_desc_t* mask,
                            attn_stream_t stream, attn_plan_t** out_plan);

/* Backward of attn_masked_fwd for a loss with gradient dout on out and, optionally, dlse on
 * lse (d lse_i / d s_ij = p_ij):
 *     dv_j = sum_i p_ij dout_i,  ds_ij = p_ij (dout_i . v_j - dout_i . out_i + dlse_i),
 *     dq_i = scale sum_j ds_ij k_j,  dk_j = scale sum_i ds_ij q_i,
 * p_ij = exp(scale q_i . k_j - lse_i) on visible pairs; dk, dv of a key/value head sum over
 * its query heads. Asynchronous on `stream`; all DEVICE pointers, 16-byte aligned:
 *   q, out, dout  bf16 [total_q][hq][head_dim]; lse fp32 [total_q][hq] as attn_masked_fwd wrote it
 *   dlse          fp32 [total_q][hq], or NULL (no gradient on lse)
 *   k, v          bf16 [total_k][hkv][head_dim], or the paged caches [num_pages][page_size][hkv][head_dim]
 *   dq            bf16 [total_q][hq][head_dim]  (0 on rows that see no key)
 *   dk, dv        bf16 shaped like k / v (0 on keys that no query sees; paged: 0 on every
 *                 cache row that no sequence reads, the whole cache is written)
 * The plan must come from attn_plan_bwd(). Allocates nothing. Errors: INVALID_ARG (plan
 * without backward lists, null or misaligned pointer, another current device than the
 * plan's), CUDA. */
attn_status_t attn_masked_bwd(const attn_plan_t* plan, const void* q, const void* k, const void* v,
                              const void* out, const float* lse, const void* dout, const float* dlse, void* dq,
                              void* dk, void* dv, attn_stream_t stream);

/* e4m3 (fp8) forward. No page names a layout for it; "Custom mask slows down attention."
 * asks whether the custom-mask path supports fp8. Inputs are e4m3 bytes (1 sign, 4
 * exponent bits with bias 7, 3 mantissa bits; no infinities) with per-tensor scales:
 * the real values are q_scale * q8, k_scale * k8, v_scale * v8. The scores
 * scale * q_scale * k_scale * (q8 . k8) are exact in fp32; P is rounded to e4m3 for the
 * P V product (the row sums use P before rounding); out (bf16) and lse (fp32) as in
 * attn_masked_fwd.
 *   q   bytes [total_q][hq][d]          k bytes [total_k][hkv][d]      (d = head_dim)
 *   vt  bytes [hkv][d][ldv]             V transposed per head by attn_fp8_transpose_v
 *   ldv >= stats.vt_keys, a multiple of 16
 * head_dim 128 (single-SM kernel) or 256 (2-SM kernel) and contiguous K/V only (else
 * UNSUPPORTED); the plan is an ordinary attn_plan() (split-KV applies). Pointers 16-byte aligned (lse: 4-byte, may be NULL).
 * Allocates nothing. Errors: INVALID_ARG (as attn_masked_fwd, or ldv / a scale out of
 * range), UNSUPPORTED, CUDA. */
attn_status_t attn_masked_fwd_fp8(const attn_plan_t* plan, const void* q, const void* k, const void* vt,
                                  int64_t ldv, float q_scale, float k_scale, float v_scale, void* out,
                                  float* lse, attn_stream_t stream);

/* V bytes [total_k][hkv][head_dim] -> vt [hkv][head_dim][ldv]: sequence b's keys go to
 * columns from the sum over earlier sequences of their key counts rounded up to 128, the
 * gaps are zero. ldv >= stats.vt_keys and a multiple of 16. Asynchronous on `stream`.
 * Errors: INVALID_ARG (paged plan, null pointer, ldv, another current device than the
 * plan's), UNSUPPORTED (head_dim % 32), CUDA. */
attn_status_t attn_fp8_transpose_v(const attn_plan_t* plan, const void* v, void* vt, int64_t ldv,
                                   attn_stream_t stream);

/* Copy the 128 x 128 tile classes (0 empty, 1 full, 2 partial) in the order sequence,
 * query tile, key tile (row-major) into host_dst[0 .. n). *n_needed (may be NULL)
 * receives the total count; a short buffer gets a prefix. */
attn_status_t attn_plan_get_tile_classes(const attn_plan_t* plan, uint8_t* host_dst, size_t n,
                                         size_t* n_needed);

/* Plan statistics (host memory). */
attn_status_t attn_plan_get_stats(const attn_plan_t* plan, attn_plan_stats_t* stats);

/* Synchronise `stream`, then read and clear the plan's device status word. Returns
 * ATTN_ERR_TIMEOUT if a bounded wait of an earlier forward expired (its output is then
 * undefined), ATTN_ERR_CUDA on a CUDA error, else ATTN_OK. */
attn_status_t attn_plan_check_status(const attn_plan_t* plan, attn_stream_t stream);

/* Testing hook for the failure path: flags bit 0 makes the next forwards skip the
 * arrival that publishes the first query tile, so that a bounded wait expires and the
 * kernel returns through its abort path; timeout_ns (> 0) sets the per-wait limit
 * (default 2 s). 0 / 0 restores the defaults. */
attn_status_t attn_plan_set_debug(attn_plan_t* plan, int32_t flags, int64_t timeout_ns);

/* Free the plan and its device workspace (after the forwards that use it finished).
 * The workspace is freed with cudaFree, which waits for the work in flight on the device;
 * attn_plan() likewise allocates with cudaMalloc and waits for `stream`. A runtime that
 * re-plans every step beside other streams' kernels keeps plans alive across steps or
 * uses attn_masked_fwd_noalloc(), which allocates and frees nothing. */
attn_status_t attn_plan_destroy(attn_plan_t* plan);

/* Host-only classification for the analytic kinds (everything but CUSTOM): the same
 * validation and 128 x 128 tile classes as attn_plan, without any CUDA call (the device
 * page_table pointer may be NULL here). classes
 * may be NULL to query *n_needed; *unmasked_pairs (may be NULL) receives the per-head
 * visible pair count. CUSTOM returns UNSUPPORTED (its bits live on the device). */
attn_status_t attn_classify_host(const attn_problem_t* problem, const attn_mask_desc_t* mask,
                                 uint8_t* classes, size_t n, size_t* n_needed,
                                 int64_t* unmasked_pairs);

/* Host-only dry run of attn_plan() for the analytic kinds (everything but CUSTOM): the
 * same validation, tile classes, work list and split-KV choice for a GPU of `num_sms`
 * SMs, reported as the statistics attn_plan_get_stats() would give; no CUDA call, no
 * device memory (the device page_table pointer may be NULL). Errors: INVALID_ARG
 * (num_sms <= 0 or as attn_plan), UNSUPPORTED (CUSTOM, or as attn_plan), OOM. */
attn_status_t attn_plan_dry_run(const attn_problem_t* problem, const attn_mask_desc_t* mask, int32_t num_sms,
                                attn_plan_stats_t* stats);

/* Statistics of the backward work lists (attn_plan_bwd() builds the same lists over
 * 128 x 128 tiles of one head). */
typedef struct {
  int64_t dq_items, dq_jobs;        /* dQ items (query tile, query head) and the key tiles they run */
  int64_t dkv_items, dkv_jobs;      /* dK/dV items (key tile, KV head) and the (query head, query tile)s they run */
  int64_t mask_tiles;               /* tiles that carry a mask (partial, or cut by the end of the keys or queries) */
  int32_t dq_ctas, dkv_ctas;        /* persistent CTAs of the two kernels */
  int64_t dq_cost, dkv_cost;        /* sum over items of (jobs + 2), the planner's cost unit */
  int64_t dq_max_cta_cost, dkv_max_cta_cost; /* largest per-CTA cost after the longest-first assignment */
  int64_t dq_max_item_cost, dkv_max_item_cost;
} attn_bwd_stats_t;

/* Host-only dry run of attn_plan_bwd() for the analytic kinds: the same validation and
 * backward work lists for a GPU of `num_sms` SMs, with no CUDA call and no device memory.
 * A paged problem's page table is not read (the check that no page is read by two
 * sequences needs it on the device). Errors: INVALID_ARG (num_sms <= 0 or as attn_plan),
 * UNSUPPORTED (CUSTOM, or as attn_plan_bwd), OOM. */
attn_status_t attn_plan_bwd_dry_run(const attn_problem_t* problem, const attn_mask_desc_t* mask, int32_t num_sms,
                                    attn_bwd_stats_t* stats);

const char* attn_status_string(attn_status_t status);

/* Forward for callers that cannot allocate device memory. No page of the masked-attention
 * pages has a counterpart of this call; it exists for embedders such as serving runtimes
 * that own every device allocation through their own pool or are not allowed to call
 * cudaMalloc / cudaFree at run time. It plans and runs in one call, like attn_plan()
 * followed by attn_masked_fwd() and attn_plan_destroy(), but the work list, the partial-
 * tile masks and the status word live in one fixed device array of
 * ATTN_NOALLOC_SCRATCH_BYTES (32 MiB) inside the library, which every GPU that loads the
 * library keeps until the process exits. It calls no cudaMalloc / cudaFree and no other
 * device allocator; the host-side planning uses ordinary host memory.
 *   - Arguments as in attn_plan() and attn_masked_fwd(); mask kinds FULL, CAUSAL,
 *     SLIDING_WINDOW, PREFIX_LM, CHUNK_CAUSAL and RANGES (CUSTOM returns
 *     ATTN_ERR_UNSUPPORTED: its device scan needs a workspace of its own).
 *   - A problem whose plan needs more than the fixed array returns ATTN_ERR_TOO_LARGE
 *     before any device work is enqueued.
 *   - The plan is copied into the array on `stream` and the forward is enqueued behind it;
 *     the call returns once the host copy source has been consumed.
 *   - The first call on a device looks up the array's device address (once per device,
 *     with that device current).
 *   - Every call reuses the same array and overwrites what the previous call left there
 *     (the status word is cleared each time), so calls whose work overlaps on the GPU --
 *     different streams, or another host thread -- race; serialise them on one stream.
 *     Calls queued back to back on one stream are fine: each copy into the array waits
 *     for the previous forward on that stream.
 *   - In-kernel waits are bounded like those of attn_masked_fwd(), but no plan outlives the
 *     call, so an expired wait cannot be queried afterwards. It shows in the output instead:
 *     when lse is given, the call first fills it with NaN (on `stream`, before the forward),
 *     and every row the kernel completes overwrites its lse with a finite value or -inf
 *     (a row that sees no key). A row whose lse is still NaN after the stream has finished
 *     was not computed; its out holds whatever the buffer held. With lse == NULL there is
 *     no such signal.
 * Errors: INVALID_ARG, UNSUPPORTED, TOO_LARGE, CUDA (launch or enqueue failures only). */
#define ATTN_NOALLOC_SCRATCH_BYTES (32u << 20)
attn_status_t attn_masked_fwd_noalloc(const attn_problem_t* problem, const attn_mask_desc_t* mask,
                                      const void* q, const void* k, const void* v, void* out, float* lse,
                                      attn_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MASKED_ATTN_B200_ATTN_H */
