/*
 * kara.h - C ABI of libkara, the sm_100a (B200) implementation of Kara's decode-time
 * sliding-window KV-cache compression and of LaCache's ladder compaction over a paged
 * (PagedAttention-style) KV cache.
 *
 * Sources (web pages; cited by title and section):
 *  [KARA]  "Kara: Efficient Reasoning LLM Serving via Sliding-Window KV Cache Compression",
 *          English abstract and "method details".
 *  [GIST]  gist.science explainer of the same paper (German / Japanese), sections 1
 *          (two-way attention score), 2 (Token2Chunk), 3 (periodic schedule) and results.
 *  [LAC]   "LaCache: Ladder-Shaped KV Caching for Efficient Long-Context Modeling of Large
 *          Language Models" (papercache.org), ladder pattern, hyper-parameters S and O,
 *          iterative compaction.
 *
 * Conventions for every call:
 *  - All tensor arguments are DEVICE pointers unless a comment says "host". The caller owns
 *    every buffer; the library keeps no pointer after a call returns. Nothing here allocates
 *    device memory: scratch space is passed in as `workspace` (size from
 *    kara_workspace_bytes(), 256-byte aligned).
 *  - Every call is asynchronous on `stream` (a cudaStream_t; 0 = legacy default stream) and
 *    returns after enqueueing its kernels, on the current CUDA device.
 *  - Calls run on the current CUDA device. The library sets its kernels' shared-memory limits
 *    and measures their occupancy once per device, the first time a call runs there; devices
 *    with ordinals 0 .. 63 are supported (a higher ordinal gives KARA_ERR_CUDA).
 *  - The return value reports what the host can check: argument shapes, alignment (16-byte
 *    aligned tensors), supported sizes, workspace size, and CUDA launch errors
 *    (KARA_ERR_CUDA). On any non-OK return nothing was enqueued.
 *  - Errors found on the device (a context shorter than the window, a block id out of range,
 *    too few free blocks, a bounded wait that ran out) are written to `dev_status`, one int32
 *    in device memory: the first error wins (later ones do not overwrite it) and the library
 *    never clears it. Read it after synchronising the stream. A call that finds such an error
 *    leaves its outputs in the state documented per call and never traps or faults.
 *  - Layout of the paged cache (one pool per layer, all layers share one block table):
 *      K, V:         bf16 [num_blocks, page_size, num_kv_heads, head_dim]
 *      block_table:  int32 [batch, max_blocks_per_seq]; entry p of row b is the block that
 *                    holds slots [16p, 16p+16) of sequence b, -1 for none
 *      ctx_len:      int32 [batch], number of cached slots of each sequence
 *      free_list:    int32 [num_blocks], a stack of free block ids; free_top (int32 [1])
 *                    entries are valid, the top is free_list[free_top-1]
 *    page_size must be 16; head_dim 64 or 128; num_q_heads a multiple of num_kv_heads with
 *    at most 8 query heads per KV head. Query head h reads KV head h / (num_q_heads /
 *    num_kv_heads).
 */
#ifndef KARA_H
#define KARA_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum kara_status {
  KARA_OK = 0,
  KARA_ERR_INVALID_ARG = 1,   /* bad shape, size, pointer or parameter combination */
  KARA_ERR_UNSUPPORTED = 2,   /* valid request outside what the library implements */
  KARA_ERR_OUT_OF_BLOCKS = 3, /* free list holds fewer blocks than the compaction needs */
  KARA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
  KARA_ERR_TIMEOUT = 5,       /* a bounded on-device wait ran out (kernel returned early) */
  KARA_ERR_WORKSPACE = 6,     /* workspace missing, too small or misaligned */
  KARA_ERR_BAD_BLOCK = 7      /* a block-table entry out of [0, num_blocks) on the device */
} kara_status;

/* Device pointers of one layer's pools. */
typedef struct kara_layer_kv {
  void* k;   /* bf16 [num_blocks, page_size, num_kv_heads, head_dim] */
  void* v;   /* bf16, same shape */
} kara_layer_kv;

/* The shared paged-cache bookkeeping (host struct holding device pointers). */
typedef struct kara_pool {
  int32_t* block_table;        /* device int32 [batch, max_blocks_per_seq] */
  int32_t* ctx_len;            /* device int32 [batch] */
  int32_t* free_list;          /* device int32 [num_blocks] */
  int32_t* free_top;           /* device int32 [1] */
  int32_t batch;
  int32_t max_blocks_per_seq;
  int32_t num_blocks;
  int32_t page_size;           /* must be 16 */
  int32_t num_kv_heads;
  int32_t head_dim;            /* 64 or 128 */
} kara_pool;

/* LaCache ladder parameters ([LAC] "implementation details and key hyper-parameters"). */
typedef struct kara_lacache_params {
  int32_t span;     /* S: consecutive layers that keep one rung */
  int32_t overlap;  /* O: layers shared by neighbouring rungs; stride S-O divides S and L */
  int32_t rung;     /* slots per rung */
  int32_t budget;   /* slots every layer keeps after compaction */
  int32_t sink;     /* leading slots kept in every layer */
  int32_t recent;   /* trailing slots kept in every layer */
} kara_lacache_params;

/* Aggregations of the window scores for kara_score_ex (the pages name none; the sum is the
 * main reading, the others are the variants it leaves open). */
typedef enum kara_agg {
  KARA_AGG_SUM = 0,    /* sum over the G query heads and the W window queries */
  KARA_AGG_MEAN = 1,   /* that sum divided by G * W */
  KARA_AGG_MAX = 2     /* the largest probability any of those queries gives the key */
} kara_agg;

/* Trims of Token2Chunk's expanded set back to k (the pages leave the trim open): the main
 * reading keeps the k members with the largest (priority, score, -position); the chunk-aware
 * trim first drops whole runs of the set that hold no anchor. */
typedef enum kara_trim {
  KARA_TRIM_TOKEN = 0,
  KARA_TRIM_CHUNK = 1
} kara_trim;

/* Operation ids for kara_workspace_bytes(). */
typedef enum kara_op {
  KARA_OP_SCORE = 1,
  KARA_OP_COMPACT = 2,
  KARA_OP_DECODE = 3,
  KARA_OP_LACACHE = 4
} kara_op;

#define KARA_MAX_LAYERS 128
#define KARA_MAX_WINDOW 4096

/*
 * kara_score - bidirectional attention scoring of the compression window ([KARA] abstract:
 * the KV pairs of the window are scored with attention in both directions and the
 * informative ones kept; [GIST] section 1: a token the current reasoning refers to strongly
 * scores high).
 *
 * For due sequence r (cache row b = seq_ids ? seq_ids[r] : r, n = ctx_len[b]) the window is
 * slots [n-window, n). For KV head g with query heads h = g*G .. g*G+G-1 (G = num_q_heads /
 * num_kv_heads):
 *     scores[r][g][j] = sum_h sum_i softmax_j( q_win[r][i][h] . K[slot n-window+j][g] * scale )
 * over window queries i and keys j, unmasked (every query sees every window key).
 *
 *  q_win      bf16 [num_seqs, window, num_q_heads, head_dim]; q_win[r][i] is the query of
 *             window position i (slot n-window+i), as used by the model's attention.
 *  k_cache    this layer's K pool (layout above).
 *  pool       host pointer; block_table and ctx_len are read, nothing is written.
 *  seq_ids    device int32 [num_seqs] or NULL (row r is cache row r).
 *  window     1 .. KARA_MAX_WINDOW.      scale  usually 1/sqrt(head_dim).
 *  scores     fp32 [num_seqs, num_kv_heads, window] (written).
 *  workspace  >= kara_workspace_bytes(KARA_OP_SCORE, ...): the fused kernel's partial key
 *             sums of items split between two clusters, or the two-pass kernels' per-query
 *             log-sum-exp of every 16-page key chunk of the window.
 *  dev_status device int32: KARA_ERR_INVALID_ARG if n < window or n exceeds the table,
 *             KARA_ERR_BAD_BLOCK for a window block id outside [0, num_blocks),
 *             KARA_ERR_TIMEOUT if a pipeline wait ran out; the scores of such a sequence are
 *             then zero or unspecified.
 * With enough (sequence, KV head) items the call runs a second kernel beside the cluster
 * kernel, on the SMs its clusters leave idle, for the last few items; both are in `stream`
 * and whatever the caller enqueues after the call sees all scores, as usual.
 */
kara_status kara_score(const void* q_win, const void* k_cache, const kara_pool* pool,
                       const int32_t* seq_ids, int32_t num_seqs, int32_t window,
                       int32_t num_q_heads, float scale, float* scores, void* workspace,
                       size_t workspace_bytes, int32_t* dev_status, cudaStream_t stream);

/*
 * kara_score_ex - kara_score (q_is_ring == 0: q is q_win [R, W, Hq, d]) or kara_score_ring
 * (q_is_ring != 0: q is the window-query ring [batch, 2W, Hq, d]) with the aggregation `agg`
 * (kara_agg). Sum and mean run the fused kernel for windows of up to 1024 keys and of 2048
 * (the latter on a cluster of 16 CTAs, where the device holds one); the max runs it for
 * windows of up to 1024 keys with head_dim 128; the other cases run the two-pass kernels.
 * Other arguments, output and errors as kara_score; an unknown agg is KARA_ERR_INVALID_ARG.
 */
kara_status kara_score_ex(const void* q, int32_t q_is_ring, const void* k_cache,
                          const kara_pool* pool, const int32_t* seq_ids, int32_t num_seqs,
                          int32_t window, int32_t num_q_heads, float scale, int32_t agg,
                          float* scores, void* workspace, size_t workspace_bytes,
                          int32_t* dev_status, cudaStream_t stream);

/*
 * kara_sum_heads / kara_expand_keep - a selection shared by the KV heads of a layer (a
 * variant the pages leave open): out[r][j] = sum over g of scores[r][g][j] (heads added in
 * ascending order), fp32 [rows, window]; kara_select and kara_token2chunk then run once per
 * row on it, and kara_expand_keep copies each row's keep [rows, k] to every head:
 * keep[r][g][t] = keep_shared[r][t], int32 [rows, num_kv_heads, k], ready for kara_compact.
 */
kara_status kara_sum_heads(const float* scores, int32_t rows, int32_t num_kv_heads,
                           int32_t window, float* out, cudaStream_t stream);
kara_status kara_expand_keep(const int32_t* keep_shared, int32_t rows, int32_t num_kv_heads,
                             int32_t k, int32_t* keep, cudaStream_t stream);

/*
 * kara_select - keep the k highest-scoring window positions ([KARA] abstract: the informative
 * KV pairs of the window are selected; [GIST] results: about 20 % kept).
 *
 * For each of `rows` rows of scores [rows, window]: the k positions with the largest score,
 * ties broken towards the lower position, written ascending to sel [rows, k] (int32).
 * -0.0 and +0.0 compare equal; NaN scores are not supported. 1 <= k <= window <=
 * KARA_MAX_WINDOW.
 */
kara_status kara_select(const float* scores, int32_t rows, int32_t window, int32_t k,
                        int32_t* sel, cudaStream_t stream);

/*
 * kara_token2chunk - expand part of the selection into flexible-length chunks and trim back
 * to budget ([KARA] abstract: a Token2Chunk module grows some of the selected KV pairs into
 * chunks; [GIST] section 2: the span between two important points is kept as one chunk).
 *
 * Per row, in window positions: anchors = the num_anchors = ceil(anchor_frac * k) selected
 * positions with the largest scores (ties: lower position; the product is rounded to 6
 * decimals before the ceiling, so that a float fraction such as 0.2f counts as 0.2); every
 * position strictly between two consecutive anchors is
 * added when there are 1..gap_limit of them; every position within `widen` of an anchor is
 * added; the union U (which contains sel) is trimmed to the k members with the largest
 * (priority, score, -position), priority 2 = anchor, 1 = in a run of consecutive U positions
 * that contains an anchor, 0 = other. keep [rows, k] is written ascending.
 *  scores fp32 [rows, window]; sel int32 [rows, k] ascending (as from kara_select).
 *  0 <= anchor_frac <= 1 (the step workload: 0.5), gap_limit >= 0, widen >= 0; otherwise
 *  KARA_ERR_INVALID_ARG.
 */
kara_status kara_token2chunk(const float* scores, const int32_t* sel, int32_t rows,
                             int32_t window, int32_t k, float anchor_frac, int32_t gap_limit,
                             int32_t widen, int32_t* keep, cudaStream_t stream);

/*
 * kara_select_chunks - kara_select and kara_token2chunk in one kernel per row: the selection
 * stays in shared memory and one launch replaces two. keep as kara_token2chunk of
 * kara_select's output, bit for bit. sel may be NULL; otherwise
 * the selection is written there too. Arguments and limits as the two calls.
 */
kara_status kara_select_chunks(const float* scores, int32_t rows, int32_t window, int32_t k,
                               float anchor_frac, int32_t gap_limit, int32_t widen,
                               int32_t* sel, int32_t* keep, cudaStream_t stream);

/*
 * kara_token2chunk_ex / kara_select_chunks_ex - kara_token2chunk / kara_select_chunks with a
 * choice of trim (kara_trim; the pages leave the trim open). KARA_TRIM_TOKEN gives the same
 * keep sets as the calls without the suffix. KARA_TRIM_CHUNK, the chunk-aware trim, treats
 * the runs of consecutive members of the expanded set U that hold no anchor as chunks ([GIST]
 * section 2: a chunk has no fixed size and the span between two important points is kept
 * whole): they are dropped whole, weakest first (a run's strength is its best score; equal
 * strengths: the later run first), as long as the whole run fits in the excess |U| - k; at
 * the first run that does not fit the dropping stops, and the rest of the excess is trimmed
 * token by token as in kara_token2chunk. Other arguments and limits as the calls without the
 * suffix; an unknown trim is KARA_ERR_INVALID_ARG.
 */
kara_status kara_token2chunk_ex(const float* scores, const int32_t* sel, int32_t rows,
                                int32_t window, int32_t k, float anchor_frac, int32_t gap_limit,
                                int32_t widen, int32_t trim, int32_t* keep, cudaStream_t stream);
kara_status kara_select_chunks_ex(const float* scores, int32_t rows, int32_t window, int32_t k,
                                  float anchor_frac, int32_t gap_limit, int32_t widen,
                                  int32_t trim, int32_t* sel, int32_t* keep, cudaStream_t stream);

/*
 * kara_compress - selection, Token2Chunk and compaction in two kernels (the compaction plan,
 * which depends only on the windows' geometry, then one kernel per (layer, due sequence, KV
 * head) that selects and expands the row in shared memory and gathers it into the fresh
 * blocks; the last CTA of each sequence finalizes it). The result equals kara_select_chunks
 * on each layer's scores followed by kara_compact, bit for bit.
 *  scores   fp32 [num_layers, num_seqs, Hkv, window] (kara_score's output per layer).
 *  keep     int32 [num_layers, num_seqs, Hkv, k] or NULL: the keep sets, written when given.
 *  Other arguments, the workspace (KARA_OP_COMPACT), the device errors and their
 *  all-or-nothing rule as kara_compact; selection arguments and limits as kara_select_chunks.
 */
kara_status kara_compress(const float* scores, const kara_layer_kv* layers, int32_t num_layers,
                          const kara_pool* pool, const int32_t* seq_ids, int32_t num_seqs,
                          int32_t window, int32_t k, float anchor_frac, int32_t gap_limit,
                          int32_t widen, int32_t* keep, void* workspace, size_t workspace_bytes,
                          int32_t* dev_status, cudaStream_t stream);

/*
 * kara_compact - write the compressed windows into fresh blocks, rewrite the block table and
 * free the old window blocks ([KARA] abstract: Kara adapted to PagedAttention).
 *
 * For each due sequence r (cache row b), n = ctx_len[b], start = n-window, off = start % 16,
 * p0 = start / 16: n_new = ceil((off+k)/16) blocks are popped from the free list (sequences in
 * order r = 0, 1, ...; each takes free_list[top-1], free_list[top-2], ... for pages p0,
 * p0+1, ...). In every layer and KV head, slot p0*16+t receives the old slot p0*16+t for
 * t < off, and slot start+t receives the old slot start+keep[l][r][g][t] for t < k. Then
 * block_table[b][p0 .. p0+n_new) = fresh ids, [p0+n_new, p0+n_old) = -1 with n_old =
 * ceil((off+window)/16), ctx_len[b] = start+k, and the n_old old window blocks are pushed on
 * the free list (sequence order, page order). Slots of the fresh blocks past start+k are left
 * unwritten.
 *  layers     HOST array of num_layers (1 .. KARA_MAX_LAYERS) pool pointers.
 *  seq_ids    device int32 [num_seqs], strictly increasing, or NULL (rows 0..num_seqs-1).
 *  keep       int32 [num_layers, num_seqs, num_kv_heads, k], strictly ascending window
 *             positions (0 <= keep < window), checked on the device before anything moves.
 *  workspace  >= kara_workspace_bytes(KARA_OP_COMPACT, ...).
 *  dev_status KARA_ERR_OUT_OF_BLOCKS / KARA_ERR_INVALID_ARG (a short context, a bad seq_ids
 *             entry, or a keep entry outside the window or out of order) / KARA_ERR_BAD_BLOCK:
 *             then no pool, table, length or free-list entry is modified.
 */
kara_status kara_compact(const kara_layer_kv* layers, int32_t num_layers, const kara_pool* pool,
                         const int32_t* seq_ids, int32_t num_seqs, int32_t window, int32_t k,
                         const int32_t* keep, void* workspace, size_t workspace_bytes,
                         int32_t* dev_status, cudaStream_t stream);

/*
 * kara_compact_noalloc - kara_compact without a workspace argument: the plan scratch lives in
 * a fixed array of KARA_COMPACT_NOALLOC_SCRATCH_BYTES inside the library, so the call
 * allocates no device memory. The pages print no counterpart of this call; it exists for
 * callers that cannot allocate device memory when they compress, such as a serving engine
 * that has given all free device memory to its KV block pool, or a C caller without a device
 * allocator.
 *
 * Same arguments, semantics and device-side errors as kara_compact. Differences:
 *  - Returns KARA_ERR_WORKSPACE, without enqueueing anything, when the plan for num_seqs
 *    sequences and budget k would exceed the fixed array (plan size in bytes:
 *    4 * (144 + 12 * num_seqs + num_seqs * ceil((15 + k) / 16)); at k = 204 that admits up
 *    to 624 sequences).
 *  - The first call on each device looks up the array's device address (once per device,
 *    with that device current); make that first call before any stream capture. The address
 *    is kept for the life of the process: after cudaDeviceReset (or any teardown of the
 *    device's primary context) it is stale, so do not call this entry point again in that
 *    process after such a reset.
 *  - Every call on a device shares the one array, which keeps the last call's contents:
 *    calls that overlap on the GPU (other streams, or threads sharing a device without
 *    ordering) race on it. Order them on one stream.
 *  - Every GPU that loads the library holds the array until the process exits.
 */
#define KARA_COMPACT_NOALLOC_SCRATCH_BYTES (64u * 1024u)
kara_status kara_compact_noalloc(const kara_layer_kv* layers, int32_t num_layers,
                                 const kara_pool* pool, const int32_t* seq_ids, int32_t num_seqs,
                                 int32_t window, int32_t k, const int32_t* keep,
                                 int32_t* dev_status, cudaStream_t stream);

/*
 * paged_decode_attn - one decode step of grouped-query attention over the (compressed) paged
 * cache ([KARA] abstract: the kept KV pairs serve subsequent decoding, with PagedAttention).
 *
 *     out[b][h] = sum_t softmax_t( q[b][h] . K[t][g(h)] * scale ) V[t][g(h)],  t < ctx_len[b]
 *  q, out     bf16 [batch, num_q_heads, head_dim] (batch = pool->batch); an empty context
 *             gives a zero row.
 *  workspace  >= kara_workspace_bytes(KARA_OP_DECODE, ...): split-KV partial results.
 *  dev_status KARA_ERR_INVALID_ARG if a context exceeds the table, KARA_ERR_BAD_BLOCK for a
 *             block id out of range (that block is skipped).
 */
kara_status paged_decode_attn(const void* q, const void* k_cache, const void* v_cache,
                              const kara_pool* pool, int32_t num_q_heads, float scale, void* out,
                              void* workspace, size_t workspace_bytes, int32_t* dev_status,
                              cudaStream_t stream);

/*
 * The decode loop around the compression calls ([KARA] abstract: compression happens during
 * decoding, on the recently generated context, instead of on a fill threshold; [GIST]
 * section 3 "Der 'Periodische' Zeitplan (KvLLM)": on a fixed schedule, every 100 steps, the
 * oldest part of the current reasoning of some selected requests is cleaned up). One decode
 * step, for a batch of `pool->batch` sequences:
 *
 *   kara_step_begin                        blocks for the slots the step appends
 *   for every layer: kara_decode_append    attention of the new token, which joins the cache
 *   kara_step_end                          ctx_len + 1; on a check step, the due sequences
 *
 * and on a check step with due sequences: kara_score_ring (per layer), kara_select,
 * kara_token2chunk, kara_compact (all layers), kara_reset_tails. State beyond the pool:
 * tail (device int32 [batch], the tokens appended since the sequence's last compression,
 * zero at the start) and, per layer, a window-query ring q_ring (bf16 [batch, 2W, Hq, d]):
 * the query of the token at slot s is kept at rows s mod W and s mod W + W, so the queries
 * of the window [n-W, n) are the W contiguous rows from (n-W) mod W. A due sequence (tail >= W
 * at a check step) is compressed over its last W slots; tail then returns to 0.
 */

/*
 * kara_step_begin - before the layers of a decode step: every sequence whose next slot
 * n = ctx_len[b] starts a page (n % 16 == 0) takes the block of page n/16 from the top of
 * the free list (stack[top-1] first, sequences in ascending order), written into its table.
 * Device-checked, all or nothing: n < 0 or n >= 16 * max_blocks_per_seq gives
 * KARA_ERR_INVALID_ARG, fewer free blocks than sequences that need one gives
 * KARA_ERR_OUT_OF_BLOCKS; then nothing changes. Needs pool->free_list and free_top.
 */
kara_status kara_step_begin(const kara_pool* pool, int32_t* dev_status, cudaStream_t stream);

/*
 * kara_decode_append - one layer of a decode step, fused: the attention of the new token and
 * its entry into the cache and the window-query ring.
 *
 *     out[b][h] = sum_{t <= n} softmax_t( q[b][h] . K[t][g(h)] * scale ) V[t][g(h)]
 * with n = ctx_len[b] (not changed here) and slot n = the new token: K[n] = k_new[b],
 * V[n] = v_new[b]. Slot n is written into k_cache / v_cache (its block taken by
 * kara_step_begin), and q[b] into rows n mod window and n mod window + window of q_ring.
 *  q, out        bf16 [batch, num_q_heads, head_dim]; k_new, v_new bf16 [batch, Hkv, head_dim].
 *  q_ring        bf16 [batch, 2*window, num_q_heads, head_dim] or NULL (no ring).
 *  workspace     >= kara_workspace_bytes(KARA_OP_DECODE, ...).
 *  dev_status    as paged_decode_attn; KARA_ERR_INVALID_ARG if slot n is past the table,
 *                KARA_ERR_BAD_BLOCK if its block id is out of range (the write is skipped).
 */
kara_status kara_decode_append(const void* q, const void* k_new, const void* v_new,
                               void* k_cache, void* v_cache, const kara_pool* pool,
                               int32_t num_q_heads, float scale, void* q_ring, int32_t window,
                               void* out, void* workspace, size_t workspace_bytes,
                               int32_t* dev_status, cudaStream_t stream);

/*
 * kara_step_end - after the layers of a decode step: ctx_len[b] += 1, and tail[b] += 1 when
 * tail is not NULL. On a check step (check != 0) a sequence is due when tail[b] >= window
 * (window > 0: Kara's tail-W trigger; tail required) or when ctx_len[b] >= capacity
 * (capacity > 0: LaCache's full cache, capacity = sink + recent + R_max of the ladder, after
 * which lacache_compact keeps `budget` slots per layer; [LAC] iterative compaction). The due
 * sequences, ascending, go to due (device int32 [batch]) and their number to due_count
 * (device int32 [1]); the caller reads the count to size the compression. window = 0 and
 * capacity = 0 on a check step is KARA_ERR_INVALID_ARG.
 */
kara_status kara_step_end(const kara_pool* pool, int32_t* tail, int32_t window,
                          int32_t capacity, int32_t check, int32_t* due, int32_t* due_count,
                          cudaStream_t stream);

/*
 * kara_score_ring - kara_score with the window queries read from the window-query ring:
 * window position i of due sequence r (cache row b = seq_ids ? seq_ids[r] : r, n = ctx_len[b])
 * is q_ring[b][(n - window) mod window + i]. q_ring bf16 [batch, 2*window, num_q_heads,
 * head_dim]; every other argument, the output and the errors as kara_score.
 */
kara_status kara_score_ring(const void* q_ring, const void* k_cache, const kara_pool* pool,
                            const int32_t* seq_ids, int32_t num_seqs, int32_t window,
                            int32_t num_q_heads, float scale, float* scores, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status, cudaStream_t stream);

/*
 * kara_reset_tails - tail[seq_ids[i]] = 0 for i < num_seqs (after their compression); ids
 * outside [0, batch) are skipped.
 */
kara_status kara_reset_tails(int32_t* tail, const int32_t* seq_ids, int32_t num_seqs,
                             int32_t batch, cudaStream_t stream);

/*
 * lacache_compact - one pass of LaCache's ladder compaction ([LAC] ladder pattern and
 * iterative compaction) through the same paged gather as kara_compact.
 *
 * For each due sequence (cache row b, n = ctx_len[b]) and layer l the kept slots are, in
 * ascending order: slots [0, sink); the ladder region's kept rungs; slots [n-recent, n). The
 * region is the R_max = (budget-sink-recent)*L/S slots before the recent tail (older slots
 * are dropped in all layers); it is cut into rungs of `rung` slots and rung j is kept in the
 * layers (j*(S-O) + t) mod L, t < S. Every layer keeps exactly `budget` slots; slot t of the
 * compacted sequence holds the t-th kept slot (every KV head of the layer alike). The
 * sequence moves to ceil(budget/16) fresh blocks (popped as in kara_compact), its ceil(n/16)
 * old blocks are pushed afterwards, and ctx_len[b] = budget.
 *  Requirements (host-checked): 1 <= S <= L, 0 <= O < S, (S-O) divides S and L,
 *  budget-sink-recent > 0 and a multiple of rung*S/(S-O). Device-checked: n >= sink + recent +
 *  R_max (a full cache), else KARA_ERR_INVALID_ARG and nothing is modified.
 */
kara_status lacache_compact(const kara_layer_kv* layers, int32_t num_layers,
                            const kara_pool* pool, const int32_t* seq_ids, int32_t num_seqs,
                            const kara_lacache_params* params, void* workspace,
                            size_t workspace_bytes, int32_t* dev_status, cudaStream_t stream);

/*
 * kara_workspace_bytes - workspace size for one call (0 if the op needs none).
 *  KARA_OP_SCORE:   num_seqs, window, num_q_heads used.
 *  KARA_OP_COMPACT: num_seqs, window (the budget k goes in `k_or_budget`).
 *  KARA_OP_DECODE:  pool->batch, num_q_heads, head_dim, max_blocks_per_seq used.
 *  KARA_OP_LACACHE: num_seqs, budget in `k_or_budget`.
 * `pool` is a host pointer (may be NULL for SCORE).
 */
size_t kara_workspace_bytes(kara_op op, const kara_pool* pool, int32_t num_seqs, int32_t window,
                            int32_t num_q_heads, int32_t k_or_budget);

/* Static, human-readable name of a status code. */
const char* kara_status_str(int32_t status);

/* Text of the CUDA error behind the calling thread's last KARA_ERR_CUDA return (with the
 * name of the step that failed), or "" if there was none. Valid until the thread's next
 * call into the library. */
const char* kara_last_error(void);

/* Number of kernel launches the library has issued in this process (launch calls that
 * returned cudaSuccess, all threads and devices), so that a caller can count the kernels a
 * sequence of calls runs: take the difference of two readings. */
uint64_t kara_launch_count(void);

/* Library version string ("kara-b200 <major>.<minor>"). */
const char* kara_version(void);

/*
 * kara_wait_probe - exercises the bounded-wait failure path on the device. The pages have no
 * counterpart of it: it exists so that failure detection can be tested without a GPU fault.
 *  One CTA; thread 0 of warp 0 waits on an mbarrier that nothing arrives on, with a budget of
 *  about `wait_ms` milliseconds of SM clock, then reports KARA_ERR_TIMEOUT to dev_status and
 *  raises the CTA's abort flag; thread 0 of warp 1 waits on a second such barrier with the
 *  library's default budget (about 2 s) and must unwind through that flag. The kernel then
 *  returns, and the context stays usable.
 *  wait_ms     1 .. 2000 (host-checked, else KARA_ERR_INVALID_ARG).
 *  dev_status  device int32, written on the device (first error wins).
 */
kara_status kara_wait_probe(int32_t wait_ms, int32_t* dev_status, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KARA_H */
