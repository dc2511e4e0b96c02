/*
 * sd_api.h -- C ABI of the top-k sparse decode library for NVIDIA B200 (sm_100a).
 *
 * One decode step over a paged KV cache, for a batch of B requests with one
 * query token each:
 *
 *   1. indexer score  s[b,g,t] = sum_h w[b,g,h] * max(0, sum_d qi[b,g,h,d] * ki[t,g,d])
 *                     for every cached token t < seqlens[b], keys read in place
 *                     from the paged indexer pool through the block table;
 *   2. top-k          per (request, KV head) the min(k, seqlen) tokens of highest
 *                     score, ties to the lower token index, written in ascending
 *                     token order and padded with -1;
 *   3. sparse attn    o[b,h] = sum_j softmax_j(scale * q[b,h] . K_j) V_j over the
 *                     selected rows of KV head g = h / (H/G), gathered from the
 *                     paged K/V pools, followed by a split combine.
 *
 * Where this comes from. The pages describe the DSA decode data flow: an
 * indexer scores the cached tokens, a top-k kernel fills a persistent top-k
 * buffer, and core sparse attention consumes it ("Overlap DSA heuristic
 * prev_topk write-back on the aux stream", Description). Predicted indices are
 * request-local token ids translated to pool rows through the block table, and
 * negative entries are invalid ("Unify sparse attention framework with clean
 * backend interfaces", review notes on DSA global index conversion). The golden
 * reference attends over selected tokens of a logical cache rebuilt from
 * pages ("Add DSA Vanilla sparse attention", Walkthrough). A typed, fixed
 * signature beats a generic keyword carrier ("Compact pseudo-KV/topological
 * sparse attention benchmark evidence", the 0.756x kwargs result). The pages
 * never write the formulas out; the readings taken (ReLU per indexer head,
 * integer head weights, lowest-index ties, ascending order) are stated in the
 * design notes.
 *
 * Conventions for every call
 *   - All array pointers are DEVICE pointers owned by the caller; the library
 *     never allocates, frees or keeps them. Arrays are dense, row-major, with
 *     the shapes given per argument. bf16 arrays are passed as raw uint16 bits.
 *   - Pools are NHD: [num_pages, page_size, kv_heads, dim]. Token t of request
 *     b lives at page block_table[b * max_pages_per_req + t / page_size],
 *     slot t % page_size.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream). Every call only
 *     enqueues work on it: no host synchronisation, no allocation, so a call can
 *     be captured in a CUDA graph. Buffers keep the addresses the caller gives.
 *   - `workspace` is caller-owned device scratch of at least the size that
 *     sd_workspace_size() returns for the same shape (256-byte aligned).
 *   - The library sets each kernel's shared-memory limit once per device and
 *     remembers it. A device reset (cudaDeviceReset) clears such settings:
 *     unload the library (or restart the process) after one.
 *   - Argument errors are found on the host before any launch and returned as
 *     a status; nothing is enqueued then. Errors in device-resident data (a
 *     seqlen beyond the block table, a block-table entry outside the pool, an
 *     index at or past seqlen) cannot be seen on the host: the kernels mask the
 *     offending token (a bad indexer page scores INT32_MIN, a bad attention
 *     row is skipped), clamp the length, and OR a bit into a sticky per-device
 *     error word that sd_get_device_errors() reads.
 *
 * Supported shapes (others return SD_ERR_UNSUPPORTED):
 *   indexer  Di in {32, 64, 128}, 1 <= Hi <= 64, G * Di <= 1024
 *   top-k    1 <= k <= 2048, max_seqlen <= 1 << 20
 *   attn     (Dk, Dv) in {(64, 64), (128, 128), (576, 512)}, H % G == 0,
 *            H / G <= 128; with v_pages == NULL, V is the first Dv columns of
 *            the K row (MLA latent rows, or MQA with V = K)
 */
#ifndef SD_API_H
#define SD_API_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sd_status {
  SD_OK = 0,
  SD_ERR_INVALID_ARG = 1,   /* null pointer, negative size, inconsistent shape */
  SD_ERR_UNSUPPORTED = 2,   /* a valid shape this build has no kernel for      */
  SD_ERR_WORKSPACE = 3,     /* workspace missing, too small or misaligned      */
  SD_ERR_CUDA = 4           /* a CUDA runtime call failed (see sd_last_cuda_error) */
} sd_status;

/* Bits of the sticky per-device error word (sd_get_device_errors). */
#define SD_DEVERR_SEQLEN 0x1u   /* seqlens[b] < 0, > max_seqlen or > the block table  */
#define SD_DEVERR_PAGE 0x2u     /* a needed block-table entry outside [0, num_pages)  */
#define SD_DEVERR_INDEX 0x4u    /* an attention index >= seqlens[b] (row skipped)     */
#define SD_DEVERR_TIMEOUT 0x8u  /* a bounded on-chip wait ran out (the kernel unwound) */

/* Geometry shared by the indexer pool and the K/V pools of one cache. */
typedef struct sd_paged_desc {
  int32_t num_pages;          /* pages in each pool                           */
  int32_t page_size;          /* tokens per page, >= 1                        */
  int32_t max_pages_per_req;  /* row stride of block_table                    */
  int32_t kv_heads;           /* G: KV heads (1 for MLA latent rows)          */
} sd_paged_desc;

/* Device scratch (bytes) that any of the three calls below needs for this
 * shape: scores (unless the caller passes its own), top-k state and split
 * attention partials. Pure function of its arguments; 0 on invalid input. */
size_t sd_workspace_size(int32_t B, int32_t G, int32_t max_seqlen, int32_t k,
                         int32_t H, int32_t Dv);

/* Steps 1 + 2: indexer scores and per-(request, KV head) top-k.
 *   qi          int8  [B, G, Hi, Di]  indexer queries
 *   w           int32 [B, G, Hi]      indexer head weights
 *   ki_pages    int8  [num_pages, page_size, G, Di]  indexer key pool, 16-byte
 *               aligned (SD_ERR_INVALID_ARG otherwise)
 *   block_table int32 [B, max_pages_per_req]  physical page per logical page
 *   seqlens     int32 [B]             cached tokens per request (incl. current)
 *   max_seqlen  host upper bound of seqlens (sizes grids and scores)
 *   indices     int32 [B, G, k]  OUT  ascending request-local tokens, -1 padded
 *   scores      int32 [B, G, max_seqlen]  OUT, nullable; entries t >= seqlens[b]
 *               are left unwritten. When NULL the scores live in the workspace. */
sd_status sd_indexer_topk(const int8_t* qi, const int32_t* w, const int8_t* ki_pages,
                          const int32_t* block_table, const int32_t* seqlens,
                          sd_paged_desc pd, int32_t B, int32_t Hi, int32_t Di,
                          int32_t max_seqlen, int32_t k, int32_t* indices, int32_t* scores,
                          void* workspace, size_t workspace_bytes, void* stream);

/* Step 3: attention over selected rows, then the split combine.
 *   q        bf16 [B, H, Dk]
 *   k_pages  bf16 [num_pages, page_size, G, Dk]
 *   v_pages  bf16 [num_pages, page_size, G, Dv], or NULL: V = K row[:Dv]
 *   indices  int32 [B, G, k] request-local tokens. Only the first min(k, seqlens[b])
 *            slots of a row are read (a selection has at most seqlen distinct
 *            tokens, so it fits there); entries < 0 in them are skipped
 *   scale    softmax scale applied to q . K
 *   out      bf16 [B, H, Dv] OUT (round to nearest even); zero when nothing is selected
 *   lse      fp32 [B, H] OUT, nullable: natural-log sum of exp(scale * q . K_j),
 *            -inf when nothing is selected */
sd_status sd_sparse_attn(const uint16_t* q, const uint16_t* k_pages, const uint16_t* v_pages,
                         const int32_t* block_table, const int32_t* seqlens,
                         const int32_t* indices, sd_paged_desc pd, int32_t B, int32_t H,
                         int32_t Dk, int32_t Dv, int32_t k, float scale, uint16_t* out,
                         float* lse, void* workspace, size_t workspace_bytes, void* stream);

/* TriAttention-style decode-time eviction of one layer ("Add TriAttention
 * KV-cache compression method", Summary and Key Design Decisions): score the
 * evictable region [n_sink, L_b - n_recent) of every request with calibrated
 * per-head queries, keep the `budget` best tokens, and compact the kept K/V
 * rows in place to the front of the request's pages.
 *   q_cal       bf16 [H, D]: one calibrated query per query head (head h reads
 *               KV head h * G / H), in the cache's precision
 *   k_pages     bf16 [num_pages, P, G, D], compacted in place; 16-byte aligned
 *   v_pages     bf16 [num_pages, P, G, D] compacted the same way, or NULL;
 *               16-byte aligned
 *   mode        SD_TRI_UNION: one selection per request (all KV heads move
 *               together); SD_TRI_PER_HEAD (or SD_TRI_PER_LAYER_PER_HEAD):
 *               one per (request, KV head)
 *   new_seqlens int32 [B] out: n_sink + budget + n_recent, or L_b when the
 *               evictable region holds at most `budget` tokens (nothing moves)
 * Score of evictable position p under query head h: z = q_cal[h] . K, summed
 * in fp32 (each bf16 x bf16 product exact; one fused multiply-add per d, so
 * equal inputs give equal scores), shifted by the head's maximum over the
 * region; a KV head's score is the maximum over its query heads, the union
 * score the maximum over KV heads. The `budget` largest are kept (ties to the
 * lower position), followed by the recent tail. The kept set is a top-budget
 * set of the exact scores up to the fp32 rounding of the sums. Pages past the new
 * lengths are free for the caller to release; the block table is unchanged.
 * max_seqlen is a host upper bound of seqlens (it sizes the workspace);
 * larger lengths are clamped and flag SD_DEVERR_SEQLEN.
 * Limits: D in {64, 128}; H / G in {1, 2, 4, 8}; H <= 256;
 * 1 <= budget <= 2048; B * G <= 65535; the bytes one token moves (union:
 * G * D * 2, per-head: D * 2; twice that with V) at most 32768.
 * block_table, seqlens and new_seqlens may be NULL when B = 0.
 * Workspace: sd_tri_workspace_size(); the caller owns every buffer.
 * Errors: SD_ERR_INVALID_ARG / SD_ERR_UNSUPPORTED / SD_ERR_WORKSPACE before
 * any launch. A block-table entry outside the pool inside a request sets
 * SD_DEVERR_PAGE and that row is skipped (the request's result is then
 * unspecified, the pools outside its pages untouched). The compaction's
 * units wait on one another with bounded waits; one that runs out sets
 * SD_DEVERR_TIMEOUT and skips its writes. */
#define SD_TRI_UNION 0
#define SD_TRI_PER_HEAD 1
#define SD_TRI_PER_LAYER_PER_HEAD 2 /* with one layer, the same as SD_TRI_PER_HEAD */
size_t sd_tri_workspace_size(int32_t B, int32_t G, int32_t H, int32_t D, int32_t max_seqlen, int32_t n_sink,
                             int32_t n_recent, int32_t budget, int32_t mode, int32_t has_v);
sd_status sd_tri_compact(const uint16_t* q_cal, uint16_t* k_pages, uint16_t* v_pages, const int32_t* block_table,
                         const int32_t* seqlens, sd_paged_desc pd, int32_t B, int32_t H, int32_t D, int32_t max_seqlen,
                         int32_t n_sink, int32_t n_recent, int32_t budget, int32_t mode, int32_t* new_seqlens,
                         void* workspace, size_t workspace_bytes, void* stream);

/* The same over n_layers layers that share the block table and lengths
 * ("Add TriAttention KV-cache compression method", Summary: union, per_head
 * and per_layer_perhead eviction modes). q_cal, k_pages and v_pages are HOST
 * arrays of n_layers device pointers (v_pages may be NULL: no V pools).
 *   SD_TRI_UNION              one selection per request for every layer and
 *                             head: score = max over layers and heads
 *   SD_TRI_PER_HEAD           one selection per (request, KV head) for every
 *                             layer: score = max over layers and that KV
 *                             head's query heads
 *   SD_TRI_PER_LAYER_PER_HEAD an independent per-head selection in each layer
 * (each head's logits shifted by that layer's and head's maximum, as above).
 * Every layer is compacted; new_seqlens holds the common new lengths.
 * Workspace: sd_tri_layers_workspace_size(). Limits and errors as above. */
size_t sd_tri_layers_workspace_size(int32_t n_layers, int32_t B, int32_t G, int32_t H, int32_t D, int32_t max_seqlen,
                                    int32_t n_sink, int32_t n_recent, int32_t budget, int32_t mode, int32_t has_v);
sd_status sd_tri_compact_layers(const uint16_t* const* q_cal, uint16_t* const* k_pages, uint16_t* const* v_pages,
                                int32_t n_layers, const int32_t* block_table, const int32_t* seqlens, sd_paged_desc pd,
                                int32_t B, int32_t H, int32_t D, int32_t max_seqlen, int32_t n_sink, int32_t n_recent,
                                int32_t budget, int32_t mode, int32_t* new_seqlens, void* workspace,
                                size_t workspace_bytes, void* stream);

/* Steps 1 + 2, and the whole decode step, with the previous step's selection
 * as a hint: the "heuristic_prev_topk" feedback of "Overlap DSA heuristic
 * prev_topk write-back on the aux stream" (Description: each decode step's
 * top-k is the next step's pre_idx hint).
 *   hint  int32 [B, G, k] request-local tokens (-1 and tokens >= seqlen are
 *         ignored), typically the previous call's `indices`; NULL = no hint.
 *         It must not be the same buffer as `indices`.
 * The result is identical to the unhinted call for any hint. A good hint (the
 * previous selection of a slowly changing query) narrows the radix passes of
 * the top-k to the range between the hint's lowest current score and the best
 * score outside it; an exact hint needs no radix pass at all. The write-back
 * of the pages (a copy into the hint buffer) is not needed: alternate two
 * `indices` buffers between steps and pass the other as the hint. Other
 * arguments and errors as for sd_indexer_topk / sd_decode_step. */
sd_status sd_indexer_topk_hinted(const int8_t* qi, const int32_t* w, const int8_t* ki_pages,
                                 const int32_t* block_table, const int32_t* seqlens, sd_paged_desc pd, int32_t B,
                                 int32_t Hi, int32_t Di, int32_t max_seqlen, int32_t k, const int32_t* hint,
                                 int32_t* indices, int32_t* scores, void* workspace, size_t workspace_bytes,
                                 void* stream);
sd_status sd_decode_step_hinted(const int8_t* qi, const int32_t* w, const int8_t* ki_pages, const uint16_t* q,
                                const uint16_t* k_pages, const uint16_t* v_pages, const int32_t* block_table,
                                const int32_t* seqlens, sd_paged_desc pd, int32_t B, int32_t Hi, int32_t Di,
                                int32_t H, int32_t Dk, int32_t Dv, int32_t max_seqlen, int32_t k, float scale,
                                const int32_t* hint, int32_t* indices, int32_t* scores, uint16_t* out, float* lse,
                                void* workspace, size_t workspace_bytes, void* stream);

/* Steps 3 + 4 for n_layers layers that share one selection: the
 * shared-indexer decode of "Overlap DSA heuristic prev_topk write-back on the
 * aux stream" (Description: layers without their own indexer reuse the top-k
 * buffer) and of "Add DSA Vanilla sparse attention" (the persistent index
 * buffer read by every layer).
 *   q        bf16 [n_layers, B, H, Dk], layer-major
 *   k_pages  HOST array of n_layers device pointers, each a latent / key pool
 *            laid out as for sd_sparse_attn (all with the geometry `pd`)
 *   v_pages  HOST array of n_layers value pools, or NULL (V inside K)
 *   block_table, seqlens, indices: one set, shared by every layer
 *   out      bf16 [n_layers, B, H, Dv]; lse fp32 [n_layers, B, H] or NULL
 * With MLA rows (G = 1, H = 128, Dk = 576, Dv = 512, V inside K), up to 16
 * layers run in one launch, so the selections are resolved to pool rows once
 * per group of layers and small batches fill the GPU; other shapes run layer
 * after layer. Workspace: sd_attn_layers_workspace_size(). Errors as for
 * sd_sparse_attn; SD_ERR_INVALID_ARG also for n_layers < 1 or a NULL pool. */
size_t sd_attn_layers_workspace_size(int32_t n_layers, int32_t B, int32_t G, int32_t k, int32_t H, int32_t Dv);
sd_status sd_sparse_attn_layers(const uint16_t* q, const uint16_t* const* k_pages, const uint16_t* const* v_pages,
                                int32_t n_layers, const int32_t* block_table, const int32_t* seqlens,
                                const int32_t* indices, sd_paged_desc pd, int32_t B, int32_t H, int32_t Dk,
                                int32_t Dv, int32_t k, float scale, uint16_t* out, float* lse, void* workspace,
                                size_t workspace_bytes, void* stream);

/* Steps 3 + 4 with the selection given in the packed forms of the unified
 * sparse runtime ("Unify sparse attention framework with clean backend
 * interfaces", runtime parameters sparse_attn_offsets and
 * sparse_attn_indices_block_size):
 *   indices     int32, all rows' entries packed (may be NULL if every row is
 *               empty); row r = b * G + g owns indices[offsets[r] ..
 *               offsets[r + 1]).
 *   offsets     int32 [B * G + 1], non-decreasing.
 *   block_size  0 or 1: an entry is a token; bs > 1: entry e selects tokens
 *               e*bs .. e*bs + bs - 1.
 *   max_selected  1 .. 2048: the most tokens any row keeps.
 * Row r attends over the valid tokens of its expansion, in list order: entries
 * < 0 are skipped, tokens at or past seqlens[b] are dropped, and only the
 * first min(max_selected, seqlens[b]) are kept. An entry whose whole block is
 * past the seqlen, decreasing offsets, or more valid tokens than kept set
 * SD_DEVERR_INDEX. Duplicates are attended as listed. Other arguments,
 * outputs and errors as for sd_sparse_attn. Workspace:
 * sd_csr_workspace_size(). */
size_t sd_csr_workspace_size(int32_t B, int32_t G, int32_t max_selected, int32_t H, int32_t Dv);
sd_status sd_sparse_attn_csr(const uint16_t* q, const uint16_t* k_pages, const uint16_t* v_pages,
                             const int32_t* block_table, const int32_t* seqlens, const int32_t* indices,
                             const int32_t* offsets, int32_t block_size, int32_t max_selected, sd_paged_desc pd,
                             int32_t B, int32_t H, int32_t Dk, int32_t Dv, float scale, uint16_t* out, float* lse,
                             void* workspace, size_t workspace_bytes, void* stream);

/* Steps 1 + 2 + 3 in one call on one stream (arguments as above). */
sd_status sd_decode_step(const int8_t* qi, const int32_t* w, const int8_t* ki_pages,
                         const uint16_t* q, const uint16_t* k_pages, const uint16_t* v_pages,
                         const int32_t* block_table, const int32_t* seqlens, sd_paged_desc pd,
                         int32_t B, int32_t Hi, int32_t Di, int32_t H, int32_t Dk, int32_t Dv,
                         int32_t max_seqlen, int32_t k, float scale, int32_t* indices,
                         int32_t* scores, uint16_t* out, float* lse, void* workspace,
                         size_t workspace_bytes, void* stream);

/* Steps 1 + 2 without any workspace (the pages have no counterpart; this is a
 * deployment convenience). It is sd_indexer_topk for callers that cannot
 * allocate device memory: a plugin that runs inside a host application which
 * owns every device allocation, or a serving loop that must not allocate once
 * it has started. Such callers cannot provide a scores workspace. Here the
 * scores live in a scratch array inside the library's device image:
 * SD_NOALLOC_MAX_SCORES int32 values (16 MiB). It is resident on every device
 * where the library's device code is loaded, whichever entry point loaded
 * it, from then until the context is destroyed.
 *   Arguments, outputs and errors are as for sd_indexer_topk. There is no
 *   scores output. The call returns SD_ERR_WORKSPACE, with nothing enqueued,
 *   when B * G * max_seqlen > SD_NOALLOC_MAX_SCORES.
 *   A call that is not being captured looks up the device's scratch address
 *   (a runtime query, not an allocation) and remembers it; a call under
 *   stream capture uses the remembered address. So make one call on a device
 *   before capturing any, and again after a device reset or anything else
 *   that destroys the primary context (that reloads the library's device
 *   image at another address): a captured graph keeps the address it was
 *   captured with and must be captured anew after such a reset. A first call
 *   on a device made under capture returns SD_ERR_INVALID_ARG.
 *   Every call on a device shares the one scratch array. Calls whose work
 *   overlaps on the GPU (other streams, other threads) race on it and give
 *   undefined results: serialise them. The array keeps the last call's scores,
 *   and that is harmless, because every score a call reads it has written
 *   first. The call never allocates or frees device memory. */
#define SD_NOALLOC_MAX_SCORES (4u << 20)
sd_status sd_indexer_topk_noalloc(const int8_t* qi, const int32_t* w, const int8_t* ki_pages,
                                  const int32_t* block_table, const int32_t* seqlens,
                                  sd_paged_desc pd, int32_t B, int32_t Hi, int32_t Di,
                                  int32_t max_seqlen, int32_t k, int32_t* indices, void* stream);

/* Stage timing for monitoring and benchmarks (no counterpart on the pages).
 * `events` points to 2 * n cudaEvent_t handles created by the caller; while
 * set, every call of this thread records events[2*i] just before and
 * events[2*i+1] just after stage i on the call's stream, for the stages
 * 0 = indexer scores, 1 = top-k, 2 = split attention, 3 = combine (a stage
 * a call does not run records nothing). n = 0 or events = NULL switches it
 * off. The handles must outlive their use; the library does not own them. */
sd_status sd_set_stage_events(void* const* events, int32_t n);

/* Test hook for the failure path of bounded waits (no counterpart on the
 * pages). The eviction compaction's units wait on one another through flags
 * in global memory (sd_tri_compact); each wait gives up after a bounded number
 * of polls, sets SD_DEVERR_TIMEOUT and skips that unit's writes, so a wait
 * that never ends cannot hang the GPU. This sets that number for compactions
 * launched afterwards by any thread of the process (it is a launch argument,
 * so a captured graph keeps the value it was captured with): polls < 0
 * restores the default of 2^22, 0 makes every such wait give up at once (the
 * compaction then leaves the pools in an unspecified state and flags the
 * timeout). Values above 2^22 return SD_ERR_INVALID_ARG. No other wait of
 * the library is affected. Nothing is enqueued; no CUDA call is made. */
sd_status sd_set_wait_limit(int32_t polls);

/* Reads (and with clear != 0 resets) the sticky device error word of the
 * current device. Synchronises the device: for tests and debugging only. */
sd_status sd_get_device_errors(uint32_t* bits, int32_t clear);

/* Human-readable name of a status. Never NULL. */
const char* sd_status_str(sd_status status);

/* The cudaError_t of the last failing CUDA call in this thread (0 if none). */
int32_t sd_last_cuda_error(void);

/* Number of kernel launches the last successful call enqueued (per thread). */
int32_t sd_last_launch_count(void);

/* Library ABI version, (major << 16) | minor. */
int32_t sd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SD_API_H */
