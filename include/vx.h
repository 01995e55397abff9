/*
 * vx.h -- C ABI of libvx: block top-k sparse attention decode over a paged KV cache,
 * hand-written CUDA for B200 (sm_100a).
 *
 * The method (Vortex: Efficient and Programmable Sparse Attention Serving for AI Agents,
 * paper note, section 系统设计 1 "vFlow", the block top-k example): a cache stage keeps
 * one key centroid per KV page; an indexer scores every page by the product of the query
 * with the centroids, keeps the top-k pages, and exact softmax attention runs on those
 * pages only.  The paged layout (batch size, pointer array, page index structure) is the
 * one of section 系统设计 2 "vTensor"; top-k is the radix top-k of section 系统设计 3
 * with an optional stochastic-early-termination mode.
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 * Pointers named *_cache, q, centroids, scores, sel, out, lse, ws, err and every array
 * of vx_page_table are DEVICE pointers; vx_geometry and vx_page_table themselves are
 * read on the host during the call and may be freed when it returns.  `stream` is a
 * cudaStream_t (NULL = the legacy default stream).
 *
 * Ownership: the caller allocates and owns every buffer and keeps it alive until the
 * stream has passed the call.  The library allocates no device memory and keeps no
 * device state, with one exception: the fixed scratch array of vx_sparse_decode_noalloc
 * (one per GPU, held until the process exits, shared by every call of that function).
 * Calls are asynchronous and stream-ordered and never synchronise the host.  Calls on
 * different streams may run concurrently when they write disjoint buffers (outputs,
 * workspace, err).
 *
 * Layouts (row-major, element types in brackets):
 *   k_cache    [num_pool_pages][num_kv_heads][page_size][head_dim_qk]  (bf16)
 *   v_cache    [num_pool_pages][num_kv_heads][page_size][head_dim_v]   (bf16); ignored
 *              when mla_shared_kv = 1: the value of a token is then the first head_dim_v
 *              dims of its key row (MLA latent).
 *   centroids  [num_pool_pages][num_kv_heads][head_dim_qk]             (bf16), keyed by
 *              physical page so a centroid moves with its page.
 *   q          [batch][num_q_heads][head_dim_qk]                       (bf16)
 *   scores     [batch][num_kv_heads][max_pages]                        (fp32)
 *   sel        [batch][num_kv_heads][k]  logical page indices          (int32), ascending,
 *              -1 in the slots past k_eff = min(k, n_b)
 *   out        [batch][num_q_heads][head_dim_v]                        (bf16)
 *   lse        [batch][num_q_heads]  natural-log sum of exp(logits)    (fp32)
 * Query head g belongs to KV head g / (num_q_heads / num_kv_heads) (GQA grouping).
 * Request b holds seq_lens[b] tokens in n_b = ceil(seq_lens[b] / page_size) logical
 * pages; logical page j is physical page page_indices[page_ptr[b] + j]; token t of the
 * request sits in slot t % page_size of logical page t / page_size.  Slots past the
 * length are never read into a result, whatever they hold.
 * Every device pointer must be 16-byte aligned.
 *
 * Errors: argument problems are found on the host before anything is launched and
 * returned as VX_ERR_INVALID_ARG / VX_ERR_UNSUPPORTED / VX_ERR_WORKSPACE; a failed
 * launch returns VX_ERR_CUDA.  vx_last_error() then holds a message (per host thread).
 * Problems in device data (a page id outside the pool, a length out of range, a
 * selected page outside the request) are found by the kernels, which skip the bad item
 * and OR a VX_DATA_* bit into *err (a device int32; may be NULL).  Kernels never trap
 * and never wait without a time limit; a wait that runs out sets VX_DATA_TIMEOUT.
 */
#ifndef VX_H
#define VX_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    VX_OK = 0,
    VX_ERR_INVALID_ARG = 1, /* NULL or misaligned pointer, bad size, inconsistent geometry */
    VX_ERR_UNSUPPORTED = 2, /* well-formed but not built: head dims, page size, group size */
    VX_ERR_WORKSPACE = 3,   /* workspace NULL or smaller than vx_workspace_size() */
    VX_ERR_CUDA = 4         /* a CUDA runtime call or kernel launch failed */
} vx_status;

/* bits OR-ed into *err by the kernels */
#define VX_DATA_BAD_PAGE_ID 1u   /* page_indices entry outside [0, num_pool_pages) */
#define VX_DATA_BAD_SEQ_LEN 2u   /* seq_lens[b] < 1 or > max_pages * page_size */
#define VX_DATA_BAD_SELECTION 4u /* sel entry >= n_b (entries < 0 are empty slots) */
#define VX_DATA_TIMEOUT 8u       /* a bounded wait inside a kernel ran out */

typedef struct {
    int32_t batch;         /* 1 <= B <= 4096 */
    int32_t num_q_heads;   /* Hq, a multiple of num_kv_heads */
    int32_t num_kv_heads;  /* Hkv: GQA a power of two <= 16, MLA 1 */
    int32_t head_dim_qk;   /* key / score dim: 64 or 128 (GQA), 576 (MLA latent+rope) */
    int32_t head_dim_v;    /* value dim: = head_dim_qk (GQA), 512 (MLA) */
    int32_t page_size;     /* P tokens per page: 16, 32 or 64 (MLA: 32 or 64) */
    int32_t mla_shared_kv; /* 1: V = first head_dim_v dims of the K row; v_cache unused */
    int64_t num_pool_pages;
} vx_geometry;

typedef struct {
    const int32_t *page_ptr;     /* [B] start of request b's row in page_indices */
    const int32_t *page_indices; /* physical page ids, row b holds n_b entries */
    const int32_t *seq_lens;     /* [B] valid tokens, 1 <= seq_lens[b] <= max_pages * P */
    int32_t max_pages;           /* host bound on n_b over the batch; sizes scores rows */
} vx_page_table;

/*
 * Cache stage: key centroid of a page = mean of the keys of its valid tokens, per KV
 * head, stored as bf16 (the cache's element type): the exact mean (fp64 sum of the bf16
 * keys, one fp64 division) rounded once to nearest-even (paper note, 系统设计 1: the
 * cache stage keeps a per-block key centroid that does not depend on the query).
 *   k_new == NULL: rebuild.  Recompute the centroid of every page of every request
 *       holding a position >= first_pos[b] (first_pos NULL: every page).  Use after a
 *       prefill or a bulk load.  v_cache, v_new unused.
 *   k_new != NULL, first_pos == NULL: append one decode token per request.  seq_lens
 *       already counts the new token and its page is installed in the table; the token
 *       (k_new [B][Hkv][Dqk], v_new [B][Hkv][Dv], v_new ignored for MLA) is written into
 *       slot (seq_lens[b]-1) % P of its page and that page's centroid is recomputed from
 *       its keys.
 *   k_new != NULL, first_pos != NULL: prefill write (a prompt or a chunk of one).
 *       Positions [first_pos[b], seq_lens[b]) of request b arrive packed in request
 *       order, k_new [N][Hkv][Dqk] and v_new [N][Hkv][Dv] with N = sum over b of
 *       seq_lens[b] - first_pos[b], request b's rows right after those of requests
 *       0..b-1; their pages are installed in the table.  One pass writes them into their
 *       slots and recomputes the centroid of every page they touch (older tokens of the
 *       first page are read from k_cache).  A request with first_pos[b] == seq_lens[b]
 *       writes nothing; first_pos[b] outside [0, seq_lens[b]] sets VX_DATA_BAD_SEQ_LEN and
 *       that request contributes no rows.
 * Writes: centroids (and, when appending or prefilling, the new tokens' slots of k_cache /
 * v_cache).
 */
vx_status vx_centroid_update(const vx_geometry *geo, const vx_page_table *table, void *k_cache,
                             void *v_cache, void *centroids, const void *k_new, const void *v_new,
                             const int32_t *first_pos, int32_t *err, void *stream);

/*
 * Indexer: scores[b][h][j] = sum over the query heads g of KV group h of
 * q[b][g][:score_dims] . centroid(page j of b, head h)[:score_dims], fp32, no softmax
 * scale (paper note, 系统设计 1: blocks are scored by a matrix product of query and
 * centroids; MLA experiment section: the rope-aware variant scores on all 576 latent +
 * rope dims, the rope-unaware one on the 512 latent dims only).
 * score_dims: 0 = head_dim_qk; else 1..head_dim_qk, a multiple of 8.
 * Writes scores[b][h][j] for j < n_b only.
 */
vx_status vx_score_pages(const vx_geometry *geo, const vx_page_table *table, const void *q,
                         const void *centroids, int32_t score_dims, float *scores, int32_t *err,
                         void *stream);

/*
 * Top-k pages per (request, KV head) row of scores (paper note, 系统设计 3: radix top-k,
 * with stochastic early termination and remapping as the faster approximate option).
 *   mode 0 (exact): the k_eff = min(k, n_b) pages of largest score; ties at the boundary
 *       go to the lower page index; -0.0 ties with +0.0.  Radix select on order-
 *       preserving 32-bit keys, most significant digit first.
 *   mode 1 (approximate): remap each score to a 12-bit code
 *       min(4095, floor((s - lo) * (4096 / (hi - lo)))) in fp32 (lo, hi: the row's min
 *       and max; hi == lo gives 0); one histogram; every page above the boundary code b*
 *       is taken and the slots left are filled from code b* in cyclic page order from
 *       offset SplitMix64(seed) draw number (b * Hkv + h) mod n_b, with no refinement.
 *   mode 2 (approximate, coarser): the same with 10-bit codes (1024 in place of 4096):
 *       a cheaper histogram for a larger boundary code.
 *   mode 3 (approximate, coarsest): the same with 8-bit codes (256).
 * Writes sel [B][Hkv][k]: chosen pages in ascending order, then -1.  k >= 1.
 * Scores must be finite; NaN scores give an unspecified (but in-range) selection.
 */
vx_status vx_topk_pages(const vx_geometry *geo, const vx_page_table *table, const float *scores,
                        int32_t k, int32_t mode, uint64_t seed, int32_t *sel, int32_t *err,
                        void *stream);

/*
 * Exact softmax attention over the selected pages only (paper note, 系统设计 1: exact
 * attention on the chosen blocks; 系统设计 3: the MLA geometry kernel), gathered through
 * the page table.  For query head g of KV head h:
 *   out = sum_t softmax_t(sm_scale * q . K_t) V_t,  lse = log sum_t exp(sm_scale q . K_t)
 * over the valid tokens of the pages in sel[b][h] (entries < 0 skipped; entries must be
 * distinct).  Split-K: the selected tokens are cut into contiguous chunks whose partial
 * (o, max, sum) are merged, in chunk order, with the log-sum-exp rule.
 *   num_splits > 0: that many chunks of equal length (in 16-token tiles; MLA: pages).
 *   num_splits 0: planned from the SM count.  MLA: the fewest equal chunks, at most one per
 *   SM, that give no chunk more pages than one per SM would (128 for 512 pages on 148
 *   SMs).  GQA: one equal chunk per warp of a persistent grid (8 warps per SM); when a
 *   warp's share is 64 tiles or more, equal chunks per warp over the first three quarters
 *   of the tiles, then shorter equal chunks over the rest, each taken by whichever warp is
 *   free first.  The chunks are fixed before launch, so results never depend on timing.
 *   sm_scale <= 0 means 1 / sqrt(head_dim_qk).
 *   lse may be NULL.  A request with no attended token gets out = 0, lse = -inf.
 * ws: device workspace for the split partials; vx_workspace_size(geo, max_pages, k,
 * num_splits) bytes are always enough (that size also covers the fused call's scores
 * and selection, which this call does not use).  No initial contents needed: when the
 * planned split has late chunks, the call first zeroes their counter, one word of ws, with
 * a 4-byte cudaMemsetAsync on `stream`.
 */
vx_status vx_sparse_decode(const vx_geometry *geo, const vx_page_table *table, const void *q,
                           const void *k_cache, const void *v_cache, const int32_t *sel, int32_t k,
                           float sm_scale, int32_t num_splits, void *out, float *lse, void *ws,
                           size_t ws_bytes, int32_t *err, void *stream);

/*
 * Flag OR-ed into the mode of the two chained steps below.  It promises that the page table
 * (page_ptr, page_indices) and seq_lens were not written by the last kernel launched on the
 * stream before the call (they came from host copies, or from an earlier kernel).  The
 * scorer then reads them, and fetches the first page ids of its range, while that kernel
 * is still finishing; q, the centroids and the caches are still read only after it has
 * completed.  Without the flag every read waits for it.  Results are the same either way.
 * A call whose table or lengths the previous kernel writes must not set the flag: the scorer
 * could read them before they are written.
 */
#define VX_TABLE_READY 0x100

/*
 * One whole decode step: vx_score_pages -> vx_topk_pages -> vx_sparse_decode, chained
 * on `stream` with programmatic dependent launch so each kernel's start overlaps the
 * previous one's tail (paper note, 系统设计 3: fusion of the sequence-local steps and
 * workload planning).  Same arguments and results as the three calls.  scores_out and
 * sel_out (may be NULL) receive the intermediate scores and selection; when NULL they
 * live in the workspace.  score_dims as in vx_score_pages.  ws: vx_workspace_size bytes,
 * no initial contents needed.
 * mode: vx_topk_pages's mode (0..3), optionally OR-ed with VX_TABLE_READY.
 */
vx_status vx_block_topk_decode(const vx_geometry *geo, const vx_page_table *table, const void *q,
                               const void *k_cache, const void *v_cache, const void *centroids,
                               int32_t k, int32_t mode, uint64_t seed, float sm_scale,
                               int32_t score_dims, int32_t num_splits, void *out, float *lse,
                               float *scores_out, int32_t *sel_out, void *ws, size_t ws_bytes,
                               int32_t *err, void *stream);

/*
 * One continuous-batching decode step: every request appends one token and then decodes
 * (paper note, 系统设计 1: the cache stage keeps each page's centroid as tokens arrive;
 * 系统设计 3: fusion of the sequence-local steps).  The append of vx_centroid_update
 * (k_new, first_pos NULL) runs first: each request's new token (k_new [B][Hkv][Dqk],
 * v_new [B][Hkv][Dv], v_new ignored for MLA) goes into slot (seq_lens[b]-1) % P of its
 * page, whose centroid is recomputed from its keys; seq_lens already counts the new token
 * and its page is installed in the table.  Then vx_block_topk_decode's score -> top-k ->
 * attention chain runs on the same stream, its first kernel launched with programmatic
 * dependent launch behind the append, so it starts while the append drains.  Arguments
 * and results as in vx_centroid_update plus vx_block_topk_decode; same workspace size.
 * mode may carry VX_TABLE_READY (the append itself never writes the table or lengths).
 */
vx_status vx_block_topk_decode_append(const vx_geometry *geo, const vx_page_table *table, const void *q,
                                      void *k_cache, void *v_cache, void *centroids, const void *k_new,
                                      const void *v_new, int32_t k, int32_t mode, uint64_t seed,
                                      float sm_scale, int32_t score_dims, int32_t num_splits, void *out,
                                      float *lse, float *scores_out, int32_t *sel_out, void *ws,
                                      size_t ws_bytes, int32_t *err, void *stream);

/*
 * The same decode step (exact top-k, full score dims) as ONE persistent kernel (paper note,
 * 系统设计 3: fusion and workload planning, taken to a single launch).  Its warps take work
 * items from two ticket counters: score a span of one request's pages, attend a span of
 * one (request, KV head) row's selected tiles (the row's last span merges the row), and,
 * in request order, select one row (exact radix top-k on a warp, ties to the lower page).
 * Every wait is on a smaller ticket or is helped along by the waiting warp, and is bounded
 * (a timeout sets VX_DATA_TIMEOUT), so the launch always ends.
 *   Geometry: GQA with head_dim_qk == head_dim_v in {64, 128}, num_kv_heads <= 16, at
 *   most 16 query heads per KV head, batch <= 1024 (else VX_ERR_UNSUPPORTED).
 *   Results: the same scores and selection bits as vx_block_topk_decode with mode 0; out
 *   and lse differ only by rounding (its own split of the attention).
 *   Speed: slower than vx_block_topk_decode on B200 for the workloads measured here (its
 *   warp-level selection is the bottleneck); kept for study and as the fused reference.
 * ws: vx_workspace_size(geo, max_pages, k, 0) bytes.  ZERO-FILL IT ONCE before its first
 * use here (e.g. cudaMemset after allocating): its first bytes hold the kernel's counters,
 * which every call leaves zero again.  No other entry point writes them, so one workspace
 * may serve every call (one call at a time).
 */
vx_status vx_block_topk_decode_persistent(const vx_geometry *geo, const vx_page_table *table, const void *q,
                                          const void *k_cache, const void *v_cache, const void *centroids,
                                          int32_t k, float sm_scale, void *out, float *lse, float *scores_out,
                                          int32_t *sel_out, void *ws, size_t ws_bytes, int32_t *err,
                                          void *stream);

/*
 * vx_sparse_decode without a caller workspace, for callers that cannot allocate device
 * memory.  This entry point has no counterpart in the paper; it exists for integration.
 * Who needs it: an inference engine that gives all free HBM to its KV-cache pool at
 * start-up and allows no later cudaMalloc, a plugin interface that hands over tensors but
 * no workspace, or a caller that must avoid the device synchronisation cudaMalloc and
 * cudaFree can cause.
 * What it does: exactly vx_sparse_decode (same arguments minus ws / ws_bytes, same
 * kernels, same split plan, so bit-identical results for the same num_splits), with the
 * split partials kept in one array of VX_NOALLOC_SCRATCH_BYTES that the library holds in
 * device memory, once per GPU, until the process exits.  It calls no cudaMalloc, cudaFree
 * or other allocating routine.
 *   - Limit: with W the chunk count after planning (num_splits, or vx_planned_splits for
 *     0, at most the number of tiles) and rows = batch * num_kv_heads, the partials take
 *     round_up_256((rows + W) * G * head_dim_v * 4) + (rows + W) * G * 2 * 4 bytes.  A
 *     problem that needs more than VX_NOALLOC_SCRATCH_BYTES is rejected with
 *     VX_ERR_WORKSPACE and a message; pass fewer splits or use vx_sparse_decode with your
 *     own workspace.
 *   - Set-up and memory: the array is placed in device memory when the part of the
 *     library that holds it is loaded on a device.  Under CUDA's default lazy module
 *     loading that is the first call of this function on the device, which therefore
 *     needs VX_NOALLOC_SCRATCH_BYTES of free device memory; the same call looks the
 *     array's device address up (cudaGetSymbolAddress, with that device current; again
 *     after a device reset).  A caller that reserves all free memory for its KV pool
 *     makes one call on each device before reserving it (or sets
 *     CUDA_MODULE_LOADING=EAGER), and makes that first call before any stream capture.
 *   - Sharing: every call on a device uses the same array, which keeps whatever the last
 *     call left in it; nothing in it has to start at zero (a call writes each partial
 *     before reading it).  Calls that overlap on the GPU (two streams, or two host
 *     threads, at once) race on the array: order them on one stream.
 */
#define VX_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)
vx_status vx_sparse_decode_noalloc(const vx_geometry *geo, const vx_page_table *table, const void *q,
                                   const void *k_cache, const void *v_cache, const int32_t *sel,
                                   int32_t k, float sm_scale, int32_t num_splits, void *out,
                                   float *lse, int32_t *err, void *stream);

/*
 * Workspace bytes that vx_sparse_decode and vx_block_topk_decode need for this geometry,
 * row bound, k and split count (0 = the planned count); 0 when the arguments are
 * invalid (see vx_last_error).  Deterministic: the same inputs give the same size.  The
 * layout starts with a fixed-size counter region of the persistent fused step (see
 * vx_block_topk_decode_persistent: zero-fill a workspace once before its first use there).
 */
size_t vx_workspace_size(const vx_geometry *geo, int32_t max_pages, int32_t k, int32_t num_splits);

/* Number of chunks the planned split (num_splits = 0) makes on the current device for this
 * geometry.  Passing it as num_splits gives that many chunks of equal length instead. */
int32_t vx_planned_splits(const vx_geometry *geo, int32_t max_pages, int32_t k);

const char *vx_status_string(vx_status s);
const char *vx_last_error(void); /* message of the last failed call on this host thread */
const char *vx_version(void);

#ifdef __cplusplus
}
#endif
#endif /* VX_H */
