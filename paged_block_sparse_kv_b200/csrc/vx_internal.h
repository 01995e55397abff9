// vx_internal.h -- argument blocks and launch entry points shared by the libvx sources.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <utility>

#include "vx_common.cuh"

namespace vx {

// ------------------------------------------------------------------ tunables
constexpr int CEN_WARPS = 8;             // centroid rebuild: warps per block
constexpr int CEN_PAGES_PER_BLOCK = 16;  // centroid rebuild: pages per block
constexpr int SCORE_WARPS = 8;           // scoring: warps per block
constexpr int SCORE_UNROLL = 4;          // scoring: pages in flight per warp
constexpr int SCORE_PAGES_PER_BLOCK = SCORE_WARPS * SCORE_UNROLL * 2;
constexpr int TOPK_THREADS = 1024;       // top-k: one block per (request, KV head) row
constexpr int TOPK_SMEM_KEYS = 12288;    // rows up to this many pages keep their keys in smem
constexpr int APPROX_BITS = 12;          // approximate top-k remap width
constexpr int APPROX_BITS_FAST = 10;     // approximate top-k, mode 2: 1024 codes
constexpr int APPROX_BITS_COARSE = 8;    // approximate top-k, mode 3: 256 codes
constexpr int DEC_WARPS = 8;             // GQA decode: worker warps per block
constexpr int DEC_STAGES = 3;            // GQA decode: 16-token tiles in flight per warp
constexpr int DEC_TILE = 16;             // GQA decode: tokens per tile (one mma M or K step)
constexpr int DEC_DYN_PCT = 25;          // GQA decode, planned split: % of tiles handed out late
constexpr int DEC_DYN_DIV = 8;           // ... in pieces of 1 / DEC_DYN_DIV of a warp's share of tiles
constexpr int DEC_DYN_MIN_PIECE = 8;     // ... only when such a piece has at least this many tiles
constexpr int MLA_MIN_PAGE = 32;         // MLA decode: pages of 32 or 64 tokens
constexpr int MLA_TILE_ROWS = 64;        // MLA decode: tokens per tile (a page of up to 64 tokens)

// ------------------------------------------------------------------ argument blocks
struct TableArgs {
    const int32_t *page_ptr;
    const int32_t *page_indices;
    const int32_t *seq_lens;
};

struct CentroidArgs {
    const int32_t *page_ptr, *page_indices, *seq_lens, *first_pos;
    void *k_cache, *v_cache, *centroids;
    const void *k_new, *v_new;
    int32_t *err;
    int32_t B, Hkv, Dqk, Dv, P, max_pages, mla_shared_kv;
    int64_t num_pool_pages;
};

struct ScoreArgs {
    const int32_t *page_ptr, *page_indices, *seq_lens;
    const __nv_bfloat16 *q, *centroids;
    float *scores;
    int32_t *err;
    int32_t B, Hq, Hkv, G, Dqk, P, max_pages, score_dims;
    int32_t qcap;             // requests whose summed query a block keeps in shared memory
    int32_t table_ready;      // the table and lengths may be read before the dependency wait
    uint32_t *zero_word;      // NULL, or a word block 0 sets to zero after the dependency wait
    int64_t num_pool_pages;
};

struct TopkArgs {
    const int32_t *seq_lens;
    const float *scores;
    int32_t *sel;
    int32_t *err;
    int32_t B, Hkv, P, max_pages, k, smem_keys;
    int32_t warp_max;  // exact rows of at most this many pages go to one warp (0: none)
    uint64_t seed;
};

struct DecodeArgs {
    const int32_t *page_ptr, *page_indices, *seq_lens, *sel;
    const __nv_bfloat16 *q;
    float *o_part;   // [slots][G][Dv] unnormalised partial outputs
    float *ml_part;  // [slots][G][2]  (running max in log2 units, running sum)
    __nv_bfloat16 *out;
    float *lse;
    int32_t *err;
    int32_t B, Hq, Hkv, G, Dqk, Dv, P, max_pages, k;
    int32_t tiles_per_page;   // P / DEC_TILE (GQA) or 1 (MLA: one page per unit)
    int64_t num_pool_pages;
    int64_t units;            // rows * k * tiles_per_page
    int64_t units_per_row;    // k * tiles_per_page
    // pieces (`chunks` in all): the first static_chunks split units [0, static_units) evenly,
    // the rest split [static_units, units) evenly (see piece_start)
    int64_t static_units;
    int32_t static_chunks;
    uint32_t *piece_ctr;      // NULL: warp w takes pieces w, static_chunks + w, + 2 static_chunks ...;
                              // else pieces past the first static_chunks come from this counter (zero at launch)
    int32_t chunks;           // split count W
    float scale_log2;         // sm_scale * log2(e)
};

// One decode work unit (a 16-token tile of a selected page) after its metadata has been
// looked up: row, tensor-map page(-head) index, token offset in the page, valid tokens.
struct Resolved {
    int32_t row, z, y, nvalid;
    bool valid;
};

// ------------------------------------------------------------------ launches
// Persistent fused step (GQA geometry, exact top-k): one launch scores, selects and attends.
// Streaming work items (score a span of one request's pages, attend a span of one row's
// tiles) come in ticket order from one counter; top-k rows, in request order, from a second
// one, taken first by the warps of the first t_blocks blocks (and by any attention item whose
// row is not taken yet).  `sync` is a fixed-size region of FUSED_SYNC_WORDS uint32 at the start
// of the workspace: [ticket, blocks_done, abort, row_ticket, scored[FUSED_MAX_B],
// row_ready[FUSED_MAX_B * FUSED_MAX_HKV], row_done[FUSED_MAX_B * FUSED_MAX_HKV]].  It is zero
// before a launch and the last block to finish clears what the launch used.
constexpr int FUSED_WARPS = 8;
constexpr int FUSED_MAX_B = 1024;
constexpr int FUSED_MAX_HKV = 16;
constexpr int FUSED_SYNC_HDR = 4;
constexpr size_t FUSED_SYNC_WORDS =
    FUSED_SYNC_HDR + (size_t)FUSED_MAX_B + 2 * (size_t)FUSED_MAX_B * FUSED_MAX_HKV;
struct FusedArgs {
    const int32_t *page_ptr, *page_indices, *seq_lens;
    const __nv_bfloat16 *q, *centroids;
    float *scores;            // [B][Hkv][max_pages]
    int32_t *sel;             // [B][Hkv][k]
    float *o_part;            // [slots][G][D] unnormalised partial outputs
    float *ml_part;           // [slots][G][2] (running max in log2 units, running sum)
    __nv_bfloat16 *out;
    float *lse;
    int32_t *err;
    uint32_t *sync;
    int32_t B, Hq, Hkv, G, D, P, max_pages, k;
    int32_t tiles_per_page;   // P / DEC_TILE
    int32_t spages;           // pages per score item (<= 32)
    int32_t dtiles;           // tiles per attention item
    int32_t t_blocks;         // blocks whose warps start on top-k rows
    int32_t dlag;             // attention items of request r join the ticket order at round r + dlag
    int64_t num_pool_pages;
    float scale_log2;         // sm_scale * log2(e)
};

constexpr int CEN_REBUILD = 0, CEN_APPEND = 1, CEN_PREFILL = 2;  // vx_centroid_update modes
cudaError_t launch_centroid(const CentroidArgs &a, int mode, cudaStream_t s);
cudaError_t launch_score(const ScoreArgs &a, cudaStream_t s, bool pdl);
cudaError_t launch_topk(const TopkArgs &a, int mode, cudaStream_t s, bool pdl);
cudaError_t launch_decode_gqa(const DecodeArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV,
                              int grid, cudaStream_t s, bool pdl);
// grid = split count (one CTA per split); tmQ views q as (64 columns, rows = batch * Hq, 9 blocks)
cudaError_t launch_decode_mla(const DecodeArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmQ, int grid,
                              cudaStream_t s, bool pdl);
cudaError_t launch_merge(const DecodeArgs &a, cudaStream_t s, bool pdl);
// grid = SM count (one block of FUSED_WARPS warps per SM)
cudaError_t launch_fused(const FusedArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV, cudaStream_t s);
// shared memory the fused kernel needs for a batch of B (0 if it cannot run it)
size_t fused_smem_bytes(int32_t B);

// Host helpers of the C ABI layer (vx_api.cu).
// Bytes of split partials vx_sparse_decode needs for this problem (validates the geometry).
vx_status decode_partial_bytes(const vx_geometry *geo, int32_t max_pages, int32_t k, int32_t num_splits,
                               size_t *bytes);
// Set the message vx_last_error() returns on this host thread; returns s.
vx_status set_error(vx_status s, const char *msg);
// Bytes of split partials of the sparse decode with the partials packed alone (outputs
// [rows + W][G][Dv] fp32, rounded up to 256 bytes, then (max, sum) [rows + W][G][2] fp32),
// W = the resolved split count.  Validates the geometry.
vx_status compact_partial_bytes(const vx_geometry *geo, int32_t max_pages, int32_t k, int32_t num_splits,
                                size_t *bytes);
// The sparse decode (same validation and kernels as vx_sparse_decode) with its split
// partials in `partials`, laid out as compact_partial_bytes describes.
vx_status sparse_decode_compact(const vx_geometry *geo, const vx_page_table *table, const void *q,
                                const void *k_cache, const void *v_cache, const int32_t *sel, int32_t k,
                                float sm_scale, int32_t num_splits, void *out, float *lse, void *partials,
                                size_t partial_bytes, int32_t *err, cudaStream_t stream);

// Launch with programmatic dependent launch enabled when `pdl` (the kernel must call
// pdl_wait() before reading what the previous kernel on the stream wrote).
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                     bool pdl, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// Raise a kernel's dynamic shared-memory limit once per device (the attribute is per
// device; the first launch on each device sets it).
template <typename F>
cudaError_t ensure_smem_limit(F kern, int bytes, std::atomic<unsigned long long> &done) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return e;
}

// chunk c of W covers units [c*T/W, (c+1)*T/W)
__host__ __device__ __forceinline__ int64_t chunk_start(int64_t c, int64_t T, int64_t W) {
    return (c * T) / W;
}
// the chunk holding unit u
__host__ __device__ __forceinline__ int64_t chunk_of(int64_t u, int64_t T, int64_t W) {
    return ((u + 1) * W - 1) / T;
}

// Pieces of the decode split: pieces 0 .. Ws-1 cut units [0, Us) into Ws equal chunks, pieces
// Ws .. W-1 cut [Us, T) into W - Ws equal chunks (Us == T and Ws == W: the plain even split).
// Every piece holds at least one unit; pieces are contiguous and in unit order, so slot
// (row + piece) is unique for every (row, piece) pair that shares a unit.
__host__ __device__ __forceinline__ int64_t piece_start(int64_t c, int64_t T, int64_t Us, int64_t Ws, int64_t W) {
    return c <= Ws ? chunk_start(c, Us, Ws) : Us + chunk_start(c - Ws, T - Us, W - Ws);
}
__host__ __device__ __forceinline__ int64_t piece_of(int64_t u, int64_t T, int64_t Us, int64_t Ws, int64_t W) {
    return u < Us ? chunk_of(u, Us, Ws) : Ws + chunk_of(u - Us, T - Us, W - Ws);
}

}  // namespace vx
