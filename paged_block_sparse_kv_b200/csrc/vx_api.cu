// vx_api.cu -- the C ABI of libvx (include/vx.h): validation, planning, launches.
//
// Host validation runs before anything is launched and touches no CUDA state, so bad
// arguments fail the same way with or without a GPU.  Workload planning (paper note,
// section 系统设计 3) picks the split count from the SM count: one persistent block of
// DEC_WARPS worker warps per SM for GQA, one tensor-core CTA per SM for MLA.
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "vx_internal.h"

namespace {

thread_local std::string g_last_error;

vx_status fail(vx_status s, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
vx_status fail(vx_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

vx_status cuda_fail(cudaError_t e, const char *where) {
    return fail(VX_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool al16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool al4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

// ------------------------------------------------------------------ validation

vx_status check_geometry(const vx_geometry *g) {
    if (!g) return fail(VX_ERR_INVALID_ARG, "geometry is NULL");
    if (g->batch < 1) return fail(VX_ERR_INVALID_ARG, "batch %d < 1", g->batch);
    if (g->num_kv_heads < 1 || g->num_q_heads < 1)
        return fail(VX_ERR_INVALID_ARG, "head counts must be >= 1 (q %d, kv %d)", g->num_q_heads, g->num_kv_heads);
    if (g->num_q_heads % g->num_kv_heads)
        return fail(VX_ERR_INVALID_ARG, "num_q_heads %d is not a multiple of num_kv_heads %d", g->num_q_heads,
                    g->num_kv_heads);
    if (g->num_pool_pages < 1) return fail(VX_ERR_INVALID_ARG, "num_pool_pages must be >= 1");
    if (g->page_size < 1 || g->head_dim_qk < 1 || g->head_dim_v < 1)
        return fail(VX_ERR_INVALID_ARG, "page_size and head dims must be >= 1");
    if (g->num_pool_pages * (int64_t)g->num_kv_heads > INT32_MAX)
        return fail(VX_ERR_INVALID_ARG, "num_pool_pages * num_kv_heads overflows int32");
    const int G = g->num_q_heads / g->num_kv_heads;
    if (g->page_size != 16 && g->page_size != 32 && g->page_size != 64)
        return fail(VX_ERR_UNSUPPORTED, "page_size %d not built (16, 32, 64)", g->page_size);
    if (g->batch > 4096) return fail(VX_ERR_UNSUPPORTED, "batch %d > 4096 not built", g->batch);
    if (g->mla_shared_kv) {
        if (g->num_kv_heads != 1 || g->head_dim_qk != 576 || g->head_dim_v != 512)
            return fail(VX_ERR_UNSUPPORTED, "MLA geometry must be 1 KV head, head_dim_qk 576, head_dim_v 512");
        if (G > 16) return fail(VX_ERR_UNSUPPORTED, "MLA supports at most 16 query heads (got %d)", G);
        if (g->page_size % vx::MLA_MIN_PAGE)
            return fail(VX_ERR_UNSUPPORTED, "MLA page_size must be 32 or 64 (got %d)", g->page_size);
    } else {
        if (g->head_dim_qk != g->head_dim_v) return fail(VX_ERR_UNSUPPORTED, "GQA needs head_dim_qk == head_dim_v");
        if (g->head_dim_qk != 64 && g->head_dim_qk != 128)
            return fail(VX_ERR_UNSUPPORTED, "GQA head_dim %d not built (64, 128)", g->head_dim_qk);
        if (G > 16) return fail(VX_ERR_UNSUPPORTED, "GQA group size %d > 16 not built", G);
        const int hkv = g->num_kv_heads;
        if (hkv > 16 || (hkv & (hkv - 1)))
            return fail(VX_ERR_UNSUPPORTED, "GQA num_kv_heads %d not built (a power of two <= 16)", hkv);
    }
    return VX_OK;
}

vx_status check_max_pages(const vx_geometry *g, int32_t max_pages) {
    if (max_pages < 1) return fail(VX_ERR_INVALID_ARG, "max_pages must be >= 1");
    if ((int64_t)max_pages * g->page_size > INT32_MAX)
        return fail(VX_ERR_INVALID_ARG, "max_pages * page_size overflows int32");
    return VX_OK;
}

vx_status check_geo(const vx_geometry *g, const vx_page_table *t) {
    vx_status s = check_geometry(g);
    if (s != VX_OK) return s;
    if (!t) return fail(VX_ERR_INVALID_ARG, "page table is NULL");
    if (!t->page_ptr || !t->page_indices || !t->seq_lens)
        return fail(VX_ERR_INVALID_ARG, "page table arrays must not be NULL");
    if (!al4(t->page_ptr) || !al4(t->page_indices) || !al4(t->seq_lens))
        return fail(VX_ERR_INVALID_ARG, "page table arrays must be 4-byte aligned");
    return check_max_pages(g, t->max_pages);
}

vx_status check_ptr(const void *p, const char *name, bool can_be_null = false) {
    if (!p) return can_be_null ? VX_OK : fail(VX_ERR_INVALID_ARG, "%s is NULL", name);
    if (!al16(p)) return fail(VX_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    return VX_OK;
}

#define VX_TRY(x)                          \
    do {                                   \
        vx_status _s = (x);                \
        if (_s != VX_OK) return _s;        \
    } while (0)

// ------------------------------------------------------------------ device facts

// SM count per device ordinal, looked up once; several host threads may race to fill an
// entry, and they all store the same value.
int sm_count_current(int *out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    static std::atomic<int> cache[64];
    if (dev < 64) {
        const int c = cache[dev].load(std::memory_order_relaxed);
        if (c > 0) {
            *out = c;
            return 0;
        }
    }
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) return -1;
    if (dev < 64) cache[dev].store(n, std::memory_order_relaxed);
    *out = n;
    return 0;
}

// ------------------------------------------------------------------ planning

struct Plan {
    int64_t rows, units, units_per_row;
    int64_t static_units;  // pieces 0 .. static_chunks-1 split [0, static_units); the rest the remainder
    int32_t tiles_per_page, chunks, static_chunks, grid;
    int G;
    bool mla;
};


vx_status plan(const vx_geometry *g, int32_t k, int32_t num_splits, Plan *p) {
    p->mla = g->mla_shared_kv != 0;
    p->G = g->num_q_heads / g->num_kv_heads;
    p->rows = (int64_t)g->batch * g->num_kv_heads;
    p->tiles_per_page = g->page_size / (p->mla ? std::min(g->page_size, vx::MLA_TILE_ROWS) : vx::DEC_TILE);
    p->units_per_row = (int64_t)k * p->tiles_per_page;
    p->units = p->rows * p->units_per_row;
    const bool planned = num_splits <= 0;
    int64_t w = num_splits;
    if (planned) {
        int sms = 0;
        if (sm_count_current(&sms) != 0) return fail(VX_ERR_CUDA, "cannot query the current device's SM count");
        w = p->mla ? (int64_t)sms : (int64_t)sms * vx::DEC_WARPS;  // MLA: one CTA per SM
    }
    if (w > p->units) w = p->units;
    if (w < 1) w = 1;
    if (planned && p->mla) {
        // the fewest CTAs that keep the most tiles a CTA gets: 512 pages on 148 SMs take 4 each
        // on 128 CTAs as on 148, with fewer partials to merge (32.6 vs 33.5 us per MLA step)
        const int64_t per = (p->units + w - 1) / w;
        w = (p->units + per - 1) / per;
    }
    if (w > INT32_MAX / 2) return fail(VX_ERR_INVALID_ARG, "num_splits too large");
    // an explicit split count, and MLA: w equal chunks.  The planned GQA split, when a warp's
    // share is long enough (DEC_DYN_DIV * DEC_DYN_MIN_PIECE tiles or more): one equal chunk per
    // warp over the first (100 - DEC_DYN_PCT)% of the tiles, then pieces of 1 / DEC_DYN_DIV of
    // a warp's share over the rest, taken by whichever warp is free first.  Shorter shares keep
    // the even split: a warp switching pieces re-resolves pages and reloads its query, which
    // costs more than the balance gains (measured: 86.0 against 75.7 us per headline step with
    // 3-tile pieces; 319.3 against 330.8 us on continuous batching with 13-tile pieces)
    int64_t ws_ = w, us = p->units, wd = 0;
    if (planned && !p->mla) {
        const int64_t piece = p->units / w / vx::DEC_DYN_DIV;
        const int64_t ud = p->units * vx::DEC_DYN_PCT / 100;
        wd = piece >= vx::DEC_DYN_MIN_PIECE ? ud / piece : 0;
        if (wd >= 1 && p->units - ud >= w && (int64_t)w + wd <= INT32_MAX / 2) {
            us = p->units - ud;
        } else {
            wd = 0;
        }
    }
    p->static_units = us;
    p->static_chunks = static_cast<int32_t>(ws_);
    p->chunks = static_cast<int32_t>(ws_ + wd);
    p->grid = p->mla ? p->chunks : (p->static_chunks + vx::DEC_WARPS - 1) / vx::DEC_WARPS;
    return VX_OK;
}

// The persistent fused step (GQA geometry, exact top-k, planned splits): its work-item sizes.
struct FusedPlan {
    bool ok;               // the geometry and batch fit the fused kernel
    int32_t spages;        // pages per score item
    int32_t dtiles;        // tiles per attention item
    int32_t t_blocks;      // blocks whose warps start on top-k rows
    int32_t dlag;          // rounds between a request's score items and its attention items
    int64_t slots;         // partial slots it may use (rows * items per row, at most)
};

constexpr int FUSED_SPAGES = 16;
constexpr double FUSED_LAG_BYTES = 120e6;
constexpr int FUSED_MAX_ITEMS_PER_ROW = 16;

FusedPlan fused_plan(const vx_geometry *g, int32_t max_pages, int32_t k) {
    FusedPlan f{false, FUSED_SPAGES, 0, 0, 1, 0};
    const int Hkv = g->num_kv_heads, D = g->head_dim_qk;
    const int G = g->num_q_heads / Hkv;
    const int lanes_per_page = Hkv * 2;  // a head row is split over 2 lanes (64 dims at D = 128, 32 at D = 64)
    if (g->mla_shared_kv || g->head_dim_v != D || (D != 64 && D != 128) || g->batch > vx::FUSED_MAX_B ||
        Hkv > vx::FUSED_MAX_HKV || lanes_per_page > 32 || 32 % lanes_per_page || G > 16 ||
        g->page_size % vx::DEC_TILE)
        return f;
    int sms = 0;
    if (sm_count_current(&sms) != 0 || sms < 1) return f;
    const int64_t tpp = g->page_size / vx::DEC_TILE;
    const int64_t row_tiles = (int64_t)std::min(k, max_pages) * tpp;
    const int64_t rows = (int64_t)g->batch * Hkv;
    // about one attention item per warp, 8..64 tiles, at most 16 items per row
    int64_t want = std::max<int64_t>(1, rows * row_tiles / ((int64_t)sms * vx::FUSED_WARPS));
    int64_t dt = 8;
    while (dt * 2 <= want && dt < 64) dt *= 2;
    while ((row_tiles + dt - 1) / dt > FUSED_MAX_ITEMS_PER_ROW) dt *= 2;
    const int64_t per_row = std::max<int64_t>(1, (row_tiles + dt - 1) / dt);
    // the merging warp keeps per_row x G weights and 2 G totals in its 24 KB region
    if ((per_row * G + 2 * G) * 4 > 16 * 1024) return f;
    f.ok = true;
    f.dtiles = static_cast<int32_t>(dt);
    f.slots = rows * per_row;
    // Attention items of request r are handed out about FUSED_LAG_BYTES of streaming after
    // its score items (about 20 us at HBM speed), so its rows are usually selected by then.
    const double req_bytes = (double)max_pages * Hkv * D * 2 +
                             (double)std::min(k, max_pages) * g->page_size * Hkv * 2.0 * D * 2;
    f.dlag = static_cast<int32_t>(std::min<double>(g->batch, std::max(1.0, std::ceil(FUSED_LAG_BYTES / req_bytes))));
    // Top-k blocks: enough warps for every row's selection to take about 40 us in total,
    // at an estimated 3 us + 1 us per 200 pages per row on a warp.
    const int64_t warp_us = rows * (3 + max_pages / 200);
    f.t_blocks = static_cast<int32_t>(std::min<int64_t>(std::min(24, sms / 4),
                                                        std::max<int64_t>(2, warp_us / (40 * vx::FUSED_WARPS))));
    return f;
}

// workspace layout, every region 256-byte aligned.  The fused step's sync words come first
// at a fixed size, so their place never depends on the batch or the page count.
struct WsLayout {
    size_t sync, scores, sel, dctr, o_part, ml_part, total;
};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

WsLayout ws_layout(const vx_geometry *g, int32_t max_pages, int32_t k, const Plan &p) {
    WsLayout l;
    const FusedPlan f = fused_plan(g, max_pages, k);
    const size_t slots = std::max<size_t>((size_t)(p.rows + p.chunks), f.ok ? (size_t)f.slots : 0);
    l.sync = 0;
    l.dctr = up256(vx::FUSED_SYNC_WORDS * sizeof(uint32_t));  // the decode's late-piece counter
    l.o_part = l.dctr + 256;
    l.ml_part = l.o_part + up256(slots * p.G * g->head_dim_v * sizeof(float));
    l.scores = l.ml_part + up256(slots * p.G * 2 * sizeof(float));
    l.sel = l.scores + up256((size_t)p.rows * max_pages * sizeof(float));
    l.total = l.sel + up256((size_t)p.rows * k * sizeof(int32_t));
    return l;
}

// bytes vx_sparse_decode uses: the split partials (the start of the layout)
size_t decode_ws_bytes(const WsLayout &l) { return l.scores; }

// ------------------------------------------------------------------ TMA descriptors

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// 3-D view [pages * heads][page_size][dim] of a bf16 cache, boxes of 64 dims x box_rows
// tokens x 1 page-head, 128-byte swizzle.
vx_status make_cache_map(CUtensorMap *map, const void *ptr, int dim, int page_size, int64_t page_heads,
                         int box_rows) {
    auto fn = encode_fn();
    if (!fn) return fail(VX_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t gdim[3] = {(cuuint64_t)dim, (cuuint64_t)page_size, (cuuint64_t)page_heads};
    cuuint64_t gstride[2] = {(cuuint64_t)dim * 2, (cuuint64_t)dim * 2 * page_size};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t estride[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), gdim, gstride, box, estride,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(VX_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return VX_OK;
}

// The query rows [batch * Hq][dim] as (64 columns, rows, dim / 64 blocks): a box of 16 rows
// lands as dim / 64 blocks of 16 rows x 128 bytes (128-byte swizzle), the layout of a
// K-major tensor-core operand with 16 rows.  Rows past the end read as zero.
vx_status make_query_map(CUtensorMap *map, const void *ptr, int dim, int64_t rows) {
    auto fn = encode_fn();
    if (!fn) return fail(VX_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t gdim[3] = {64, (cuuint64_t)rows, (cuuint64_t)(dim / 64)};
    cuuint64_t gstride[2] = {(cuuint64_t)dim * 2, 128};
    cuuint32_t box[3] = {64, 16, (cuuint32_t)(dim / 64)};
    cuuint32_t estride[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), gdim, gstride, box, estride,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(VX_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return VX_OK;
}

// A tile of box_rows token rows in one copy, laid out as the per-64-column boxes of
// make_cache_map: the 4-D view (64 columns, rows, dim / 64 column blocks, page-heads) puts
// the column block outside the rows, so shared memory receives block 0's box_rows x 128
// bytes, then block 1's, each 128-byte row swizzled by its row index.
vx_status make_cache_map_blocks(CUtensorMap *map, const void *ptr, int dim, int page_size, int64_t page_heads,
                                int box_rows) {
    auto fn = encode_fn();
    if (!fn) return fail(VX_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
    cuuint64_t gdim[4] = {64, (cuuint64_t)page_size, (cuuint64_t)(dim / 64), (cuuint64_t)page_heads};
    cuuint64_t gstride[3] = {(cuuint64_t)dim * 2, 128, (cuuint64_t)dim * 2 * page_size};
    cuuint32_t box[4] = {64, (cuuint32_t)box_rows, (cuuint32_t)(dim / 64), 1};
    cuuint32_t estride[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(ptr), gdim, gstride, box, estride,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(VX_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return VX_OK;
}

// ------------------------------------------------------------------ shared launch pieces

// piece_ctr: NULL, or a workspace word zeroed earlier on the stream (by the step's scorer or a
// memset); late pieces are then handed out to whichever warp is free first
vx_status do_decode(const vx_geometry *g, const vx_page_table *t, const void *q, const void *k_cache,
                    const void *v_cache, const int32_t *sel, int32_t k, float sm_scale, const Plan &p,
                    const WsLayout &l, void *ws, void *out, float *lse, int32_t *err, cudaStream_t s, bool pdl,
                    uint32_t *piece_ctr = nullptr) {
    vx::DecodeArgs a{};
    a.page_ptr = t->page_ptr;
    a.page_indices = t->page_indices;
    a.seq_lens = t->seq_lens;
    a.sel = sel;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.o_part = reinterpret_cast<float *>(static_cast<char *>(ws) + l.o_part);
    a.ml_part = reinterpret_cast<float *>(static_cast<char *>(ws) + l.ml_part);
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.lse = lse;
    a.err = err;
    a.B = g->batch;
    a.Hq = g->num_q_heads;
    a.Hkv = g->num_kv_heads;
    a.G = p.G;
    a.Dqk = g->head_dim_qk;
    a.Dv = g->head_dim_v;
    a.P = g->page_size;
    a.max_pages = t->max_pages;
    a.k = k;
    a.tiles_per_page = p.tiles_per_page;
    a.num_pool_pages = g->num_pool_pages;
    a.units = p.units;
    a.units_per_row = p.units_per_row;
    a.chunks = p.chunks;
    a.static_units = p.static_units;
    a.static_chunks = p.static_chunks;
    a.piece_ctr = piece_ctr;
    const float scale = sm_scale > 0.f ? sm_scale : 1.0f / std::sqrt((float)g->head_dim_qk);
    a.scale_log2 = scale * 1.4426950408889634f;
    const int64_t page_heads = g->num_pool_pages * g->num_kv_heads;
    cudaError_t e;
    if (p.mla) {
        CUtensorMap tmK, tmQ;
        VX_TRY(make_cache_map_blocks(&tmK, k_cache, g->head_dim_qk, g->page_size, page_heads,
                                     g->page_size / p.tiles_per_page));
        VX_TRY(make_query_map(&tmQ, q, g->head_dim_qk, (int64_t)g->batch * g->num_q_heads));
        e = vx::launch_decode_mla(a, tmK, tmQ, p.grid, s, pdl);
    } else {
        CUtensorMap tmK, tmV;
        VX_TRY(make_cache_map_blocks(&tmK, k_cache, g->head_dim_qk, g->page_size, page_heads, vx::DEC_TILE));
        VX_TRY(make_cache_map_blocks(&tmV, v_cache, g->head_dim_v, g->page_size, page_heads, vx::DEC_TILE));
        e = vx::launch_decode_gqa(a, tmK, tmV, p.grid, s, pdl);
    }
    if (e != cudaSuccess) return cuda_fail(e, "sparse decode launch");
    e = vx::launch_merge(a, s, true);
    if (e != cudaSuccess) return cuda_fail(e, "merge launch");
    return VX_OK;
}

vx::ScoreArgs score_args(const vx_geometry *g, const vx_page_table *t, const void *q, const void *centroids,
                         int32_t score_dims, float *scores, int32_t *err) {
    vx::ScoreArgs a{};
    a.page_ptr = t->page_ptr;
    a.page_indices = t->page_indices;
    a.seq_lens = t->seq_lens;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.centroids = static_cast<const __nv_bfloat16 *>(centroids);
    a.scores = scores;
    a.err = err;
    a.B = g->batch;
    a.Hq = g->num_q_heads;
    a.Hkv = g->num_kv_heads;
    a.G = g->num_q_heads / g->num_kv_heads;
    a.Dqk = g->head_dim_qk;
    a.P = g->page_size;
    a.max_pages = t->max_pages;
    a.score_dims = score_dims > 0 ? score_dims : g->head_dim_qk;
    a.num_pool_pages = g->num_pool_pages;
    return a;
}

vx::TopkArgs topk_args(const vx_geometry *g, const vx_page_table *t, const float *scores, int32_t k, uint64_t seed,
                       int32_t *sel, int32_t *err) {
    vx::TopkArgs a{};
    a.seq_lens = t->seq_lens;
    a.scores = scores;
    a.sel = sel;
    a.err = err;
    a.B = g->batch;
    a.Hkv = g->num_kv_heads;
    a.P = g->page_size;
    a.max_pages = t->max_pages;
    a.k = k;
    a.smem_keys = t->max_pages < vx::TOPK_SMEM_KEYS ? t->max_pages : vx::TOPK_SMEM_KEYS;
    a.seed = seed;
    return a;
}

vx_status check_score_dims(const vx_geometry *g, int32_t score_dims) {
    if (score_dims < 0 || score_dims > g->head_dim_qk || (score_dims % 8) != 0)
        return fail(VX_ERR_INVALID_ARG, "score_dims %d must be 0 or a multiple of 8 in [8, head_dim_qk]", score_dims);
    return VX_OK;
}

vx_status check_k_mode(int32_t k, int32_t mode) {
    if (k < 1) return fail(VX_ERR_INVALID_ARG, "k %d < 1", k);
    if (mode < 0 || mode > 3)
        return fail(VX_ERR_INVALID_ARG,
                    "mode %d must be 0 (exact), 1 (approximate, 4096 codes), 2 (1024 codes) or 3 (256 codes)", mode);
    return VX_OK;
}

}  // namespace

namespace vx {

vx_status decode_partial_bytes(const vx_geometry *geo, int32_t max_pages, int32_t k, int32_t num_splits,
                               size_t *bytes) {
    VX_TRY(check_geometry(geo));
    VX_TRY(check_max_pages(geo, max_pages));
    VX_TRY(check_k_mode(k, 0));
    Plan p;
    VX_TRY(plan(geo, k, num_splits, &p));
    *bytes = decode_ws_bytes(ws_layout(geo, max_pages, k, p));
    return VX_OK;
}

vx_status set_error(vx_status s, const char *msg) {
    g_last_error = msg;
    return s;
}

vx_status compact_partial_bytes(const vx_geometry *geo, int32_t max_pages, int32_t k, int32_t num_splits,
                                size_t *bytes) {
    VX_TRY(check_geometry(geo));
    VX_TRY(check_max_pages(geo, max_pages));
    VX_TRY(check_k_mode(k, 0));
    Plan p;
    VX_TRY(plan(geo, k, num_splits, &p));
    const size_t slots = (size_t)(p.rows + p.chunks);
    *bytes = up256(slots * p.G * geo->head_dim_v * sizeof(float)) + slots * p.G * 2 * sizeof(float);
    return VX_OK;
}

vx_status sparse_decode_compact(const vx_geometry *geo, const vx_page_table *table, const void *q,
                                const void *k_cache, const void *v_cache, const int32_t *sel, int32_t k,
                                float sm_scale, int32_t num_splits, void *out, float *lse, void *partials,
                                size_t partial_bytes, int32_t *err, cudaStream_t stream) {
    VX_TRY(check_geo(geo, table));
    VX_TRY(check_ptr(q, "q"));
    VX_TRY(check_ptr(k_cache, "k_cache"));
    if (!geo->mla_shared_kv) VX_TRY(check_ptr(v_cache, "v_cache"));
    VX_TRY(check_ptr(sel, "sel"));
    VX_TRY(check_ptr(out, "out"));
    VX_TRY(check_ptr(lse, "lse", true));
    VX_TRY(check_k_mode(k, 0));
    if (err && !al4(err)) return fail(VX_ERR_INVALID_ARG, "err must be 4-byte aligned");
    if (!std::isfinite(sm_scale)) return fail(VX_ERR_INVALID_ARG, "sm_scale must be finite");
    Plan p;
    VX_TRY(plan(geo, k, num_splits, &p));
    const size_t slots = (size_t)(p.rows + p.chunks);
    WsLayout l{};
    l.o_part = 0;
    l.ml_part = up256(slots * p.G * geo->head_dim_v * sizeof(float));
    l.total = l.ml_part + slots * p.G * 2 * sizeof(float);
    if (!partials || !al16(partials)) return fail(VX_ERR_WORKSPACE, "partial buffer is NULL or not 16-byte aligned");
    if (partial_bytes < l.total)
        return fail(VX_ERR_WORKSPACE, "partial buffer of %zu bytes < %zu needed", partial_bytes, l.total);
    return do_decode(geo, table, q, k_cache, v_cache, sel, k, sm_scale, p, l, partials, out, lse, err, stream, false);
}

}  // namespace vx

// ==================================================================== C ABI

extern "C" {

const char *vx_status_string(vx_status s) {
    switch (s) {
        case VX_OK: return "VX_OK";
        case VX_ERR_INVALID_ARG: return "VX_ERR_INVALID_ARG";
        case VX_ERR_UNSUPPORTED: return "VX_ERR_UNSUPPORTED";
        case VX_ERR_WORKSPACE: return "VX_ERR_WORKSPACE";
        case VX_ERR_CUDA: return "VX_ERR_CUDA";
    }
    return "VX_UNKNOWN_STATUS";
}

const char *vx_last_error(void) { return g_last_error.c_str(); }

const char *vx_version(void) { return "libvx 0.1 (sm_100a)"; }

size_t vx_workspace_size(const vx_geometry *geo, int32_t max_pages, int32_t k, int32_t num_splits) {
    if (check_geometry(geo) != VX_OK || check_max_pages(geo, max_pages) != VX_OK) return 0;
    if (k < 1) {
        fail(VX_ERR_INVALID_ARG, "k %d < 1", k);
        return 0;
    }
    Plan p;
    if (plan(geo, k, num_splits, &p) != VX_OK) return 0;
    return ws_layout(geo, max_pages, k, p).total;
}

int32_t vx_planned_splits(const vx_geometry *geo, int32_t max_pages, int32_t k) {
    if (check_geometry(geo) != VX_OK || check_max_pages(geo, max_pages) != VX_OK) return 0;
    if (k < 1) {
        fail(VX_ERR_INVALID_ARG, "k %d < 1", k);
        return 0;
    }
    Plan p;
    if (plan(geo, k, 0, &p) != VX_OK) return 0;
    return p.chunks;
}

vx_status vx_centroid_update(const vx_geometry *geo, const vx_page_table *table, void *k_cache, void *v_cache,
                             void *centroids, const void *k_new, const void *v_new, const int32_t *first_pos,
                             int32_t *err, void *stream) {
    VX_TRY(check_geo(geo, table));
    VX_TRY(check_ptr(k_cache, "k_cache"));
    VX_TRY(check_ptr(centroids, "centroids"));
    // k_new with first_pos: a prefill chunk per request; k_new alone: one appended token
    const int mode = k_new ? (first_pos ? vx::CEN_PREFILL : vx::CEN_APPEND) : vx::CEN_REBUILD;
    if (k_new) {
        VX_TRY(check_ptr(k_new, "k_new"));
        if (!geo->mla_shared_kv) {
            VX_TRY(check_ptr(v_cache, "v_cache"));
            VX_TRY(check_ptr(v_new, "v_new"));
        }
    }
    if (first_pos && !al4(first_pos)) return fail(VX_ERR_INVALID_ARG, "first_pos must be 4-byte aligned");
    if (err && !al4(err)) return fail(VX_ERR_INVALID_ARG, "err must be 4-byte aligned");
    vx::CentroidArgs a{};
    a.page_ptr = table->page_ptr;
    a.page_indices = table->page_indices;
    a.seq_lens = table->seq_lens;
    a.first_pos = mode == vx::CEN_APPEND ? nullptr : first_pos;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.centroids = centroids;
    a.k_new = k_new;
    a.v_new = v_new;
    a.err = err;
    a.B = geo->batch;
    a.Hkv = geo->num_kv_heads;
    a.Dqk = geo->head_dim_qk;
    a.Dv = geo->head_dim_v;
    a.P = geo->page_size;
    a.max_pages = table->max_pages;
    a.mla_shared_kv = geo->mla_shared_kv;
    a.num_pool_pages = geo->num_pool_pages;
    cudaError_t e = vx::launch_centroid(a, mode, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "centroid launch");
    return VX_OK;
}

vx_status vx_score_pages(const vx_geometry *geo, const vx_page_table *table, const void *q, const void *centroids,
                         int32_t score_dims, float *scores, int32_t *err, void *stream) {
    VX_TRY(check_geo(geo, table));
    VX_TRY(check_ptr(q, "q"));
    VX_TRY(check_ptr(centroids, "centroids"));
    VX_TRY(check_ptr(scores, "scores"));
    VX_TRY(check_score_dims(geo, score_dims));
    if (err && !al4(err)) return fail(VX_ERR_INVALID_ARG, "err must be 4-byte aligned");
    cudaError_t e = vx::launch_score(score_args(geo, table, q, centroids, score_dims, scores, err),
                                     static_cast<cudaStream_t>(stream), false);
    if (e != cudaSuccess) return cuda_fail(e, "score launch");
    return VX_OK;
}

vx_status vx_topk_pages(const vx_geometry *geo, const vx_page_table *table, const float *scores, int32_t k,
                        int32_t mode, uint64_t seed, int32_t *sel, int32_t *err, void *stream) {
    VX_TRY(check_geo(geo, table));
    VX_TRY(check_ptr(scores, "scores"));
    VX_TRY(check_ptr(sel, "sel"));
    VX_TRY(check_k_mode(k, mode));
    if (err && !al4(err)) return fail(VX_ERR_INVALID_ARG, "err must be 4-byte aligned");
    cudaError_t e = vx::launch_topk(topk_args(geo, table, scores, k, seed, sel, err), mode,
                                    static_cast<cudaStream_t>(stream), false);
    if (e != cudaSuccess) return cuda_fail(e, "top-k launch");
    return VX_OK;
}

vx_status vx_sparse_decode(const vx_geometry *geo, const vx_page_table *table, const void *q, const void *k_cache,
                           const void *v_cache, const int32_t *sel, int32_t k, float sm_scale, int32_t num_splits,
                           void *out, float *lse, void *ws, size_t ws_bytes, int32_t *err, void *stream) {
    VX_TRY(check_geo(geo, table));
    VX_TRY(check_ptr(q, "q"));
    VX_TRY(check_ptr(k_cache, "k_cache"));
    if (!geo->mla_shared_kv) VX_TRY(check_ptr(v_cache, "v_cache"));
    VX_TRY(check_ptr(sel, "sel"));
    VX_TRY(check_ptr(out, "out"));
    VX_TRY(check_ptr(lse, "lse", true));
    VX_TRY(check_k_mode(k, 0));
    if (err && !al4(err)) return fail(VX_ERR_INVALID_ARG, "err must be 4-byte aligned");
    if (!std::isfinite(sm_scale)) return fail(VX_ERR_INVALID_ARG, "sm_scale must be finite");
    Plan p;
    VX_TRY(plan(geo, k, num_splits, &p));
    const WsLayout l = ws_layout(geo, table->max_pages, k, p);
    if (!ws || !al16(ws)) return fail(VX_ERR_WORKSPACE, "workspace is NULL or not 16-byte aligned");
    if (ws_bytes < decode_ws_bytes(l))
        return fail(VX_ERR_WORKSPACE, "workspace of %zu bytes < %zu needed", ws_bytes, decode_ws_bytes(l));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t *dctr = nullptr;
    if (p.chunks > p.static_chunks) {  // late pieces: zero their counter first
        dctr = reinterpret_cast<uint32_t *>(static_cast<char *>(ws) + l.dctr);
        const cudaError_t e = cudaMemsetAsync(dctr, 0, sizeof(uint32_t), s);
        if (e != cudaSuccess) return cuda_fail(e, "piece counter reset");
    }
    return do_decode(geo, table, q, k_cache, v_cache, sel, k, sm_scale, p, l, ws, out, lse, err, s, false, dctr);
}

}  // extern "C"

namespace {

// The chained step score -> top-k -> decode -> merge; `append` (k_new non-NULL) first writes
// each request's new token and recomputes its page's centroid, and the scorer then follows
// with programmatic dependent launch.
vx_status fused_step(const vx_geometry *geo, const vx_page_table *table, const void *q, const void *k_cache,
                     const void *v_cache, const void *centroids, void *k_cache_w, void *v_cache_w, void *centroids_w,
                     const void *k_new, const void *v_new, int32_t k, int32_t mode, uint64_t seed, float sm_scale,
                     int32_t score_dims, int32_t num_splits, void *out, float *lse, float *scores_out, int32_t *sel_out,
                     void *ws, size_t ws_bytes, int32_t *err, void *stream) {
    VX_TRY(check_geo(geo, table));
    VX_TRY(check_ptr(q, "q"));
    VX_TRY(check_ptr(k_cache, "k_cache"));
    if (!geo->mla_shared_kv) VX_TRY(check_ptr(v_cache, "v_cache"));
    VX_TRY(check_ptr(centroids, "centroids"));
    VX_TRY(check_ptr(out, "out"));
    VX_TRY(check_ptr(lse, "lse", true));
    VX_TRY(check_ptr(scores_out, "scores_out", true));
    VX_TRY(check_ptr(sel_out, "sel_out", true));
    const bool table_ready = (mode & VX_TABLE_READY) != 0;
    mode &= ~VX_TABLE_READY;
    VX_TRY(check_k_mode(k, mode));
    VX_TRY(check_score_dims(geo, score_dims));
    if (err && !al4(err)) return fail(VX_ERR_INVALID_ARG, "err must be 4-byte aligned");
    if (!std::isfinite(sm_scale)) return fail(VX_ERR_INVALID_ARG, "sm_scale must be finite");
    Plan p;
    VX_TRY(plan(geo, k, num_splits, &p));
    const WsLayout l = ws_layout(geo, table->max_pages, k, p);
    if (!ws || !al16(ws)) return fail(VX_ERR_WORKSPACE, "workspace is NULL or not 16-byte aligned");
    if (ws_bytes < l.total)
        return fail(VX_ERR_WORKSPACE, "workspace of %zu bytes < %zu needed", ws_bytes, l.total);
    if (k_new) {
        VX_TRY(check_ptr(k_new, "k_new"));
        if (!geo->mla_shared_kv) VX_TRY(check_ptr(v_new, "v_new"));
    }
    float *scores = scores_out ? scores_out : reinterpret_cast<float *>(static_cast<char *>(ws) + l.scores);
    int32_t *sel = sel_out ? sel_out : reinterpret_cast<int32_t *>(static_cast<char *>(ws) + l.sel);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (k_new) {
        vx::CentroidArgs ca{};
        ca.page_ptr = table->page_ptr;
        ca.page_indices = table->page_indices;
        ca.seq_lens = table->seq_lens;
        ca.first_pos = nullptr;
        ca.k_cache = k_cache_w;
        ca.v_cache = v_cache_w;
        ca.centroids = centroids_w;
        ca.k_new = k_new;
        ca.v_new = v_new;
        ca.err = err;
        ca.B = geo->batch;
        ca.Hkv = geo->num_kv_heads;
        ca.Dqk = geo->head_dim_qk;
        ca.Dv = geo->head_dim_v;
        ca.P = geo->page_size;
        ca.max_pages = table->max_pages;
        ca.mla_shared_kv = geo->mla_shared_kv;
        ca.num_pool_pages = geo->num_pool_pages;
        e = vx::launch_centroid(ca, vx::CEN_APPEND, s);
        if (e != cudaSuccess) return cuda_fail(e, "centroid append launch");
    }
    // the scorer may always launch early: before its dependency wait it reads nothing, or
    // (table_ready) only the page table and lengths
    uint32_t *dctr = reinterpret_cast<uint32_t *>(static_cast<char *>(ws) + l.dctr);
    vx::ScoreArgs sa = score_args(geo, table, q, centroids, score_dims, scores, err);
    sa.table_ready = table_ready ? 1 : 0;
    sa.zero_word = dctr;  // zeroed after the scorer's dependency wait, counted by the decode
    e = vx::launch_score(sa, s, true);
    if (e != cudaSuccess) return cuda_fail(e, "score launch");
    e = vx::launch_topk(topk_args(geo, table, scores, k, seed, sel, err), mode, s, true);
    if (e != cudaSuccess) return cuda_fail(e, "top-k launch");
    return do_decode(geo, table, q, k_cache, v_cache, sel, k, sm_scale, p, l, ws, out, lse, err, s, true,
                     p.chunks > p.static_chunks ? dctr : nullptr);
}

}  // namespace

extern "C" {

vx_status vx_block_topk_decode(const vx_geometry *geo, const vx_page_table *table, const void *q, const void *k_cache,
                               const void *v_cache, const void *centroids, int32_t k, int32_t mode, uint64_t seed,
                               float sm_scale, int32_t score_dims, int32_t num_splits, void *out, float *lse,
                               float *scores_out, int32_t *sel_out, void *ws, size_t ws_bytes, int32_t *err,
                               void *stream) {
    return fused_step(geo, table, q, k_cache, v_cache, centroids, nullptr, nullptr, nullptr, nullptr, nullptr, k, mode,
                      seed, sm_scale, score_dims, num_splits, out, lse, scores_out, sel_out, ws, ws_bytes, err,
                      stream);
}

vx_status vx_block_topk_decode_append(const vx_geometry *geo, const vx_page_table *table, const void *q,
                                      void *k_cache, void *v_cache, void *centroids, const void *k_new,
                                      const void *v_new, int32_t k, int32_t mode, uint64_t seed, float sm_scale,
                                      int32_t score_dims, int32_t num_splits, void *out, float *lse, float *scores_out,
                                      int32_t *sel_out, void *ws, size_t ws_bytes, int32_t *err, void *stream) {
    if (!k_new) return fail(VX_ERR_INVALID_ARG, "k_new is NULL (use vx_block_topk_decode for a step without append)");
    return fused_step(geo, table, q, k_cache, v_cache, centroids, k_cache, v_cache, centroids, k_new, v_new, k, mode,
                      seed, sm_scale, score_dims, num_splits, out, lse, scores_out, sel_out, ws, ws_bytes, err,
                      stream);
}

vx_status vx_block_topk_decode_persistent(const vx_geometry *geo, const vx_page_table *table, const void *q,
                                          const void *k_cache, const void *v_cache, const void *centroids, int32_t k,
                                          float sm_scale, void *out, float *lse, float *scores_out, int32_t *sel_out,
                                          void *ws, size_t ws_bytes, int32_t *err, void *stream) {
    VX_TRY(check_geo(geo, table));
    VX_TRY(check_ptr(q, "q"));
    VX_TRY(check_ptr(k_cache, "k_cache"));
    VX_TRY(check_ptr(v_cache, "v_cache"));
    VX_TRY(check_ptr(centroids, "centroids"));
    VX_TRY(check_ptr(out, "out"));
    VX_TRY(check_ptr(lse, "lse", true));
    VX_TRY(check_ptr(scores_out, "scores_out", true));
    VX_TRY(check_ptr(sel_out, "sel_out", true));
    VX_TRY(check_k_mode(k, 0));
    if (geo->mla_shared_kv) return fail(VX_ERR_UNSUPPORTED, "the persistent fused step is for the GQA geometry");
    if (err && !al4(err)) return fail(VX_ERR_INVALID_ARG, "err must be 4-byte aligned");
    if (!std::isfinite(sm_scale)) return fail(VX_ERR_INVALID_ARG, "sm_scale must be finite");
    Plan p;
    VX_TRY(plan(geo, k, 0, &p));
    const WsLayout l = ws_layout(geo, table->max_pages, k, p);
    if (!ws || !al16(ws)) return fail(VX_ERR_WORKSPACE, "workspace is NULL or not 16-byte aligned");
    if (ws_bytes < l.total)
        return fail(VX_ERR_WORKSPACE, "workspace of %zu bytes < %zu needed", ws_bytes, l.total);
    float *scores = scores_out ? scores_out : reinterpret_cast<float *>(static_cast<char *>(ws) + l.scores);
    int32_t *sel = sel_out ? sel_out : reinterpret_cast<int32_t *>(static_cast<char *>(ws) + l.sel);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const FusedPlan f = fused_plan(geo, table->max_pages, k);
    if (!f.ok)
        return fail(VX_ERR_UNSUPPORTED, "the persistent fused step needs head_dim_qk == head_dim_v in {64, 128}, "
                                        "num_kv_heads <= 16, <= 16 query heads per KV head and batch <= %d",
                    vx::FUSED_MAX_B);
    {
        // one persistent launch: score -> exact top-k -> attention -> merge
        vx::FusedArgs a{};
        a.page_ptr = table->page_ptr;
        a.page_indices = table->page_indices;
        a.seq_lens = table->seq_lens;
        a.q = static_cast<const __nv_bfloat16 *>(q);
        a.centroids = static_cast<const __nv_bfloat16 *>(centroids);
        a.scores = scores;
        a.sel = sel;
        a.o_part = reinterpret_cast<float *>(static_cast<char *>(ws) + l.o_part);
        a.ml_part = reinterpret_cast<float *>(static_cast<char *>(ws) + l.ml_part);
        a.out = static_cast<__nv_bfloat16 *>(out);
        a.lse = lse;
        a.err = err;
        a.sync = reinterpret_cast<uint32_t *>(static_cast<char *>(ws) + l.sync);
        a.B = geo->batch;
        a.Hq = geo->num_q_heads;
        a.Hkv = geo->num_kv_heads;
        a.G = p.G;
        a.D = geo->head_dim_qk;
        a.P = geo->page_size;
        a.max_pages = table->max_pages;
        a.k = k;
        a.tiles_per_page = geo->page_size / vx::DEC_TILE;
        a.spages = f.spages;
        a.dtiles = f.dtiles;
        a.t_blocks = f.t_blocks;
        a.dlag = f.dlag;
        a.num_pool_pages = geo->num_pool_pages;
        const float scale = sm_scale > 0.f ? sm_scale : 1.0f / std::sqrt((float)geo->head_dim_qk);
        a.scale_log2 = scale * 1.4426950408889634f;
        const int64_t page_heads = geo->num_pool_pages * geo->num_kv_heads;
        CUtensorMap tmK, tmV;
        VX_TRY(make_cache_map(&tmK, k_cache, geo->head_dim_qk, geo->page_size, page_heads, vx::DEC_TILE));
        VX_TRY(make_cache_map(&tmV, v_cache, geo->head_dim_v, geo->page_size, page_heads, vx::DEC_TILE));
        cudaError_t e = vx::launch_fused(a, tmK, tmV, s);
        if (e != cudaSuccess) return cuda_fail(e, "fused step launch");
        return VX_OK;
    }
}

}  // extern "C"
