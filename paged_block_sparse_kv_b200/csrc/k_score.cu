// k_score.cu -- indexer: group-summed query . page centroid for every page of a request.
//
// Vortex paper note, section 系统设计 1: blocks are scored by a matrix product of the
// current query with the cached centroids; the MLA experiment section scores on the
// 576-dim latent + rope key (rope-aware) and, as a variant, on the 512 latent dims.
//
// The contraction over the G query heads of a KV group is done first (fp32), so the
// kernel is a GEMV per (request, KV head) that must stream every page's centroid row
// (all KV heads contiguous, Hkv * Dqk bf16) exactly once at HBM speed.
//
// Work layout: a persistent grid of one block of SCORE_WARPS warps per SM; all pages of
// all requests form one flat list (each block derives the per-request page prefix from
// seq_lens), and every warp takes an equal contiguous range of it.
// Data path: each warp owns a ring of SCORE_STAGES stages in shared memory; a stage
// holds up to PPS consecutive pages of one request, each page row fetched by one 1-D TMA
// bulk copy (completion counted on the stage's mbarrier).
// Query: each block first sums the G query heads of every KV head (fp32, heads in order)
// for the first requests its page range touches (up to SCORE_QCAP, in shared memory, one
// load round for the whole block); a warp meeting another request sums it itself in the
// same order.
// Compute: lane l works on page l / (Hkv*S) of the stage, KV head (l / S) % Hkv and
// segment l % S of that head's row (DPL = D / S dims, kept as the summed query in
// registers), so a dot product is DPL FMAs plus a log2(S)-step shuffle; each lane walks
// its 16-byte chunks in an order rotated by its place in the page's lane group, which keeps
// the shared-memory reads free of bank conflicts when a group spans 8 or more lanes and
// fixes every page's sum order whatever stage slot it lands in.  Scores are collected in a per-warp [Hkv][32] buffer and
// written as coalesced 128-byte rows.
#include "vx_internal.h"

namespace vx {

constexpr int SCORE_STAGES = 4;        // stages in flight per warp
constexpr int SCORE_MAX_BATCH = 4096;  // requests whose prefix fits the block's shared memory
constexpr int SCORE_MAX_HKV = 16;
constexpr int SCORE_QCAP = 4;          // requests whose summed query a block keeps in shared memory

// dims per lane for a head dim (the head row is split over D / DPL lanes)
template <int D>
struct ScoreSplit {
    static constexpr int DPL = D == 576 ? 72 : (D == 128 ? 64 : 32);
    static constexpr int S = D / DPL;    // lanes per head row
    static constexpr int NCH = DPL / 8;  // 16-byte chunks per lane
};

struct ScoreMeta {
    int32_t b, j, n;  // request, first logical page, pages in the stage
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}

// Block-wide exclusive scan over SCORE_WARPS warps; `tmp` holds SCORE_WARPS ints.
__device__ __forceinline__ int score_block_scan(int v, int *tmp, int &total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(FULL, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) tmp[warp] = x;
    __syncthreads();
    int before = 0;
    total = 0;
#pragma unroll
    for (int w = 0; w < SCORE_WARPS; ++w) {
        const int t = tmp[w];
        if (w < warp) before += t;
        total += t;
    }
    __syncthreads();
    return before + x - v;
}

template <int D>
__global__ void __launch_bounds__(SCORE_WARPS * 32, 1) k_score_pages(ScoreArgs a) {
    // q and the centroids may come from the previous kernel on the stream, and so may the
    // table and lengths unless the call rules that out (table_ready: they are read first)
    if (!a.table_ready) pdl_wait();
    using SP = ScoreSplit<D>;
    constexpr int DPL = SP::DPL, S = SP::S, NCH = SP::NCH;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int lanes_per_page = a.Hkv * S;        // divides 32 (checked on the host)
    const int pps = 32 / lanes_per_page;         // pages per stage
    const uint32_t row_bytes = (uint32_t)a.Hkv * D * 2u;
    const uint32_t stage_bytes = ((uint32_t)pps * row_bytes + 127u) & ~127u;
    const int my_page = lane / lanes_per_page;
    const int my_head = (lane / S) % a.Hkv;
    const int my_seg = lane % S;
    // chunk rotation of the dot products: fixed by (head, segment), not by the page's slot in
    // a stage, so a page's sum order never depends on how stages were cut (16-byte reads of
    // the lanes of one page group hit distinct banks once the group spans 8 lanes)
    const int rot_lane = (lane % lanes_per_page) % NCH;

    extern __shared__ __align__(128) uint8_t smem[];
    int *prefix = reinterpret_cast<int *>(smem);  // B + 1: pages of request b = [prefix[b], prefix[b+1])
    int *pptr = prefix + a.B + 1;                 // B: page_ptr
    const uint32_t head_bytes = ((uint32_t)(2 * a.B + 1) * 4u + 127u) & ~127u;
    // each warp's area starts on a 128-byte boundary: its ring takes bulk copies (16-byte
    // aligned destinations) and 16-byte shared loads, whatever the stage count
    const size_t per_warp_bytes =
        (SCORE_STAGES * stage_bytes + SCORE_MAX_HKV * 32 * 4 + SCORE_STAGES * (8 + sizeof(ScoreMeta)) + 127) &
        ~size_t(127);
    uint8_t *per_warp = smem + head_bytes + (size_t)warp * per_warp_bytes;
    const uint32_t ring0 = smem_u32(per_warp);
    float *tbuf = reinterpret_cast<float *>(per_warp + SCORE_STAGES * stage_bytes);  // [Hkv][32]
    const uint32_t bar0 = smem_u32(per_warp + SCORE_STAGES * stage_bytes + SCORE_MAX_HKV * 32 * 4);
    ScoreMeta *meta = reinterpret_cast<ScoreMeta *>(per_warp + SCORE_STAGES * stage_bytes + SCORE_MAX_HKV * 32 * 4 +
                                                    SCORE_STAGES * 8);
    __shared__ int scan_tmp[SCORE_WARPS];

    if (lane == 0) {
        for (int s = 0; s < SCORE_STAGES; ++s) mbar_init(bar0 + 8u * s, 1);
        fence_mbar_init();
    }
    bool bad_len = false;  // reported after the dependency wait (err may be the previous kernel's output)
    {   // per-request page prefix and row starts
        const int per = ceil_div(a.B, blockDim.x);
        const int b0 = min(a.B, (int)threadIdx.x * per), b1 = min(a.B, b0 + per);
        int local = 0;
        for (int b = b0; b < b1; ++b) {
            const int32_t L = a.seq_lens[b];
            const bool ok = L >= 1 && L <= a.max_pages * a.P;
            bad_len |= !ok;
            local += ok ? ceil_div(L, a.P) : 0;
            pptr[b] = a.page_ptr[b];
        }
        int total;
        int run = score_block_scan(local, scan_tmp, total);
        for (int b = b0; b < b1; ++b) {
            prefix[b] = run;
            const int32_t L = a.seq_lens[b];
            run += (L >= 1 && L <= a.max_pages * a.P) ? ceil_div(L, a.P) : 0;
        }
        if (threadIdx.x == 0) prefix[a.B] = total;
        __syncthreads();
    }
    const int64_t T = prefix[a.B];
    const int64_t W = (int64_t)gridDim.x * SCORE_WARPS;
    const int64_t wid = (int64_t)blockIdx.x * SCORE_WARPS + warp;
    auto request_of = [&](int64_t p) -> int {  // last b with prefix[b] <= p
        int lo = 0, hi = a.B - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (prefix[mid] <= p) lo = mid;
            else hi = mid - 1;
        }
        return lo;
    };

    const int64_t p_begin = wid * T / W, p_end = (wid + 1) * T / W;
    // the first batch's page-table reads go out before the block sums the queries, so the
    // two round trips overlap
    int32_t pre_raw = -1, pre_b = -1, pre_j = 0;
    if (p_begin + lane < p_end) {
        pre_b = request_of(p_begin + lane);
        pre_j = static_cast<int32_t>(p_begin + lane - prefix[pre_b]);
        pre_raw = a.page_indices[pptr[pre_b] + pre_j];
    }
    // the block's first requests, whose group-summed queries it keeps in shared memory
    int qb0 = 0, qn = 0;
    {
        const int64_t bp0 = (int64_t)blockIdx.x * SCORE_WARPS * T / W;
        const int64_t bp1 = ((int64_t)blockIdx.x + 1) * SCORE_WARPS * T / W;
        if (bp0 < bp1 && a.qcap > 0) {
            qb0 = request_of(bp0);
            qn = min(a.qcap, request_of(bp1 - 1) - qb0 + 1);
        }
    }
    if (a.table_ready) {
        // their query rows go to L2 while the previous kernel finishes (q itself is read only
        // after the wait)
        const char *q0 = reinterpret_cast<const char *>(a.q + (size_t)qb0 * a.Hq * D);
        const int lines = static_cast<int>(((size_t)qn * a.Hq * D * 2 + 127) / 128);
        for (int i = threadIdx.x; i < lines; i += blockDim.x) prefetch_l2(q0 + (size_t)i * 128);
        pdl_wait();
    }
    if (bad_len && blockIdx.x == 0) set_err(a.err, VX_DATA_BAD_SEQ_LEN);
    // the decode kernel later in the same step counts its late pieces from this word
    if (a.zero_word && blockIdx.x == 0 && threadIdx.x == 0) *a.zero_word = 0u;

    // ---- group-summed queries of the block's first requests, computed once per block: each
    // thread sums one (request, KV head, 8-dim chunk) over the group's heads in head order
    float *qs = reinterpret_cast<float *>(smem + head_bytes + (size_t)SCORE_WARPS * per_warp_bytes);  // [qcap][Hkv][D]
    {
        constexpr int CPR = D / 8;  // 8-dim chunks per head row
        for (int idx = threadIdx.x; idx < qn * a.Hkv * CPR; idx += blockDim.x) {
            const int ch = idx % CPR, bh = idx / CPR;
            const int h = bh % a.Hkv, bq = bh / a.Hkv;
            float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (ch * 8 < a.score_dims) {
                const __nv_bfloat16 *src = a.q + ((size_t)(qb0 + bq) * a.Hq + (size_t)h * a.G) * D + ch * 8;
                for (int g0 = 0; g0 < a.G; g0 += 16) {  // 16 heads' loads in flight, added in head order
                    uint4 v[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        v[i] = g0 + i < a.G ? __ldg(reinterpret_cast<const uint4 *>(src + (size_t)(g0 + i) * D))
                                            : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        if (g0 + i >= a.G) break;
                        float f[8];
                        bf16x8_to_f32(v[i], f);
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[e] += f[e];
                    }
                }
            }
            float4 *dst = reinterpret_cast<float4 *>(qs + ((size_t)bq * a.Hkv + h) * D + ch * 8);
            dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
        __syncthreads();
    }
    if (p_begin >= p_end) return;

    // lane resolves flat page p: request, logical page, physical page (-1: skip)
    auto resolve = [&](int64_t p, int32_t &rb, int32_t &rj) -> int32_t {
        rb = -1;
        rj = 0;
        if (p >= p_end) return -1;
        const int lo = request_of(p);
        rb = lo;
        rj = static_cast<int32_t>(p - prefix[lo]);
        const int32_t id = a.page_indices[pptr[lo] + rj];
        if (id < 0 || id >= a.num_pool_pages) {
            set_err(a.err, VX_DATA_BAD_PAGE_ID);
            return -1;
        }
        return id;
    };

    // summed query of request b for this lane's head and segment, chunk c of qreg holding
    // chunk (c + rot_lane) % NCH: from the block's shared copy when the block summed it, else
    // the same sums (heads in order, fp32) from global memory
    float qreg[NCH][8];
    auto load_query = [&](int b) {
        if (b >= qb0 && b < qb0 + qn) {
            const float *src = qs + ((size_t)(b - qb0) * a.Hkv + my_head) * D + my_seg * DPL;
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                const float4 *p = reinterpret_cast<const float4 *>(src + ((c + rot_lane) % NCH) * 8);
                const float4 x = p[0], y = p[1];
                qreg[c][0] = x.x;
                qreg[c][1] = x.y;
                qreg[c][2] = x.z;
                qreg[c][3] = x.w;
                qreg[c][4] = y.x;
                qreg[c][5] = y.y;
                qreg[c][6] = y.z;
                qreg[c][7] = y.w;
            }
            return;
        }
        const __nv_bfloat16 *qb = a.q + ((size_t)b * a.Hq + (size_t)my_head * a.G) * D + my_seg * DPL;
#pragma unroll
        for (int c = 0; c < NCH; ++c)
#pragma unroll
            for (int i = 0; i < 8; ++i) qreg[c][i] = 0.f;
        for (int g = 0; g < a.G; g += 2) {  // two heads' loads in flight, added in head order
            uint4 v0[NCH], v1[NCH];
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                const int ch = (c + rot_lane) % NCH;
                const bool live = my_seg * DPL + ch * 8 < a.score_dims;
                v0[c] = live ? __ldg(reinterpret_cast<const uint4 *>(qb + (size_t)g * D + ch * 8))
                             : make_uint4(0u, 0u, 0u, 0u);
                v1[c] = (live && g + 1 < a.G)
                            ? __ldg(reinterpret_cast<const uint4 *>(qb + (size_t)(g + 1) * D + ch * 8))
                            : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                float f[8];
                bf16x8_to_f32(v0[c], f);
#pragma unroll
                for (int i = 0; i < 8; ++i) qreg[c][i] += f[i];
                if (g + 1 < a.G) {
                    bf16x8_to_f32(v1[c], f);
#pragma unroll
                    for (int i = 0; i < 8; ++i) qreg[c][i] += f[i];
                }
            }
        }
    };

    // score transpose buffer: window of 32 logical pages [wj, wj + 32) of request wb
    int wb = -1, wj = 0;
    uint32_t wmask = 0;
    auto flush_window = [&]() {
        __syncwarp();
        if (wmask) {
            float *dst = a.scores + (size_t)wb * a.Hkv * a.max_pages + wj + lane;
            const bool mine = (wmask >> lane) & 1u;
            for (int h = 0; h < a.Hkv; ++h)
                if (mine) dst[(size_t)h * a.max_pages] = tbuf[h * 32 + lane];
        }
        __syncwarp();
        wmask = 0;
    };

    int64_t batch = p_begin;
    int32_t my_b = pre_b, my_j = pre_j;
    int32_t my_id = pre_raw;
    if (my_b >= 0 && (my_id < 0 || my_id >= a.num_pool_pages)) {
        set_err(a.err, VX_DATA_BAD_PAGE_ID);
        my_id = -1;
    }
    uint32_t pending = __ballot_sync(FULL, my_id >= 0);
    uint32_t issued = 0, consumed = 0;
    bool failed = false;
    int cur_b = -1;
    for (;;) {
        // fill stages: up to pps consecutive pending pages of one request each
        while (issued - consumed < SCORE_STAGES) {
            if (pending == 0) {
                batch += 32;
                if (batch >= p_end) break;
                my_id = resolve(batch + lane, my_b, my_j);
                pending = __ballot_sync(FULL, my_id >= 0);
                continue;
            }
            const int st = static_cast<int>(issued % SCORE_STAGES);
            const uint32_t bar = bar0 + 8u * st;
            const uint32_t dst = ring0 + (uint32_t)st * stage_bytes;
            // choose the stage's pages (warp-uniform): lanes of `pending`, in order
            uint32_t take = 0;
            int n = 0, sb = -1, sj = 0;
            while (n < pps && pending) {
                const int src = __ffs(pending) - 1;
                const int32_t rb = __shfl_sync(FULL, my_b, src);
                const int32_t rj = __shfl_sync(FULL, my_j, src);
                if (n > 0 && (rb != sb || rj != sj + n)) break;  // one request, consecutive pages
                if (n == 0) {
                    sb = rb;
                    sj = rj;
                }
                take |= 1u << src;
                pending &= pending - 1;
                ++n;
            }
            if (lane == 0) {
                meta[st].b = sb;
                meta[st].j = sj;
                meta[st].n = n;
                mbar_arrive_expect_tx(bar, (uint32_t)n * row_bytes);  // all bytes announced first
            }
            __syncwarp();
            // no proxy fence: this stage's earlier shared-memory reads have completed, their
            // values were consumed before the __syncwarp that released the stage
            if ((take >> lane) & 1u) {
                const uint32_t slot = __popc(take & ((1u << lane) - 1u));
                bulk_load(dst + slot * row_bytes, a.centroids + (size_t)my_id * a.Hkv * D, row_bytes, bar);
            }
            __syncwarp();
            ++issued;
        }
        if (consumed == issued) break;
        const int st = static_cast<int>(consumed % SCORE_STAGES);
        if (cur_b < 0) {  // first stage: fetch its request's query while the rows are in flight
            cur_b = meta[st].b;
            load_query(cur_b);
        }
        const bool ok = __all_sync(FULL, mbar_wait_bounded(bar0 + 8u * st, (consumed / SCORE_STAGES) & 1u));
        if (!ok) {
            failed = true;
            break;
        }
        const ScoreMeta m = meta[st];
        if (m.b != cur_b) {
            load_query(m.b);
            cur_b = m.b;
        }
        // dot products: this lane's (page, head, segment)
        float dot = 0.f;
        if (my_page < m.n) {
            const uint32_t src = ring0 + (uint32_t)st * stage_bytes + (uint32_t)my_page * row_bytes +
                                 (uint32_t)(my_head * D + my_seg * DPL) * 2u;
            float acc4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int c = 0; c < NCH; ++c) {
                const int ch = (c + rot_lane) % NCH;
                uint4 v;
                asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                             : "r"(src + (uint32_t)ch * 16u));
                float f[8];
                bf16x8_to_f32(v, f);
#pragma unroll
                for (int i = 0; i < 8; ++i) acc4[i & 3] = fmaf(f[i], qreg[c][i], acc4[i & 3]);
            }
            dot = (acc4[0] + acc4[1]) + (acc4[2] + acc4[3]);
        }
#pragma unroll
        for (int off = 1; off < S; off <<= 1) dot += __shfl_xor_sync(FULL, dot, off);
        __syncwarp();  // every lane is done with this stage before it is refilled
        ++consumed;
        // record the stage's scores in the transpose window (a stage spans at most two
        // 32-page windows since pps <= 16)
        const int jpage = m.j + my_page;
        for (int part = 0; part < 2; ++part) {
            const int lo = part == 0 ? m.j : ((m.j & ~31) + 32);
            const int hi = min(m.j + m.n, (lo & ~31) + 32);
            if (lo >= hi) break;
            if (m.b != wb || (lo & ~31) != wj) {
                flush_window();
                wb = m.b;
                wj = lo & ~31;
            }
            if (my_seg == 0 && my_page < m.n && jpage >= lo && jpage < hi) tbuf[my_head * 32 + (jpage - wj)] = dot;
            const int cnt = hi - lo;
            wmask |= (cnt >= 32 ? 0xffffffffu : ((1u << cnt) - 1u)) << (lo - wj);
        }
    }
    if (failed) {
        if (lane == 0) set_err(a.err, VX_DATA_TIMEOUT);
        for (uint32_t i = consumed; i < issued; ++i)
            (void)mbar_wait_bounded(bar0 + 8u * (i % SCORE_STAGES), (i / SCORE_STAGES) & 1u);
        return;
    }
    flush_window();
}

template <int D>
static cudaError_t launch_score_d(const ScoreArgs &a, cudaStream_t s, bool pdl) {
    using SP = ScoreSplit<D>;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const int lpp = a.Hkv * SP::S;
    if (a.B > SCORE_MAX_BATCH || a.Hkv > SCORE_MAX_HKV || lpp > 32 || 32 % lpp) return cudaErrorInvalidValue;
    const size_t row_bytes = (size_t)a.Hkv * D * 2;
    const size_t stage_bytes = ((32 / lpp) * row_bytes + 127) & ~size_t(127);
    const size_t head = ((size_t)(2 * a.B + 1) * 4 + 127) & ~size_t(127);
    const size_t per_warp =
        (SCORE_STAGES * stage_bytes + SCORE_MAX_HKV * 32 * 4 + SCORE_STAGES * (8 + sizeof(ScoreMeta)) + 127) &
        ~size_t(127);
    size_t smem = head + (size_t)SCORE_WARPS * per_warp;
    // largest need: 4096 requests' prefix (32.9 KB) + 8 warps x 20.6 KB (MLA stages) < 200 KB
    constexpr int SCORE_SMEM_LIMIT = 200 * 1024;
    if (smem > (size_t)SCORE_SMEM_LIMIT) return cudaErrorInvalidValue;
    // what is left holds the summed queries of up to SCORE_QCAP requests per block
    ScoreArgs b = a;
    const size_t q_row = (size_t)a.Hkv * D * sizeof(float);
    b.qcap = (int32_t)std::min<size_t>(SCORE_QCAP, (SCORE_SMEM_LIMIT - smem) / q_row);
    smem += (size_t)b.qcap * q_row;
    static std::atomic<unsigned long long> done;
    e = ensure_smem_limit(k_score_pages<D>, SCORE_SMEM_LIMIT, done);
    if (e != cudaSuccess) return e;
    return launch_k(k_score_pages<D>, dim3(sms), dim3(SCORE_WARPS * 32), smem, s, pdl, b);
}

cudaError_t launch_score(const ScoreArgs &a, cudaStream_t s, bool pdl) {
    switch (a.Dqk) {
        case 64: return launch_score_d<64>(a, s, pdl);
        case 128: return launch_score_d<128>(a, s, pdl);
        case 576: return launch_score_d<576>(a, s, pdl);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace vx
