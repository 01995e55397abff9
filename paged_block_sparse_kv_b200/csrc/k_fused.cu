// k_fused.cu -- the whole GQA decode step (score -> exact top-k -> sparse attention -> merge)
// as one persistent kernel.
//
// Vortex paper note, section 系统设计 3: kernel fusion and workload planning; the indexer
// (section 系统设计 1: centroid scores, block top-k) and the sparse attention over the kept
// blocks run back to back every decode step.  Here they share one launch, so the stages of
// different requests overlap instead of waiting for whole-batch kernel boundaries.
//
// Work items (warp granularity):
//   S(b, j0, j1)  score pages [j0, j1) of request b for all KV heads (centroid rows by 1-D
//                 TMA bulk copies into a per-warp 4-stage ring, group-summed query in
//                 registers), then add j1 - j0 to scored[b];
//   T(b, h)       wait until scored[b] == n_b, radix-select row (b, h)'s k_eff largest
//                 scores on the warp (11/11/10-bit digits, ties to the lower page), write
//                 sel, then set row_ready;
//   D(b, h, i)    wait for row_ready, attend tiles [i*dtiles, (i+1)*dtiles) of the row's
//                 selected pages (TMA tensor loads into a per-warp 3-stage ring, mma.sync),
//                 write the partial (o, m, l); the row's last item to finish merges the
//                 row's partials (log-sum-exp rule) into out and lse.
// S and D items come from one ticket counter: round r holds the S items of request r and
// the D items of request r - dlag.  T items come, in row order, from a second counter: the
// warps of the first t_blocks blocks take them first, and a D item whose row nobody has
// taken yet takes T tickets itself instead of waiting.  So every wait ends: S never waits,
// T waits only on S, and D waits only on a T that a running warp holds.  All waits are
// bounded (%globaltimer); a timeout sets the error word and an abort flag that ends the
// other waits.  The last block to finish clears the sync words, so every launch finds them
// zero.
#include "vx_attend.cuh"

namespace vx {

namespace {

constexpr int F_SSTAGES = 4;               // score ring stages per warp
constexpr int F_DSTAGES = 3;               // attention ring stages per warp
constexpr int F_REGION = 24 * 1024;        // per-warp shared-memory region (rings / top-k keys)
constexpr int F_SMALL = 128;               // per-warp mbarriers and tile metadata
constexpr int F_BINS = 2048;               // top-k histogram bins (11-bit digits)
constexpr int F_KEYS = (F_REGION - F_BINS * 4) / 4;  // top-k keys kept in shared memory (4096)
constexpr unsigned SYNC_TICKET = 0, SYNC_DONE = 1, SYNC_ABORT = 2, SYNC_ROW = 3;

enum ItemType { ITEM_S = 0, ITEM_T = 1, ITEM_D = 2 };
struct Item {
    int type, b, h, i0, i1;  // S: pages [i0, i1); D: item index i0
};

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Lane 0 waits until *p >= target, for at most WAIT_LIMIT_NS, or until the abort flag is
// set.  A timeout sets the error word and the abort flag.  Returns whether *p reached target.
__device__ __noinline__ bool wait_at_least(const uint32_t *p, uint32_t target, uint32_t *abort_flag,
                                           int32_t *err) {
    if (ld_acquire(p) >= target) return true;
    const unsigned long long t0 = globaltimer();
    for (;;) {
        __nanosleep(200);
        if (ld_acquire(p) >= target) return true;
        if (ld_acquire(abort_flag)) return false;
        if (globaltimer() - t0 > WAIT_LIMIT_NS) {
            set_err(err, VX_DATA_TIMEOUT);
            atomicExch(abort_flag, 1u);
            return false;
        }
    }
}

// Warp-aggregated shared-memory histogram increment (bin < 0: nothing); every lane calls it.
__device__ __forceinline__ void hist_add(int *hist, int bin, int lane) {
    const unsigned peers = __match_any_sync(FULL, bin);
    if (bin >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
}

__device__ __forceinline__ uint32_t order_key_f(float s) {  // order-preserving, -0 ties +0
    uint32_t f = __float_as_uint(s);
    if (f == 0x80000000u) f = 0u;
    return (f & 0x80000000u) ? ~f : (f | 0x80000000u);
}

__device__ __forceinline__ void bulk_load_1d(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
                 : "memory");
}

// Block-wide exclusive prefix of value(i), i < n, into out[0..n] (out[n] = total); contiguous
// runs per thread.  Contains __syncthreads; every thread of the block calls it.
template <class F>
__device__ __forceinline__ void block_prefix(int n, F &&value, int32_t *out, int *tmp) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int per = (n + (int)blockDim.x - 1) / (int)blockDim.x;
    const int i0 = min(n, tid * per), i1 = min(n, i0 + per);
    int local = 0;
    for (int i = i0; i < i1; ++i) local += value(i);
    int x = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(FULL, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) tmp[warp] = x;
    __syncthreads();
    int before = 0, total = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) {
        if (w < warp) before += tmp[w];
        total += tmp[w];
    }
    int run = before + x - local;
    for (int i = i0; i < i1; ++i) {
        out[i] = run;
        run += value(i);
    }
    if (tid == 0) out[n] = total;
    __syncthreads();
}

}  // namespace

// dims per lane for scoring a head row of D dims (the row is split over D / DPL lanes)
template <int D>
struct FScoreSplit {
    static constexpr int DPL = D == 128 ? 64 : 32;
    static constexpr int S = D / DPL;
    static constexpr int NCH = DPL / 8;
};

template <int D, int NT>
__global__ void __launch_bounds__(FUSED_WARPS * 32, 1)
    k_fused(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV, const FusedArgs a) {
    using SP = FScoreSplit<D>;
    constexpr int DPL = SP::DPL, S = SP::S, NCH = SP::NCH;
    constexpr int KB = D / 64;                   // 64-column TMA boxes per attention tile
    constexpr int BOX_BYTES = DEC_TILE * 128;    // 16 rows x 128 bytes
    constexpr int TILE_BYTES = KB * BOX_BYTES;   // 16 x D bf16
    constexpr int STAGE_BYTES = 2 * TILE_BYTES;  // K tile + V tile
    constexpr int MT = D / 16;
    static_assert(F_DSTAGES * STAGE_BYTES <= F_REGION, "attention ring fits the warp region");

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;  // 128-byte swizzle wants 1 KB alignment
    uint8_t *basep = smem_raw + (base - raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g4 = lane >> 2, q4 = lane & 3;
    const uint32_t region = base + (uint32_t)warp * F_REGION;
    uint8_t *region_p = basep + (size_t)warp * F_REGION;
    uint8_t *small_p = basep + (size_t)FUSED_WARPS * F_REGION + (size_t)warp * F_SMALL;
    const uint32_t sbar = smem_u32(small_p);                 // F_SSTAGES mbarriers
    const uint32_t dbar = sbar + 8u * F_SSTAGES;             // F_DSTAGES mbarriers
    int32_t *dmeta = reinterpret_cast<int32_t *>(small_p + 8 * (F_SSTAGES + F_DSTAGES));  // valid tokens per stage
    int32_t *npg = reinterpret_cast<int32_t *>(basep + (size_t)FUSED_WARPS * (F_REGION + F_SMALL));
    int32_t *ditems = npg + a.B;        // attention items per row of request b
    int32_t *lens = ditems + a.B;       // [B] seq_lens
    int32_t *ppt = lens + a.B;          // [B] page_ptr
    int32_t *dpre = ppt + a.B;          // [B + 1] partial slots before request b
    int32_t *rpre = dpre + a.B + 1;     // [B + dlag + 1] tickets before round r
    __shared__ int scan_tmp[FUSED_WARPS];
    __shared__ int last_block;

    uint32_t *sync = a.sync;
    uint32_t *abort_flag = sync + SYNC_ABORT;
    uint32_t *scored = sync + FUSED_SYNC_HDR;                                  // [B]
    uint32_t *row_ready = scored + FUSED_MAX_B;                                // [B * Hkv]
    uint32_t *row_done = row_ready + (size_t)FUSED_MAX_B * FUSED_MAX_HKV;      // [B * Hkv]

    if (lane == 0) {
        for (int s = 0; s < F_SSTAGES + F_DSTAGES; ++s) mbar_init(sbar + 8u * s, 1);
        fence_mbar_init();
    }
    if (tid == 0) {
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    // ---- per-request tables (every block builds its own copy)
    for (int b = tid; b < a.B; b += blockDim.x) {
        const int32_t L = a.seq_lens[b];
        const int n = (L >= 1 && L <= a.max_pages * a.P) ? ceil_div(L, a.P) : 0;
        npg[b] = n;
        lens[b] = L;
        ppt[b] = a.page_ptr[b];
        ditems[b] = max(1, ceil_div(min(a.k, n) * a.tiles_per_page, a.dtiles));
    }
    __syncthreads();
    const int nrounds = a.B + a.dlag;
    block_prefix(nrounds, [&](int r) {
        int c = 0;
        if (r < a.B) c += ceil_div(npg[r], a.spages);
        if (r >= a.dlag && r - a.dlag < a.B) c += a.Hkv * ditems[r - a.dlag];
        return c;
    }, rpre, scan_tmp);
    block_prefix(a.B, [&](int b) { return a.Hkv * ditems[b]; }, dpre, scan_tmp);
    const uint32_t total = (uint32_t)rpre[nrounds];
    const uint32_t nrows = (uint32_t)(a.B * a.Hkv);

    // ticket -> work item (round r: S items of request r, then D items of request r - dlag)
    auto item_of = [&](uint32_t t) -> Item {
        int lo = 0, hi = nrounds - 1;  // last r with rpre[r] <= t
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if ((uint32_t)rpre[mid] <= t) lo = mid;
            else hi = mid - 1;
        }
        const int r = lo;
        int o = (int)(t - (uint32_t)rpre[r]);
        Item it{ITEM_D, 0, 0, 0, 0};
        if (r < a.B) {
            const int si = ceil_div(npg[r], a.spages);
            if (o < si) {
                it.type = ITEM_S;
                it.b = r;
                it.i0 = o * a.spages;
                it.i1 = min(npg[r], it.i0 + a.spages);
                return it;
            }
            o -= si;
        }
        const int b = r - a.dlag;
        it.b = b;
        it.h = o / ditems[b];
        it.i0 = o % ditems[b];
        return it;
    };

    uint32_t s_seq = 0, d_seq = 0;  // uses of the score / attention rings (stage = seq % stages)
    bool aborted = false;           // this warp's ring state is unusable: take no more items

    // ================================================================ S: score pages
    // lane = (page of the stage, KV head, segment of DPL dims); the query sum in registers
    const int lpp = a.Hkv * S;       // lanes per page (divides 32, checked on the host)
    const int pps = 32 / lpp;        // pages per stage
    const uint32_t row_bytes = (uint32_t)a.Hkv * D * 2u;
    const uint32_t sstage_bytes = (uint32_t)pps * row_bytes;
    const int my_page = lane / lpp, my_head = (lane / S) % a.Hkv, my_seg = lane % S;
    // chunk rotation, fixed by (head, segment) as in the standalone scorer: a page's sum
    // order does not depend on its slot in a stage
    const int rot_lane = (lane % lpp) % NCH;
    float qreg[NCH][8];
    auto load_query_sum = [&](int b) {
        // the group's heads summed in head order (fp32), chunk c of qreg holding chunk
        // (c + rot_lane) % NCH: the standalone scorer's sums, bit for bit
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
                v0[c] = __ldg(reinterpret_cast<const uint4 *>(qb + (size_t)g * D + ch * 8));
                v1[c] = g + 1 < a.G ? __ldg(reinterpret_cast<const uint4 *>(qb + (size_t)(g + 1) * D + ch * 8))
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

    auto do_score = [&](int b, int j0, int j1) {
        const int cnt = j1 - j0;  // <= 32
        const int32_t pp = ppt[b];
        int32_t id = -1;
        if (lane < cnt) {
            id = a.page_indices[pp + j0 + lane];
            if (id < 0 || id >= a.num_pool_pages) {
                set_err(a.err, VX_DATA_BAD_PAGE_ID);
                id = -1;
            }
        }
        const uint32_t valid = __ballot_sync(FULL, id >= 0);
        const int nst = ceil_div(cnt, pps);
        const uint32_t seq0 = s_seq;
        fence_proxy_async_smem();  // the region may hold generic writes of an earlier item
        auto issue = [&](int i) {
            const uint32_t seq = seq0 + (uint32_t)i;
            const int st = (int)(seq % F_SSTAGES);
            const uint32_t bar = sbar + 8u * st;
            const int p0 = i * pps, p1 = min(cnt, p0 + pps);
            const uint32_t smask = (p1 >= 32 ? 0xffffffffu : ((1u << p1) - 1u)) & ~((1u << p0) - 1u);
            const uint32_t take = valid & smask;
            if (lane == 0) mbar_arrive_expect_tx(bar, (uint32_t)__popc(take) * row_bytes);
            __syncwarp();
            if ((take >> lane) & 1u)
                bulk_load_1d(region + (uint32_t)st * sstage_bytes + (uint32_t)(lane - p0) * row_bytes,
                             a.centroids + (size_t)id * a.Hkv * D, row_bytes, bar);
            __syncwarp();
        };
        const int first = min(nst, F_SSTAGES);
        for (int i = 0; i < first; ++i) issue(i);
        s_seq = seq0 + (uint32_t)nst;
        load_query_sum(b);
        float *srow = a.scores + ((size_t)b * a.Hkv + my_head) * a.max_pages + j0;
        for (int i = 0; i < nst; ++i) {
            const uint32_t seq = seq0 + (uint32_t)i;
            const int st = (int)(seq % F_SSTAGES);
            if (!__all_sync(FULL, mbar_wait_bounded(sbar + 8u * st, (seq / F_SSTAGES) & 1u))) {
                if (lane == 0) {
                    set_err(a.err, VX_DATA_TIMEOUT);
                    atomicExch(abort_flag, 1u);
                }
                for (int r = i + 1; r < min(nst, i + F_SSTAGES); ++r) {
                    const uint32_t sq = seq0 + (uint32_t)r;
                    (void)mbar_wait_bounded(sbar + 8u * (sq % F_SSTAGES), (sq / F_SSTAGES) & 1u);
                }
                aborted = true;
                return;
            }
            const int page = i * pps + my_page;
            float dot = 0.f;
            if (page < cnt) {
                const uint32_t src = region + (uint32_t)st * sstage_bytes + (uint32_t)my_page * row_bytes +
                                     (uint32_t)(my_head * D + my_seg * DPL) * 2u;
                float acc4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < NCH; ++c) {
                    const int ch = (c + rot_lane) % NCH;  // rotated: distinct banks
                    uint4 v;
                    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                                 : "r"(src + (uint32_t)ch * 16u));
                    float f[8];
                    bf16x8_to_f32(v, f);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc4[e & 3] = fmaf(f[e], qreg[c][e], acc4[e & 3]);
                }
                dot = (acc4[0] + acc4[1]) + (acc4[2] + acc4[3]);
            }
#pragma unroll
            for (int off = 1; off < S; off <<= 1) dot += __shfl_xor_sync(FULL, dot, off);
            const int32_t pid = __shfl_sync(FULL, id, min(page, 31));
            if (my_seg == 0 && page < cnt) srow[page] = pid >= 0 ? dot : -INFINITY;
            __syncwarp();  // every lane is done with this stage before it is refilled
            if (i + F_SSTAGES < nst) issue(i + F_SSTAGES);
        }
        __syncwarp();
        if (lane == 0) {
            __threadfence();  // the scores above, before the count that publishes them
            atomicAdd(&scored[b], (uint32_t)cnt);
        }
    };
    // ================================================================ T: exact top-k of a row
    // Radix select on order-preserving keys (11/11/10-bit digits, MSB first) with the
    // histogram in the warp's shared region, early exit once the boundary bucket holds
    // exactly the slots left; the chosen pages leave in ascending page order, boundary ties
    // to the lower page.
    auto do_topk = [&](int b, int h) {
        const int row = b * a.Hkv + h;
        int32_t *out = a.sel + (size_t)row * a.k;
        const int n = npg[b];
        auto publish = [&]() {
            __syncwarp();
            if (lane == 0) {
                __threadfence();  // sel above, before the flag that publishes it
                atomicExch(&row_ready[row], 1u);
            }
        };
        if (n == 0) {  // bad length: empty selection
            for (int i = lane; i < a.k; i += 32) out[i] = -1;
            if (lane == 0 && h == 0) set_err(a.err, VX_DATA_BAD_SEQ_LEN);
            publish();
            return;
        }
        const int keff = min(a.k, n);
        if (keff == n) {  // every page is chosen
            for (int i = lane; i < a.k; i += 32) out[i] = i < n ? i : -1;
            publish();
            return;
        }
        bool ok = true;
        if (lane == 0) ok = wait_at_least(&scored[b], (uint32_t)n, abort_flag, a.err);
        ok = __shfl_sync(FULL, ok, 0);
        __syncwarp();
        if (!ok) {  // aborted: publish an empty selection
            for (int i = lane; i < a.k; i += 32) out[i] = -1;
            publish();
            return;
        }
        const float *rs = a.scores + (size_t)row * a.max_pages;
        int *hist = reinterpret_cast<int *>(region_p);
        uint32_t *keys = reinterpret_cast<uint32_t *>(region_p + F_BINS * 4);
        const bool in_smem = n <= F_KEYS;
        auto key_at = [&](int j) -> uint32_t { return in_smem ? keys[j] : order_key_f(__ldcg(rs + j)); };

        // first sweep: keys to shared memory and the top digit's histogram
        for (int i = lane; i < F_BINS; i += 32) hist[i] = 0;
        __syncwarp();
        for (int j0 = 0; j0 < n; j0 += 128) {
            float v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = j0 + u * 32 + lane;
                v[u] = j < n ? __ldcg(rs + j) : 0.f;
            }
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int j = j0 + u * 32 + lane;
                const uint32_t key = order_key_f(v[u]);
                if (j < n && in_smem) keys[j] = key;
                hist_add(hist, j < n ? (int)(key >> 21) : -1, lane);
            }
        }
        __syncwarp();
        uint32_t prefix = 0, mask = 0;
        int remaining = keff;
#pragma unroll 1
        for (int pass = 0; pass < 3; ++pass) {
            const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
            const int bins = pass == 2 ? 1024 : 2048;
            const uint32_t dmask = (uint32_t)bins - 1u;
            if (pass > 0) {
                for (int i = lane; i < bins; i += 32) hist[i] = 0;
                __syncwarp();
                for (int j0 = 0; j0 < n; j0 += 32) {
                    const int j = j0 + lane;
                    const uint32_t key = j < n ? key_at(j) : 0u;
                    hist_add(hist, (j < n && (key & mask) == prefix) ? (int)((key >> shift) & dmask) : -1, lane);
                }
                __syncwarp();
            }
            // the bin holding the remaining-th largest key, from the top: lane l owns bins
            // [(31 - l) * per, (32 - l) * per), so lane 0 holds the highest
            const int per = bins / 32;
            const int bin0 = (31 - lane) * per;
            int own = 0;
            for (int i = 0; i < per; ++i) own += hist[bin0 + i];
            int incl = own;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(FULL, incl, off);
                if (lane >= off) incl += y;
            }
            int above = incl - own;
            const bool mine = above < remaining && incl >= remaining;
            int digit = 0, above_d = 0, cnt = 0;
            if (mine) {
                for (int i = per - 1; i >= 0; --i) {
                    const int c = hist[bin0 + i];
                    if (above + c >= remaining) {
                        digit = bin0 + i;
                        above_d = above;
                        cnt = c;
                        break;
                    }
                    above += c;
                }
            }
            const int src = __ffs(__ballot_sync(FULL, mine)) - 1;
            digit = __shfl_sync(FULL, digit, src);
            above_d = __shfl_sync(FULL, above_d, src);
            cnt = __shfl_sync(FULL, cnt, src);
            remaining -= above_d;
            prefix |= static_cast<uint32_t>(digit) << shift;
            mask |= dmask << shift;
            __syncwarp();  // the histogram is read before the next pass clears it
            if (cnt == remaining) break;  // the whole boundary bucket is taken
        }
        // ordered compaction
        const unsigned lt = (1u << lane) - 1u;
        int pos = 0, eq_seen = 0;
        for (int j0 = 0; j0 < n; j0 += 32) {
            const int j = j0 + lane;
            const uint32_t mk = (j < n ? key_at(j) : 0u) & mask;
            const bool gt = j < n && mk > prefix;
            const bool eq = j < n && mk == prefix;
            const unsigned eqb = __ballot_sync(FULL, eq);
            const int rank = eq_seen + __popc(eqb & lt);
            eq_seen += __popc(eqb);
            const bool chosen = gt || (eq && rank < remaining);
            const unsigned cb = __ballot_sync(FULL, chosen);
            const int p = pos + __popc(cb & lt);
            if (chosen && p < a.k) out[p] = j;
            pos += __popc(cb);
        }
        for (int i = pos + lane; i < a.k; i += 32) out[i] = -1;
        publish();
    };
    // ================================================================ D: attend a span of a row
    auto do_attend = [&](int b, int h, int idx) {
        const int row = b * a.Hkv + h;
        const int n = npg[b];
        const int di = ditems[b];
        const int row_units = min(a.k, n) * a.tiles_per_page;
        const int u0 = idx * a.dtiles, u1 = min(row_units, u0 + a.dtiles);

        // wait for the row's selection; while nobody holds the row's top-k ticket yet, take
        // top-k tickets (in row order) and do them here, so the wait always ends
        bool ok = true;
        if (u0 < u1) {
            for (;;) {
                uint32_t ready = 0, tk = 0xffffffffu;
                if (lane == 0) {
                    ready = ld_acquire(&row_ready[row]);
                    if (!ready && ld_acquire(&sync[SYNC_ROW]) <= (uint32_t)row) tk = atomicAdd(&sync[SYNC_ROW], 1u);
                }
                ready = __shfl_sync(FULL, ready, 0);
                tk = __shfl_sync(FULL, tk, 0);
                if (ready) break;
                if (tk < nrows) {
                    do_topk((int)(tk / a.Hkv), (int)(tk % a.Hkv));
                    continue;
                }
                if (lane == 0) ok = wait_at_least(&row_ready[row], 1u, abort_flag, a.err);
                ok = __shfl_sync(FULL, ok, 0);
                break;
            }
            __syncwarp();
        }
        // the group's query heads as mma B fragments
        uint32_t qf[NT][MT][2];
        float acc[NT][MT][4];
        float m_run[NT][2], l_run[NT][2];
        {
            const __nv_bfloat16 *qb = a.q + ((size_t)b * a.Hq + (size_t)h * a.G) * D;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int head = nt * 8 + g4;
#pragma unroll
                for (int kk = 0; kk < MT; ++kk) {
                    if (head < a.G) {
                        const uint32_t *qp = reinterpret_cast<const uint32_t *>(qb + (size_t)head * D + kk * 16 + 2 * q4);
                        qf[nt][kk][0] = qp[0];
                        qf[nt][kk][1] = qp[4];  // +8 dims
                    } else {
                        qf[nt][kk][0] = 0u;
                        qf[nt][kk][1] = 0u;
                    }
                }
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[nt][mt][e] = 0.f;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    m_run[nt][i] = -INFINITY;
                    l_run[nt][i] = 0.f;
                }
            }
        }
        if (ok && u0 < u1) {
            fence_proxy_async_smem();  // the region may hold generic writes of an earlier item
            const int32_t L = lens[b];
            const int32_t pp = ppt[b];
            const int32_t *selr = a.sel + (size_t)row * a.k;
            // lane resolves unit u of the row: (TMA z, y, valid tokens) or invalid
            auto resolve = [&](int u, int32_t &z, int32_t &y, int32_t &nv) -> bool {
                if (u >= u1) return false;
                const int i = u / a.tiles_per_page, sub = u - i * a.tiles_per_page;
                const int32_t j = __ldcg(selr + i);
                if (j < 0) return false;
                if (j >= n) {
                    set_err(a.err, VX_DATA_BAD_SELECTION);
                    return false;
                }
                const int tok0 = j * a.P + sub * DEC_TILE;
                nv = min(DEC_TILE, L - tok0);
                if (nv <= 0) return false;
                const int32_t phys = a.page_indices[pp + j];
                if (phys < 0 || phys >= a.num_pool_pages) {
                    set_err(a.err, VX_DATA_BAD_PAGE_ID);
                    return false;
                }
                z = phys * a.Hkv + h;
                y = sub * DEC_TILE;
                return true;
            };
            int ub = u0;
            int32_t rz = 0, ry = 0, rnv = 0;
            bool rv = resolve(ub + lane, rz, ry, rnv);
            uint32_t pending = __ballot_sync(FULL, rv);
            uint32_t issued = 0, consumed = 0;
            for (;;) {
                while (issued - consumed < F_DSTAGES) {
                    if (pending == 0) {
                        ub += 32;
                        if (ub >= u1) break;
                        rv = resolve(ub + lane, rz, ry, rnv);
                        pending = __ballot_sync(FULL, rv);
                        continue;
                    }
                    const int src = __ffs(pending) - 1;
                    pending &= pending - 1;
                    const int32_t z = __shfl_sync(FULL, rz, src);
                    const int32_t y = __shfl_sync(FULL, ry, src);
                    const int32_t nv = __shfl_sync(FULL, rnv, src);
                    const uint32_t seq = d_seq + issued;
                    const int st = (int)(seq % F_DSTAGES);
                    if (lane == 0) {
                        dmeta[st] = nv;
                        const uint32_t bar = dbar + 8u * st;
                        const uint32_t sK = region + (uint32_t)st * STAGE_BYTES;
                        mbar_arrive_expect_tx(bar, STAGE_BYTES);
#pragma unroll
                        for (int kb = 0; kb < KB; ++kb) {
                            tma_load_3d(sK + kb * BOX_BYTES, &tmK, kb * 64, y, z, bar);
                            tma_load_3d(sK + TILE_BYTES + kb * BOX_BYTES, &tmV, kb * 64, y, z, bar);
                        }
                    }
                    __syncwarp();
                    ++issued;
                }
                if (consumed == issued) break;
                const uint32_t seq = d_seq + consumed;
                const int st = (int)(seq % F_DSTAGES);
                if (!__all_sync(FULL, mbar_wait_bounded(dbar + 8u * st, (seq / F_DSTAGES) & 1u))) {
                    if (lane == 0) {
                        set_err(a.err, VX_DATA_TIMEOUT);
                        atomicExch(abort_flag, 1u);
                    }
                    for (uint32_t r = consumed + 1; r < issued; ++r) {
                        const uint32_t sq = d_seq + r;
                        (void)mbar_wait_bounded(dbar + 8u * (sq % F_DSTAGES), (sq / F_DSTAGES) & 1u);
                    }
                    aborted = true;
                    consumed = issued;
                    break;
                }
                const int nvalid = dmeta[st];
                const uint32_t sK = region + (uint32_t)st * STAGE_BYTES;
                attend_tile<D, NT>(sK, sK + TILE_BYTES, nvalid, a.scale_log2, qf, acc, m_run, l_run, lane);
                __syncwarp();  // every lane is done with this stage before it is refilled
                ++consumed;
            }
            d_seq += issued;
        }
        // the row sum of each head over this warp's tokens
        float lt[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                float v = l_run[nt][i];
                v += __shfl_xor_sync(FULL, v, 4);
                v += __shfl_xor_sync(FULL, v, 8);
                v += __shfl_xor_sync(FULL, v, 16);
                lt[nt][i] = v;
            }
        const size_t head0 = (size_t)b * a.Hq + (size_t)h * a.G;  // first query head of the group
        if (di == 1) {  // the row in one item: final values directly
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int head = nt * 8 + 2 * q4 + (e & 1);
                        const int dim = mt * 16 + g4 + 8 * (e >> 1);
                        const float l = lt[nt][e & 1];
                        if (head < a.G) a.out[(head0 + head) * D + dim] = __float2bfloat16_rn(l > 0.f ? acc[nt][mt][e] / l : 0.f);
                    }
            if (a.lse && g4 == 0) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int i = 0; i < 2; ++i) {
                        const int head = nt * 8 + 2 * q4 + i;
                        if (head < a.G)
                            a.lse[head0 + head] =
                                lt[nt][i] > 0.f ? (m_run[nt][i] + log2f(lt[nt][i])) * 0.69314718055994531f : -INFINITY;
                    }
            }
            return;
        }
        // partial of this item at slot dpre[b] + h * di + idx
        const int64_t slot0 = (int64_t)dpre[b] + (int64_t)h * di;
        const int64_t slot = slot0 + idx;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int head = nt * 8 + 2 * q4 + (e & 1);
                    const int dim = mt * 16 + g4 + 8 * (e >> 1);
                    if (head < a.G) a.o_part[(slot * a.G + head) * D + dim] = acc[nt][mt][e];
                }
        if (g4 == 0) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int head = nt * 8 + 2 * q4 + i;
                    if (head < a.G) {
                        float *ml = a.ml_part + (slot * a.G + head) * 2;
                        ml[0] = m_run[nt][i];
                        ml[1] = lt[nt][i];
                    }
                }
        }
        __syncwarp();
        uint32_t before = 0;
        if (lane == 0) {
            __threadfence();  // the partial above, before the count that publishes it
            before = atomicAdd(&row_done[row], 1u);
            if (before == (uint32_t)di - 1) __threadfence();  // every other partial is visible
        }
        before = __shfl_sync(FULL, before, 0);
        __syncwarp();
        if (before != (uint32_t)di - 1) return;
        // ---- last item of the row: merge its di partials (log-sum-exp rule, partial order)
        float *wsm = reinterpret_cast<float *>(region_p);  // [di][G] weights, then lsum[G], M[G]
        float *lsum_s = wsm + di * a.G, *max_s = lsum_s + a.G;
        for (int g = 0; g < a.G; ++g) {
            float M = -INFINITY;
            for (int i = lane; i < di; i += 32) M = fmaxf(M, __ldcg(a.ml_part + ((slot0 + i) * a.G + g) * 2));
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, off));
            float ls = 0.f;
            for (int i = lane; i < di; i += 32) {
                const float *ml = a.ml_part + ((slot0 + i) * a.G + g) * 2;
                const float m = __ldcg(ml);
                const float w = (M == -INFINITY || m == -INFINITY) ? 0.f : exp2f(m - M);
                wsm[i * a.G + g] = w;
                if (w != 0.f) ls += w * __ldcg(ml + 1);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) ls += __shfl_xor_sync(FULL, ls, off);
            if (lane == 0) {
                lsum_s[g] = ls;
                max_s[g] = M;
            }
        }
        __syncwarp();
        constexpr int D4 = D / 4;
        for (int p = lane; p < a.G * D4; p += 32) {
            const int g = p / D4, d = (p - g * D4) * 4;
            float o[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
            for (int i = 0; i < di; ++i) {
                const float w = wsm[i * a.G + g];
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(a.o_part + ((slot0 + i) * a.G + g) * D + d));
                if (w != 0.f) {  // an empty partial holds no output values
                    o[0] += w * v.x;
                    o[1] += w * v.y;
                    o[2] += w * v.z;
                    o[3] += w * v.w;
                }
            }
            const float ls = lsum_s[g];
            const float inv = ls > 0.f ? 1.f / ls : 0.f;
            __nv_bfloat16 *dst = a.out + (head0 + g) * D + d;
            *reinterpret_cast<uint32_t *>(dst) = pack_bf16x2(o[0] * inv, o[1] * inv);
            *reinterpret_cast<uint32_t *>(dst + 2) = pack_bf16x2(o[2] * inv, o[3] * inv);
        }
        if (a.lse)
            for (int g = lane; g < a.G; g += 32)
                a.lse[head0 + g] = lsum_s[g] > 0.f ? (max_s[g] + log2f(lsum_s[g])) * 0.69314718055994531f : -INFINITY;
        __syncwarp();  // the weights are read before the region is reused
    };
    // ================================================================ the ticket loop
    // The next ticket is requested before the current item runs (its latency hides behind
    // the item).  Still deadlock-free: the smallest unfinished ticket is always being
    // processed (a prefetched ticket is larger than the one its warp works on), and its
    // dependencies are smaller tickets, all finished.
    if ((int)blockIdx.x < a.t_blocks) {  // top-k rows first, in request order
        for (;;) {
            uint32_t r = 0;
            if (lane == 0) r = atomicAdd(&sync[SYNC_ROW], 1u);
            r = __shfl_sync(FULL, r, 0);
            if (r >= nrows) break;
            do_topk((int)(r / a.Hkv), (int)(r % a.Hkv));
        }
    }
    uint32_t t = 0;
    if (lane == 0) t = atomicAdd(&sync[SYNC_TICKET], 1u);
    t = __shfl_sync(FULL, t, 0);
    while (t < total) {
        uint32_t next = 0;
        if (lane == 0) next = atomicAdd(&sync[SYNC_TICKET], 1u);
        const Item it = item_of(t);
        if (it.type == ITEM_S) do_score(it.b, it.i0, it.i1);
        else do_attend(it.b, it.h, it.i0);
        if (aborted) break;  // this warp's rings are unusable; waits on its items end by the abort flag
        t = __shfl_sync(FULL, next, 0);
    }

    // ---- the last block to finish clears the sync words for the next launch
    __syncthreads();
    if (tid == 0) {
        __threadfence();
        last_block = atomicAdd(&sync[SYNC_DONE], 1u) == gridDim.x - 1;
        if (last_block) __threadfence();
    }
    __syncthreads();
    if (last_block) {
        for (int i = tid; i < a.B; i += blockDim.x) scored[i] = 0u;
        for (int i = tid; i < a.B * a.Hkv; i += blockDim.x) {
            row_ready[i] = 0u;
            row_done[i] = 0u;
        }
        __syncthreads();
        if (tid == 0) {
            sync[SYNC_TICKET] = 0u;
            sync[SYNC_ABORT] = 0u;
            sync[SYNC_ROW] = 0u;
            sync[SYNC_DONE] = 0u;
        }
    }
}

size_t fused_smem_bytes(int32_t B) {
    if (B < 1 || B > FUSED_MAX_B) return 0;
    return 1024 + (size_t)FUSED_WARPS * (F_REGION + F_SMALL) + (size_t)(7 * B + 2) * sizeof(int32_t);  // dlag <= B
}

template <int D, int NT>
static cudaError_t launch_fused_dn(const FusedArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV,
                                   cudaStream_t s) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    const size_t smem = fused_smem_bytes(a.B);
    if (smem == 0) return cudaErrorInvalidValue;
    static std::atomic<unsigned long long> done;
    e = ensure_smem_limit(k_fused<D, NT>, (int)fused_smem_bytes(FUSED_MAX_B), done);
    if (e != cudaSuccess) return e;
    return launch_k(k_fused<D, NT>, dim3(sms), dim3(FUSED_WARPS * 32), smem, s, false, tmK, tmV, a);
}

cudaError_t launch_fused(const FusedArgs &a, const CUtensorMap &tmK, const CUtensorMap &tmV, cudaStream_t s) {
    const int nt = (a.G + 7) / 8;
    if (a.D == 128 && nt == 1) return launch_fused_dn<128, 1>(a, tmK, tmV, s);
    if (a.D == 128 && nt == 2) return launch_fused_dn<128, 2>(a, tmK, tmV, s);
    if (a.D == 64 && nt == 1) return launch_fused_dn<64, 1>(a, tmK, tmV, s);
    if (a.D == 64 && nt == 2) return launch_fused_dn<64, 2>(a, tmK, tmV, s);
    return cudaErrorInvalidValue;
}

}  // namespace vx
