// vx_topk.cuh -- top-k pages of one (request, KV head) row of scores, by one thread block.
//
// Vortex paper note, section 系统设计 3: radix top-k, the bottleneck of the indexer
// stage, with stochastic early termination and remapping as the faster approximate
// form (its kernel-ablation section reports recall@k > 0.97 for that form).
//
// Scores become order-preserving uint32 keys (-0.0 folded onto +0.0), kept in shared
// memory when the row fits.
//   exact:  MSB-first radix select with 11/11/10-bit digits: a shared histogram per
//           digit, the digit holding the k-th largest key found by a block suffix scan,
//           early exit once the boundary bucket holds exactly the slots left.
//   approx: fp32 remap of each score to a 12-bit (mode 1), 10-bit (mode 2) or 8-bit (mode 3) code between
//           the row's min and max, one histogram of the codes, the boundary code b* from a
//           block suffix scan, no refinement: the slots left are filled from code b* in
//           cyclic page order from a SplitMix64-drawn offset.
// Both finish with an ordered compaction over contiguous per-thread runs (one block-wide
// exclusive scan of packed counts), so the chosen pages come out in ascending page order
// and boundary ties go to the lower page index (exact) or to the first pages after the
// drawn offset (approx).  Exact rows of at most TOPK_WARP_MAX pages can be done by one
// warp (warp_topk_small).  Used by the top-k kernel (one block per row); kept in a header so
// that another kernel can select rows it has just scored.
#pragma once

#include "vx_internal.h"

namespace vx {

constexpr int TOPK_SMALL_MAX = 6144;  // rows up to this many pages use 256-thread blocks
constexpr int TOPK_HIST = 1 << APPROX_BITS;

__device__ __forceinline__ uint32_t order_key(float s) {
    uint32_t f = __float_as_uint(s);
    if (f == 0x80000000u) f = 0u;  // -0.0 ties with +0.0
    return (f & 0x80000000u) ? ~f : (f | 0x80000000u);
}

// SplitMix64 (Steele, Lea and Flood 2014): draw number i of the generator seeded with seed.
__device__ __forceinline__ uint64_t splitmix64(uint64_t seed, uint64_t i) {
    uint64_t z = seed + (i + 1ull) * 0x9e3779b97f4a7c15ull;
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ull;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebull;
    return z ^ (z >> 31);
}

// Block-wide exclusive scan of one int per thread; also returns the total.  `tmp` holds
// 32 ints of shared memory.  Contains __syncthreads.
template <int THREADS, typename V = int>
__device__ __forceinline__ V block_exclusive_scan(V v, V *tmp, V &total) {
    constexpr int NW = THREADS / 32;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    V x = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const V y = __shfl_up_sync(FULL, x, off);
        if (lane >= off) x += y;
    }
    if (lane == 31) tmp[warp] = x;
    __syncthreads();
    if (warp == 0) {
        V w = lane < NW ? tmp[lane] : V(0);
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const V y = __shfl_up_sync(FULL, w, off);
            if (lane >= off) w += y;
        }
        if (lane < NW) tmp[lane] = w;  // inclusive over warps
    }
    __syncthreads();
    total = tmp[NW - 1];
    const V before = (warp > 0 ? tmp[warp - 1] : V(0)) + x - v;
    __syncthreads();  // tmp may be reused right after
    return before;
}

struct TopkShared {
    int hist[TOPK_HIST];
    int scan_tmp[32];
    unsigned long long scan_tmp64[32];
    int bcast[4];
    float fmin[32], fmax[32];
};

// The bin holding the `need`-th largest element of the first `bins` histogram entries,
// searching from the top: writes (bin, count above it, its count) to sh.bcast.
template <int THREADS>
__device__ __forceinline__ void block_find_bin(TopkShared &sh, int bins, int need) {
    // bins per thread: bins / THREADS when bins is a multiple of THREADS, else one for the
    // first `bins` threads (fewer bins than threads); thread 0 owns the top bins
    const int tid = static_cast<int>(threadIdx.x);
    const int per = bins >= THREADS ? bins / THREADS : (tid < bins ? 1 : 0);
    const int base = bins >= THREADS ? (THREADS - 1 - tid) * per : bins - 1 - tid;
    int own = 0;
    for (int i = 0; i < per; ++i) own += sh.hist[base + i];
    int total;
    int above = block_exclusive_scan<THREADS>(own, sh.scan_tmp, total);
    for (int i = per - 1; i >= 0; --i) {
        const int c = sh.hist[base + i];
        if (above < need && above + c >= need) {
            sh.bcast[0] = base + i;
            sh.bcast[1] = above;
            sh.bcast[2] = c;
        }
        above += c;
    }
    __syncthreads();
}

// One sweep over a row of n scores: every thread issues TOPK_SWEEP_UNROLL loads before it
// uses any of them, then calls f(j, score) for each.
constexpr int TOPK_SWEEP_UNROLL = 8;
template <int THREADS, class F>
__device__ __forceinline__ void sweep_row(const float *row, int n, F &&f) {
    for (int j0 = 0; j0 < n; j0 += THREADS * TOPK_SWEEP_UNROLL) {
        float v[TOPK_SWEEP_UNROLL];
#pragma unroll
        for (int i = 0; i < TOPK_SWEEP_UNROLL; ++i) {
            const int j = j0 + i * THREADS + (int)threadIdx.x;
            v[i] = j < n ? row[j] : 0.f;
        }
#pragma unroll
        for (int i = 0; i < TOPK_SWEEP_UNROLL; ++i) {
            const int j = j0 + i * THREADS + (int)threadIdx.x;
            if (j < n) f(j, v[i]);
        }
    }
}

static_assert(TOPK_SMEM_KEYS % 4 == 0, "the key buffer is read in 16-byte vectors");

// exact rows up to this many pages are selected by one warp when the launch has many rows:
// a row is then slower than with the whole block, but the block's other warps leave and more
// rows share an SM (measured: 1.16x faster over 2048 rows of 64-4103 pages, slower over 16 or
// 256 rows, where each row's latency sets the kernel time)
constexpr int TOPK_WARP_MAX = 512;

// Exact top-k of a short row (k_eff < n <= TOPK_WARP_MAX) by one warp, with no block barrier:
// the same radix select on order-preserving keys, in four 8-bit digits (a 256-bin histogram
// private to the warp), then the ordered compaction over contiguous per-lane runs with warp
// scans.  The chosen set is unique, so the result equals the block path's.
static __device__ __noinline__ void warp_topk_small(const float *__restrict__ row, int n, int keff, int32_t *out, int k,
                                             uint32_t *skeys, int *hist) {
    const int lane = threadIdx.x & 31;
    {   // keys of the row (up to 16 loads per lane in flight)
        float v[TOPK_WARP_MAX / 32];
#pragma unroll
        for (int i = 0; i < TOPK_WARP_MAX / 32; ++i) {
            const int j = lane + 32 * i;
            v[i] = j < n ? row[j] : 0.f;
        }
#pragma unroll
        for (int i = 0; i < TOPK_WARP_MAX / 32; ++i) {
            const int j = lane + 32 * i;
            if (j < n) skeys[j] = order_key(v[i]);
        }
    }
    __syncwarp();
    uint32_t prefix = 0, mask = 0;
    int remaining = keff;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        for (int i = lane; i < 256; i += 32) hist[i] = 0;
        __syncwarp();
        for (int j = lane; j < n; j += 32) {
            const uint32_t key = skeys[j];
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
        }
        __syncwarp();
        // lane l owns bins 255 - 8l down to 248 - 8l, so lane order is bin order from the top
        int c[8], own = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            c[i] = hist[255 - 8 * lane - i];
            own += c[i];
        }
        int incl = own;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(FULL, incl, off);
            if (lane >= off) incl += y;
        }
        int acc = incl - own, found = -1, f_above = 0, f_cnt = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (acc < remaining && acc + c[i] >= remaining) {
                found = 255 - 8 * lane - i;
                f_above = acc;
                f_cnt = c[i];
            }
            acc += c[i];
        }
        const int src = __ffs(__ballot_sync(FULL, found >= 0)) - 1;
        const int digit = __shfl_sync(FULL, found, src);
        const int above = __shfl_sync(FULL, f_above, src);
        const int cnt = __shfl_sync(FULL, f_cnt, src);
        remaining -= above;
        prefix |= static_cast<uint32_t>(digit) << shift;
        mask |= 0xffu << shift;
        __syncwarp();  // the histogram is cleared again by the next pass
        if (cnt == remaining) break;  // the whole boundary bucket is taken
    }
    // ordered compaction: lane l owns the run [l*R, l*R + R), R a multiple of 4 (16-byte reads)
    const int R = (((n + 31) / 32) + 3) & ~3;
    const int r0 = min(n, lane * R), r1 = min(n, r0 + R);
    int gt = 0, eq = 0;
    for (int j4 = r0; j4 < r1; j4 += 4) {
        const uint4 k4 = *reinterpret_cast<const uint4 *>(skeys + j4);
        const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            if (j4 + e < r1) {
                const uint32_t mk = kk[e] & mask;
                gt += mk > prefix;
                eq += mk == prefix;
            }
        }
    }
    int gt_incl = gt, eq_incl = eq;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y1 = __shfl_up_sync(FULL, gt_incl, off), y2 = __shfl_up_sync(FULL, eq_incl, off);
        if (lane >= off) {
            gt_incl += y1;
            eq_incl += y2;
        }
    }
    const int gt_total = __shfl_sync(FULL, gt_incl, 31), eq_total = __shfl_sync(FULL, eq_incl, 31);
    int eq_rank = eq_incl - eq;
    int pos = (gt_incl - gt) + min(eq_rank, remaining);
    for (int j4 = r0; j4 < r1; j4 += 4) {
        const uint4 k4 = *reinterpret_cast<const uint4 *>(skeys + j4);
        const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int j = j4 + e;
            if (j < r1) {
                const uint32_t mk = kk[e] & mask;
                bool take = mk > prefix;
                if (mk == prefix) take = eq_rank++ < remaining;
                if (take) {
                    if (pos < k) out[pos] = j;
                    ++pos;
                }
            }
        }
    }
    const int sel_total = gt_total + min(eq_total, remaining);
    for (int i = sel_total + lane; i < k; i += 32) out[i] = -1;
}

// Top-k of row (b, h) by the whole block (THREADS threads), written to a.sel.
// ABITS = 0: exact radix select; otherwise the approximate mode with 2^ABITS remap codes.
// `sh` and `skeys` (a.smem_keys entries, rounded up to 4, 16-byte aligned) are shared memory.
// dependent: the scores come from the previous kernel on the stream (wait for it before the
// first score is read, and let the next kernel launch once the radix passes are done);
// otherwise the caller has made them visible already.
template <int ABITS, int THREADS>
__device__ __forceinline__ void topk_row(const TopkArgs &a, int b, int h, TopkShared &sh, uint32_t *skeys,
                                         bool dependent) {
    constexpr bool APPROX = ABITS > 0;
    constexpr int NCODES = APPROX ? (1 << ABITS) : 2;  // remap codes of the approximate mode
    static_assert(NCODES <= TOPK_HIST && (!APPROX || NCODES % THREADS == 0 || NCODES < THREADS),
                  "codes tile the block");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int32_t *out = a.sel + ((size_t)b * a.Hkv + h) * a.k;
    const float *row = a.scores + ((size_t)b * a.Hkv + h) * a.max_pages;
    const int32_t L = a.seq_lens[b];
    if (L < 1 || L > a.max_pages * a.P) {
        for (int i = tid; i < a.k; i += THREADS) out[i] = -1;
        if (tid == 0 && h == 0) set_err(a.err, VX_DATA_BAD_SEQ_LEN);
        return;
    }
    const int n = ceil_div(L, a.P);
    const int keff = min(a.k, n);
    if (keff == n) {  // every page is chosen
        for (int i = tid; i < a.k; i += THREADS) out[i] = i < n ? i : -1;
        return;
    }
    // Everything above reads only inputs of the call, complete before this grid starts (it
    // runs in plain stream order or after the scorer, whose own dependency wait returned before
    // any of its blocks could end); the scores come from the previous kernel.
    if (dependent) pdl_wait();
    const bool in_smem = n <= a.smem_keys;
    if constexpr (!APPROX && THREADS == 256) {
        if (n <= a.warp_max && in_smem) {  // uniform for the block: one warp does the row
            if (warp == 0) warp_topk_small(row, n, keff, out, a.k, skeys, sh.hist);
            return;
        }
    }

    // per-thread contiguous run [r0, r1) used by the ordered compaction; run starts are
    // multiples of 4 so a run is read from shared memory as 16-byte vectors
    const int per = (ceil_div(n, THREADS) + 3) & ~3;
    const int r0 = min(n, tid * per), r1 = min(n, r0 + per);

    uint32_t prefix = 0, mask = 0;  // chosen iff (key & mask) > prefix, or == and rank < remaining
    int remaining = keff;           // slots to take from the boundary bucket
    int offset = 0;                 // approx: start of the cyclic fill
    float lo = 0.f, scale = 0.f;
    bool flat = false;

    if constexpr (!APPROX) {
        // first sweep: keys to shared memory and the histogram of the top digit
        for (int i = tid; i < 2048; i += THREADS) sh.hist[i] = 0;
        __syncthreads();
        sweep_row<THREADS>(row, n, [&](int j, float v) {
            const uint32_t key = order_key(v);
            if (in_smem) skeys[j] = key;
            atomicAdd(&sh.hist[key >> 21], 1);
        });
        __syncthreads();
#pragma unroll
        for (int pass = 0; pass < 3; ++pass) {
            const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
            const int bins = pass == 2 ? 1024 : 2048;
            const uint32_t dmask = (uint32_t)bins - 1u;
            if (pass > 0) {
                for (int i = tid; i < bins; i += THREADS) sh.hist[i] = 0;
                __syncthreads();
                for (int j = tid; j < n; j += THREADS) {
                    const uint32_t key = in_smem ? skeys[j] : order_key(row[j]);
                    if ((key & mask) == prefix) atomicAdd(&sh.hist[(key >> shift) & dmask], 1);
                }
                __syncthreads();
            }
            block_find_bin<THREADS>(sh, bins, remaining);
            const int digit = sh.bcast[0], above = sh.bcast[1], cnt = sh.bcast[2];
            remaining -= above;
            prefix |= static_cast<uint32_t>(digit) << shift;
            mask |= dmask << shift;
            __syncthreads();
            if (cnt == remaining) break;  // the whole boundary bucket is taken
        }
    } else {
        // row min / max
        // first sweep: min / max, raw scores staged in shared memory
        float mn = INFINITY, mx = -INFINITY;
        sweep_row<THREADS>(row, n, [&](int j, float v) {
            if (in_smem) skeys[j] = __float_as_uint(v);
            mn = fminf(mn, v);
            mx = fmaxf(mx, v);
        });
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(FULL, mn, off));
            mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, off));
        }
        if (lane == 0) {
            sh.fmin[warp] = mn;
            sh.fmax[warp] = mx;
        }
        for (int i = tid; i < NCODES; i += THREADS) sh.hist[i] = 0;
        __syncthreads();
        mn = sh.fmin[0];
        mx = sh.fmax[0];
        for (int w = 1; w < THREADS / 32; ++w) {
            mn = fminf(mn, sh.fmin[w]);
            mx = fmaxf(mx, sh.fmax[w]);
        }
        lo = mn;
        const float range = __fsub_rn(mx, mn);
        scale = __fdiv_rn(static_cast<float>(NCODES), range);
        flat = !(mx > mn) || isinf(scale);
        for (int j = tid; j < n; j += THREADS) {  // each thread rereads only what it staged
            uint32_t code = 0;
            if (!flat) {
                const float v = in_smem ? __uint_as_float(skeys[j]) : row[j];
                const float f = floorf(__fmul_rn(__fsub_rn(v, lo), scale));
                code = f >= float(NCODES - 1) ? NCODES - 1 : static_cast<uint32_t>(f);
            }
            if (in_smem) skeys[j] = code;
            atomicAdd(&sh.hist[code], 1);
        }
        __syncthreads();
        block_find_bin<THREADS>(sh, NCODES, keff);
        prefix = static_cast<uint32_t>(sh.bcast[0]);
        mask = 0xffffffffu;
        remaining = keff - sh.bcast[1];
        offset = static_cast<int>(splitmix64(a.seed, (uint64_t)b * a.Hkv + h) % (uint64_t)n);
    }

    // the key of page j computed from its score (rows too long for shared memory)
    auto key_of_row = [&](int j) -> uint32_t {
        if constexpr (APPROX) {
            if (flat) return 0u;
            const float f = floorf(__fmul_rn(__fsub_rn(row[j], lo), scale));
            return f >= float(NCODES - 1) ? NCODES - 1 : static_cast<uint32_t>(f);
        } else {
            return order_key(row[j]);
        }
    };
    // calls fn(j, key of page j) for the pages j of this thread's run, in order
    auto run_keys = [&](auto &&fn) {
        if (in_smem) {
            for (int j4 = r0; j4 < r1; j4 += 4) {
                const uint4 k4 = *reinterpret_cast<const uint4 *>(skeys + j4);
                const uint32_t kk[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (j4 + e < r1) fn(j4 + e, kk[e]);
            }
        } else {
            for (int j = r0; j < r1; ++j) fn(j, key_of_row(j));
        }
    };
    if (dependent) pdl_trigger();  // the decode kernel may land now; only the compaction is left
    // -------- ordered compaction
    if constexpr (!APPROX) {
        // one counting sweep: keys above the boundary bucket and in it, per thread run; one
        // scan of both (packed in 64 bits) gives each run its first output slot, since the
        // bucket's members go out in page order until the slots left are used
        unsigned long long cnt = 0;
        run_keys([&](int, uint32_t key) {
            const uint32_t mk = key & mask;
            cnt += mk > prefix ? (1ull << 32) : (mk == prefix ? 1ull : 0ull);
        });
        unsigned long long tot;
        const unsigned long long before = block_exclusive_scan<THREADS, unsigned long long>(cnt, sh.scan_tmp64, tot);
        int eq_rank = static_cast<int>(before & 0xffffffffu);
        int pos = static_cast<int>(before >> 32) + min(eq_rank, remaining);
        const int sel_total = static_cast<int>(tot >> 32) + min(static_cast<int>(tot & 0xffffffffu), remaining);
        run_keys([&](int j, uint32_t key) {
            const uint32_t mk = key & mask;
            bool take = mk > prefix;
            if (mk == prefix) take = eq_rank++ < remaining;
            if (take) {
                if (pos < a.k) out[pos] = j;
                ++pos;
            }
        });
        for (int i = sel_total + tid; i < a.k; i += THREADS) out[i] = -1;
        return;
    }
    // approx: members of the boundary code are taken in cyclic page order from `offset`: first
    // those at or after it (take_hi of them), then those before it (take_lo).  One counting
    // sweep per run (above / member / member before the offset) and one scan give each run
    // its first output slot.
    int gt_l = 0, eq_l = 0, lo_l = 0;
    run_keys([&](int j, uint32_t key) {
        const uint32_t mk = key & mask;
        if (mk > prefix) ++gt_l;
        else if (mk == prefix) {
            ++eq_l;
            if (j < offset) ++lo_l;
        }
    });
    int gt_before, eq_before, lo_before, gt_total, eq_total, lo_total;
    if (n < (1 << 21)) {  // three 21-bit counts in one 64-bit scan
        const unsigned long long v = ((unsigned long long)gt_l << 42) | ((unsigned long long)eq_l << 21) | (unsigned long long)lo_l;
        unsigned long long tot;
        const unsigned long long bef = block_exclusive_scan<THREADS, unsigned long long>(v, sh.scan_tmp64, tot);
        constexpr unsigned long long M21 = (1ull << 21) - 1ull;
        gt_before = (int)(bef >> 42);
        eq_before = (int)((bef >> 21) & M21);
        lo_before = (int)(bef & M21);
        gt_total = (int)(tot >> 42);
        eq_total = (int)((tot >> 21) & M21);
        lo_total = (int)(tot & M21);
    } else {
        const unsigned long long v = ((unsigned long long)gt_l << 32) | (unsigned long long)eq_l;
        unsigned long long tot;
        const unsigned long long bef = block_exclusive_scan<THREADS, unsigned long long>(v, sh.scan_tmp64, tot);
        gt_before = (int)(bef >> 32);
        eq_before = (int)(bef & 0xffffffffu);
        gt_total = (int)(tot >> 32);
        eq_total = (int)(tot & 0xffffffffu);
        lo_before = block_exclusive_scan<THREADS>(lo_l, sh.scan_tmp, lo_total);
    }
    const int take_hi = min(remaining, eq_total - lo_total);
    const int take_lo = min(lo_total, remaining - take_hi);
    int pos = gt_before + min(lo_before, take_lo) + min(eq_before - lo_before, take_hi);
    const int sel_total = gt_total + take_hi + take_lo;
    {
        int lo_rank = lo_before, hi_rank = eq_before - lo_before;
        run_keys([&](int j, uint32_t key) {
            const uint32_t mk = key & mask;
            bool take = mk > prefix;
            if (mk == prefix) take = (j < offset) ? lo_rank++ < take_lo : hi_rank++ < take_hi;
            if (take) {
                if (pos < a.k) out[pos] = j;
                ++pos;
            }
        });
    }
    for (int i = sel_total + tid; i < a.k; i += THREADS) out[i] = -1;
}

}  // namespace vx
