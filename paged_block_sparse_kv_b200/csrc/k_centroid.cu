// k_centroid.cu -- cache stage: per-page key centroid (rebuild, decode-append, and the
// prefill write of many tokens per request with the centroids of the pages they touch).
//
// Vortex paper note, section 系统设计 1: block top-k keeps, per KV block (page), the mean
// of the page's keys as a query-independent statistic, updated as tokens are appended.
//
// One warp computes one (page, KV head) centroid.  Keys are read with 16-byte
// non-coherent loads (one lane = 8 bf16 of a row); for head dims whose row is at most a
// warp wide, several rows are read per instruction and the partial sums are combined
// with XOR shuffles.  Sums are taken in fp64, where a sum of up to 64 bf16 values is
// exact, the mean is one IEEE fp64 division, and the stored bf16 is a single
// round-to-nearest-even of that double (no fp32 detour), so the stored centroid is the
// correctly rounded mean.
#include "vx_internal.h"

namespace vx {

// Round a double to the nearest bf16, ties to even, directly from the double.
__device__ __forceinline__ uint16_t f64_to_bf16_rne(double x) {
    const unsigned long long u = static_cast<unsigned long long>(__double_as_longlong(x));
    const uint16_t sign = static_cast<uint16_t>((u >> 48) & 0x8000u);
    const int ebits = static_cast<int>((u >> 52) & 0x7ff);
    if (ebits == 0x7ff) return (u & 0xfffffffffffffull) ? uint16_t(0x7fc0) : uint16_t(sign | 0x7f80);
    const double ax = fabs(x);
    if (ax == 0.0) return sign;
    const int e = ebits - 1023;  // ax in [2^e, 2^(e+1)) for normal doubles (ours always are)
    if (e < -126) {
        // bf16 subnormal range: spacing 2^-133
        const long long q = __double2ll_rn(ax * 0x1p133);  // exact scaling, RNE to integer
        return static_cast<uint16_t>(sign | static_cast<uint16_t>(q));  // q == 128 -> min normal
    }
    // 8 significant bits: scale into [128, 256) and round to an integer, ties to even
    long long q = __double2ll_rn(scalbn(ax, 7 - e));
    int ee = e;
    if (q == 256) {
        q = 128;
        ++ee;
    }
    if (ee > 127) return static_cast<uint16_t>(sign | 0x7f80);
    return static_cast<uint16_t>(sign | ((ee + 127) << 7) | (static_cast<int>(q) & 0x7f));
}

// Centroid of rows [0, m) of one (page, head) block of D bf16 each, written to `dst`.
// If alt != nullptr, row alt_slot is read from alt instead of the block (the token being
// appended, not yet visible in the cache to this warp).
template <int D>
__device__ __forceinline__ void centroid_warp(const __nv_bfloat16 *__restrict__ rows, int m,
                                              const __nv_bfloat16 *__restrict__ alt, int alt_slot,
                                              __nv_bfloat16 *__restrict__ dst, int lane) {
    constexpr int CPR = D / 8;  // 16-byte chunks per row
    if constexpr (CPR <= 32) {
        static_assert(32 % CPR == 0, "row chunks must tile a warp");
        constexpr int RPL = 32 / CPR;  // rows per warp-wide load
        const int chunk = lane % CPR;
        double acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0;
#pragma unroll 4
        for (int t = lane / CPR; t < m; t += RPL) {
            const void *src = (t == alt_slot) ? static_cast<const void *>(alt + chunk * 8)
                                              : static_cast<const void *>(rows + (size_t)t * D + chunk * 8);
            float f[8];
            bf16x8_to_f32(ld_nc_v4(src), f);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] += static_cast<double>(f[i]);
        }
#pragma unroll
        for (int off = CPR; off < 32; off <<= 1)
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(FULL, acc[i], off);
        if (lane < CPR) {
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t lo = f64_to_bf16_rne(acc[2 * i] / m);
                const uint32_t hi = f64_to_bf16_rne(acc[2 * i + 1] / m);
                w[i] = lo | (hi << 16);
            }
            *reinterpret_cast<uint4 *>(dst + chunk * 8) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    } else {
        // wide rows (MLA latent + rope): each lane owns whole chunks and walks the rows
        for (int chunk = lane; chunk < CPR; chunk += 32) {
            double acc[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] = 0.0;
#pragma unroll 8
            for (int t = 0; t < m; ++t) {
                const void *src = (t == alt_slot) ? static_cast<const void *>(alt + chunk * 8)
                                                  : static_cast<const void *>(rows + (size_t)t * D + chunk * 8);
                float f[8];
                bf16x8_to_f32(ld_nc_v4(src), f);
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] += static_cast<double>(f[i]);
            }
            uint32_t w[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t lo = f64_to_bf16_rne(acc[2 * i] / m);
                const uint32_t hi = f64_to_bf16_rne(acc[2 * i + 1] / m);
                w[i] = lo | (hi << 16);
            }
            *reinterpret_cast<uint4 *>(dst + chunk * 8) = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

// Rebuild: grid (ceil(max_pages / CEN_PAGES_PER_BLOCK), B); CEN_WARPS warps per block.
template <int D>
__global__ void __launch_bounds__(CEN_WARPS * 32) k_centroid_rebuild(CentroidArgs a) {
    const int b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t L = a.seq_lens[b];
    if (L < 1 || L > a.max_pages * a.P) {
        if (blockIdx.x == 0 && threadIdx.x == 0) set_err(a.err, VX_DATA_BAD_SEQ_LEN);
        return;
    }
    const int n = ceil_div(L, a.P);
    int j_first = 0;
    if (a.first_pos) {
        const int32_t fp = a.first_pos[b];
        j_first = fp <= 0 ? 0 : fp / a.P;
    }
    const int j_lo = j_first + blockIdx.x * CEN_PAGES_PER_BLOCK;
    const int j_hi = min(n, j_lo + CEN_PAGES_PER_BLOCK);
    const int items = (j_hi - j_lo) * a.Hkv;
    const auto *kc = static_cast<const __nv_bfloat16 *>(a.k_cache);
    auto *cen = static_cast<__nv_bfloat16 *>(a.centroids);
    for (int it = warp; it < items; it += CEN_WARPS) {
        const int j = j_lo + it / a.Hkv, h = it % a.Hkv;
        const int32_t phys = a.page_indices[a.page_ptr[b] + j];
        if (phys < 0 || phys >= a.num_pool_pages) {
            if (lane == 0) set_err(a.err, VX_DATA_BAD_PAGE_ID);
            continue;
        }
        const int m = min(a.P, L - j * a.P);
        const size_t blk = (size_t)phys * a.Hkv + h;
        centroid_warp<D>(kc + blk * a.P * D, m, nullptr, -1, cen + blk * D, lane);
    }
}

// Append: grid (B); one warp per KV head.  Writes the new token's K (and V) into its
// slot, then recomputes that page's centroid with the new row taken from k_new.
template <int D>
__global__ void k_centroid_append(CentroidArgs a) {
    // a dependent scorer (vx_block_topk_decode_append) may launch now; it waits for this
    // grid's end and writes before it reads anything
    pdl_trigger();
    const int b = blockIdx.x;
    const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (h >= a.Hkv) return;
    const int32_t L = a.seq_lens[b];
    if (L < 1 || L > a.max_pages * a.P) {
        if (h == 0 && lane == 0) set_err(a.err, VX_DATA_BAD_SEQ_LEN);
        return;
    }
    const int pos = L - 1, j = pos / a.P, slot = pos % a.P;
    const int32_t phys = a.page_indices[a.page_ptr[b] + j];
    if (phys < 0 || phys >= a.num_pool_pages) {
        if (lane == 0) set_err(a.err, VX_DATA_BAD_PAGE_ID);
        return;
    }
    const size_t blk = (size_t)phys * a.Hkv + h;
    auto *kc = static_cast<__nv_bfloat16 *>(a.k_cache);
    const auto *kn = static_cast<const __nv_bfloat16 *>(a.k_new) + ((size_t)b * a.Hkv + h) * D;
    for (int c = lane; c < D / 8; c += 32)
        *reinterpret_cast<uint4 *>(kc + (blk * a.P + slot) * D + c * 8) = ld_nc_v4(kn + c * 8);
    if (!a.mla_shared_kv) {
        auto *vc = static_cast<__nv_bfloat16 *>(a.v_cache);
        const auto *vn = static_cast<const __nv_bfloat16 *>(a.v_new) + ((size_t)b * a.Hkv + h) * a.Dv;
        for (int c = lane; c < a.Dv / 8; c += 32)
            *reinterpret_cast<uint4 *>(vc + (blk * a.P + slot) * a.Dv + c * 8) = ld_nc_v4(vn + c * 8);
    }
    centroid_warp<D>(kc + blk * a.P * D, slot + 1, kn, slot,
                     static_cast<__nv_bfloat16 *>(a.centroids) + blk * D, lane);
}

// New tokens request i writes in a prefill: seq_lens[i] - first_pos[i], or none for a request
// whose length or first position is out of range (reported by its own blocks).
__device__ __forceinline__ int64_t prefill_count(const CentroidArgs &a, int i) {
    const int32_t L = a.seq_lens[i], fp = a.first_pos[i];
    return (L >= 1 && L <= a.max_pages * a.P && fp >= 0 && fp <= L) ? (int64_t)(L - fp) : 0;
}

// One (page, head) of a prefill: rows [first_new, m) come from the packed input (new_row(t))
// and are stored into the page, rows [0, first_new) are the page's older tokens; the fp64
// sum of all m rows gives the centroid, as in centroid_warp.  New rows are loaded in groups
// (4 rows per lane when a row spans at most a warp, 16 for the wide MLA rows, where a lane
// walks every row of its chunk) before any is stored, so a lane keeps several loads in flight.
template <int D, typename RowF>
__device__ __forceinline__ void prefill_page(RowF new_row, __nv_bfloat16 *__restrict__ page_rows, int first_new,
                                             int m, __nv_bfloat16 *__restrict__ dst, int lane) {
    constexpr int CPR = D / 8;  // 16-byte chunks per row
    constexpr int RPL = CPR <= 32 ? 32 / CPR : 1;  // rows per warp-wide pass
    static_assert(CPR > 32 || 32 % CPR == 0, "row chunks must tile a warp");
    constexpr int NG = CPR <= 32 ? 4 : 16;  // rows loaded per group
    for (int chunk0 = CPR <= 32 ? lane % CPR : lane; chunk0 < CPR; chunk0 += 32) {
        const int chunk = chunk0;
        const int t0 = CPR <= 32 ? lane / CPR : 0;
        double acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0;
        auto add = [&](uint4 v) {
            float f[8];
            bf16x8_to_f32(v, f);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[i] += static_cast<double>(f[i]);
        };
        int t = t0;
        for (; t < min(first_new, m); t += RPL) add(ld_nc_v4(page_rows + (size_t)t * D + chunk * 8));
        for (; t < m; t += NG * RPL) {
            uint4 v[NG];
#pragma unroll
            for (int g = 0; g < NG; ++g)
                if (t + g * RPL < m) v[g] = ld_nc_v4(new_row(t + g * RPL) + chunk * 8);
#pragma unroll
            for (int g = 0; g < NG; ++g) {
                if (t + g * RPL < m) {
                    *reinterpret_cast<uint4 *>(page_rows + (size_t)(t + g * RPL) * D + chunk * 8) = v[g];
                    add(v[g]);
                }
            }
        }
        if constexpr (CPR <= 32) {
#pragma unroll
            for (int off = CPR; off < 32; off <<= 1)
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] += __shfl_xor_sync(FULL, acc[i], off);
            if (lane >= CPR) break;
        }
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t lo = f64_to_bf16_rne(acc[2 * i] / m);
            const uint32_t hi = f64_to_bf16_rne(acc[2 * i + 1] / m);
            w[i] = lo | (hi << 16);
        }
        *reinterpret_cast<uint4 *>(dst + chunk * 8) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// Prefill write: grid (ceil(max_pages / CEN_PAGES_PER_BLOCK), B); CEN_WARPS warps per block,
// one warp per (page, KV head) from the page holding first_pos[b] on.  Request b's new rows
// start in the packed input after the new rows of requests 0..b-1 (a block-wide sum).
template <int D>
__global__ void __launch_bounds__(CEN_WARPS * 32) k_centroid_prefill(CentroidArgs a) {
    const int b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __shared__ long long s_part[CEN_WARPS];
    long long part = 0;
    for (int i = threadIdx.x; i < b; i += blockDim.x) part += prefill_count(a, i);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(FULL, part, off);
    if (lane == 0) s_part[warp] = part;
    __syncthreads();
    int64_t row0 = 0;  // packed row of request b's first new token
#pragma unroll
    for (int w = 0; w < CEN_WARPS; ++w) row0 += s_part[w];

    const int32_t L = a.seq_lens[b], fp = a.first_pos[b];
    if (L < 1 || L > a.max_pages * a.P || fp < 0 || fp > L) {
        if (blockIdx.x == 0 && threadIdx.x == 0) set_err(a.err, VX_DATA_BAD_SEQ_LEN);
        return;
    }
    const int n = ceil_div(L, a.P);
    const int j_lo = fp / a.P + blockIdx.x * CEN_PAGES_PER_BLOCK;
    const int j_hi = min(n, j_lo + CEN_PAGES_PER_BLOCK);
    const int items = (j_hi - j_lo) * a.Hkv;  // <= 0 when fp == L or past the last page
    auto *kc = static_cast<__nv_bfloat16 *>(a.k_cache);
    auto *vc = static_cast<__nv_bfloat16 *>(a.v_cache);
    const auto *kn = static_cast<const __nv_bfloat16 *>(a.k_new);
    const auto *vn = static_cast<const __nv_bfloat16 *>(a.v_new);
    auto *cen = static_cast<__nv_bfloat16 *>(a.centroids);
    for (int it = warp; it < items; it += CEN_WARPS) {
        const int j = j_lo + it / a.Hkv, h = it % a.Hkv;
        const int32_t phys = a.page_indices[a.page_ptr[b] + j];
        if (phys < 0 || phys >= a.num_pool_pages) {
            if (lane == 0) set_err(a.err, VX_DATA_BAD_PAGE_ID);
            continue;
        }
        const int m = min(a.P, L - j * a.P);
        const int first_new = max(0, fp - j * a.P);  // slots >= first_new are new tokens
        const size_t blk = (size_t)phys * a.Hkv + h;
        // packed row of slot t (t >= first_new)
        auto row_of = [&](int t) -> int64_t { return row0 + (int64_t)j * a.P + t - fp; };
        if (!a.mla_shared_kv) {
            const int vch = a.Dv / 8;
            const int total = (m - first_new) * vch;
            for (int c0 = lane; c0 < total; c0 += 32 * 4) {
                uint4 v[4];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int c = c0 + g * 32;
                    if (c < total) {
                        const int t = first_new + c / vch, ch = c % vch;
                        v[g] = ld_nc_v4(vn + (row_of(t) * a.Hkv + h) * a.Dv + ch * 8);
                    }
                }
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int c = c0 + g * 32;
                    if (c < total) {
                        const int t = first_new + c / vch, ch = c % vch;
                        *reinterpret_cast<uint4 *>(vc + (blk * a.P + t) * a.Dv + ch * 8) = v[g];
                    }
                }
            }
        }
        prefill_page<D>([&](int t) { return kn + (row_of(t) * a.Hkv + h) * D; }, kc + blk * a.P * D, first_new, m,
                        cen + blk * D, lane);
    }
}

template <int D>
static cudaError_t launch_centroid_d(const CentroidArgs &a, int mode, cudaStream_t s) {
    const dim3 grid((a.max_pages + CEN_PAGES_PER_BLOCK - 1) / CEN_PAGES_PER_BLOCK, a.B);
    if (mode == CEN_APPEND) {
        k_centroid_append<D><<<a.B, a.Hkv * 32, 0, s>>>(a);
    } else if (mode == CEN_PREFILL) {
        k_centroid_prefill<D><<<grid, CEN_WARPS * 32, 0, s>>>(a);
    } else {
        k_centroid_rebuild<D><<<grid, CEN_WARPS * 32, 0, s>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_centroid(const CentroidArgs &a, int mode, cudaStream_t s) {
    switch (a.Dqk) {
        case 64: return launch_centroid_d<64>(a, mode, s);
        case 128: return launch_centroid_d<128>(a, mode, s);
        case 576: return launch_centroid_d<576>(a, mode, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace vx
