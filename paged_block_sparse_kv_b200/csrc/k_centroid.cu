// k_centroid.cu -- cache stage: per-page key centroid (rebuild and decode-append).
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

template <int D>
static cudaError_t launch_centroid_d(const CentroidArgs &a, bool append, cudaStream_t s) {
    if (append) {
        k_centroid_append<D><<<a.B, a.Hkv * 32, 0, s>>>(a);
    } else {
        dim3 grid((a.max_pages + CEN_PAGES_PER_BLOCK - 1) / CEN_PAGES_PER_BLOCK, a.B);
        k_centroid_rebuild<D><<<grid, CEN_WARPS * 32, 0, s>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_centroid(const CentroidArgs &a, bool append, cudaStream_t s) {
    switch (a.Dqk) {
        case 64: return launch_centroid_d<64>(a, append, s);
        case 128: return launch_centroid_d<128>(a, append, s);
        case 576: return launch_centroid_d<576>(a, append, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace vx
