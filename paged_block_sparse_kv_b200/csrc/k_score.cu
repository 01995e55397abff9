// k_score.cu -- indexer: group-summed query . page centroid for every page of a request.
//
// Vortex paper note, section 系统设计 1: blocks are scored by a matrix product of the
// current query with the cached centroids; the MLA experiment section scores on the
// 576-dim latent + rope key (rope-aware) and, as a variant, on the 512 latent dims.
//
// The contraction over the G query heads of a KV group is done first (fp32, exact for a
// few bf16 values), so the kernel is a GEMV per (request, KV head): it streams each
// page's centroid row (all KV heads contiguous, Hkv * Dqk bf16) once with 16-byte
// non-coherent loads, several pages in flight per warp.  Each lane keeps the summed
// query for the 8 dims it multiplies in registers; partial dots of one head are
// combined with XOR shuffles inside the lane segment that covers that head.
#include "vx_internal.h"

namespace vx {

constexpr int SCORE_MAX_ITS = 4;  // 16-byte loads per lane per page (Hkv * Dqk <= 1024)

template <int D>
__global__ void __launch_bounds__(SCORE_WARPS * 32) k_score_pages(ScoreArgs a) {
    pdl_launch_dependents();
    pdl_wait();  // q and the centroids may be written by the previous kernel
    constexpr int CH = D / 8;                 // 16-byte chunks per head row
    constexpr bool SEGMENTED = CH <= 32;      // a head row fits in a lane segment
    const int b = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t L = a.seq_lens[b];
    if (L < 1 || L > a.max_pages * a.P) {
        if (blockIdx.x == 0 && threadIdx.x == 0) set_err(a.err, VX_DATA_BAD_SEQ_LEN);
        return;
    }
    const int n = ceil_div(L, a.P);
    const int j_lo = blockIdx.x * SCORE_PAGES_PER_BLOCK;
    if (j_lo >= n) return;
    const int j_hi = min(n, j_lo + SCORE_PAGES_PER_BLOCK);
    const int E = a.Hkv * CH;  // chunks per page row

    extern __shared__ float qsum[];  // [Hkv][D]
    for (int i = threadIdx.x; i < a.Hkv * D; i += blockDim.x) {
        const int h = i / D, d = i % D;
        float s = 0.f;
        if (d < a.score_dims) {
            const __nv_bfloat16 *qb = a.q + ((size_t)b * a.Hq + (size_t)h * a.G) * D + d;
            for (int g = 0; g < a.G; ++g) s += __bfloat162float(qb[(size_t)g * D]);
        }
        qsum[i] = s;
    }
    __syncthreads();

    // this lane's chunks are the same for every page: keep their query values in registers
    float qreg[SCORE_MAX_ITS][8];
#pragma unroll
    for (int it = 0; it < SCORE_MAX_ITS; ++it) {
        const int ci = it * 32 + lane;
#pragma unroll
        for (int i = 0; i < 8; ++i) qreg[it][i] = (ci < E) ? qsum[ci * 8 + i] : 0.f;
    }

    const int32_t *row = a.page_indices + a.page_ptr[b];
    for (int jb = j_lo + warp * SCORE_UNROLL; jb < j_hi; jb += SCORE_WARPS * SCORE_UNROLL) {
        int32_t phys[SCORE_UNROLL];
        uint4 v[SCORE_UNROLL][SCORE_MAX_ITS];
#pragma unroll
        for (int u = 0; u < SCORE_UNROLL; ++u) {
            const int j = jb + u;
            phys[u] = -1;
            if (j < j_hi) {
                const int32_t p = row[j];
                if (p >= 0 && p < a.num_pool_pages) phys[u] = p;
                else if (lane == 0) set_err(a.err, VX_DATA_BAD_PAGE_ID);
            }
        }
#pragma unroll
        for (int u = 0; u < SCORE_UNROLL; ++u) {
            const __nv_bfloat16 *c = a.centroids + (size_t)max(phys[u], 0) * a.Hkv * D;
#pragma unroll
            for (int it = 0; it < SCORE_MAX_ITS; ++it) {
                const int ci = it * 32 + lane;
                v[u][it] = (phys[u] >= 0 && ci < E) ? ld_nc_v4(c + ci * 8) : make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int u = 0; u < SCORE_UNROLL; ++u) {
            if (phys[u] < 0) continue;  // warp-uniform
            const int j = jb + u;
            float tot = 0.f;
#pragma unroll
            for (int it = 0; it < SCORE_MAX_ITS; ++it) {
                if (it * 32 >= E) break;
                float f[8];
                bf16x8_to_f32(v[u][it], f);
                float dot = 0.f;
#pragma unroll
                for (int i = 0; i < 8; ++i) dot = fmaf(f[i], qreg[it][i], dot);
                if constexpr (SEGMENTED) {
#pragma unroll
                    for (int off = CH / 2; off > 0; off >>= 1) dot += __shfl_xor_sync(FULL, dot, off);
                    const int ci = it * 32 + lane;
                    if ((lane % CH) == 0 && ci < E) {
                        const int h = ci / CH;
                        a.scores[((size_t)b * a.Hkv + h) * a.max_pages + j] = dot;
                    }
                } else {
                    tot += dot;
                }
            }
            if constexpr (!SEGMENTED) {
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) tot += __shfl_xor_sync(FULL, tot, off);
                if (lane == 0) a.scores[(size_t)b * a.Hkv * a.max_pages + j] = tot;  // Hkv == 1
            }
        }
    }
}

template <int D>
static cudaError_t launch_score_d(const ScoreArgs &a, cudaStream_t s, bool pdl) {
    dim3 grid((a.max_pages + SCORE_PAGES_PER_BLOCK - 1) / SCORE_PAGES_PER_BLOCK, a.B);
    const size_t smem = sizeof(float) * a.Hkv * D;
    return launch_k(k_score_pages<D>, grid, dim3(SCORE_WARPS * 32), smem, s, pdl, a);
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
