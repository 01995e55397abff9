// k_topk.cu -- top-k pages per (request, KV head) row of scores: one block per row (256
// threads for rows up to 1024 pages, 512 up to TOPK_SMALL_MAX when the launch has few rows,
// 1024 beyond); the selection itself is topk_row in vx_topk.cuh.  In launches with at least
// 4 rows per SM, exact rows of at most TOPK_WARP_MAX pages are done by one warp of the block.
#include "vx_topk.cuh"

namespace vx {

template <int ABITS, int THREADS>
__global__ void __launch_bounds__(THREADS, THREADS >= 1024 ? 1 : 2048 / THREADS) k_topk(TopkArgs a) {
    __shared__ TopkShared sh;
    extern __shared__ __align__(16) uint32_t skeys[];  // a.smem_keys entries, rounded up to 4
    topk_row<ABITS, THREADS>(a, blockIdx.y, blockIdx.x, sh, skeys, true);
}

template <int THREADS>
static cudaError_t launch_topk_t(const TopkArgs &a, int mode, cudaStream_t s, bool pdl) {
    const dim3 grid(a.Hkv, a.B);
    const size_t smem = sizeof(uint32_t) * (size_t)((a.smem_keys + 3) & ~3);  // 16-byte run reads
    auto kern = mode == 0   ? k_topk<0, THREADS>
                : mode == 1 ? k_topk<APPROX_BITS, THREADS>
                : mode == 2 ? k_topk<APPROX_BITS_FAST, THREADS>
                            : k_topk<APPROX_BITS_COARSE, THREADS>;
    static std::atomic<unsigned long long> done[4];
    cudaError_t e = ensure_smem_limit(kern, (int)(sizeof(uint32_t) * TOPK_SMEM_KEYS), done[mode]);
    if (e != cudaSuccess) return e;
    return launch_k(kern, grid, dim3(THREADS), smem, s, pdl, a);
}

cudaError_t launch_topk(const TopkArgs &a, int mode, cudaStream_t s, bool pdl) {
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return e;
    TopkArgs b = a;
    b.warp_max = (int64_t)a.B * a.Hkv >= 4 * (int64_t)sms ? TOPK_WARP_MAX : 0;
    // few rows of 1025..TOPK_SMALL_MAX pages: 512 threads shorten a row's sweeps (measured: 75.2
    // against 76.0 us per headline step, 256 rows of up to 2048 pages); with many rows the
    // one-warp path of the 256-thread block is the faster one
    if (a.max_pages > 1024 && a.max_pages <= TOPK_SMALL_MAX && b.warp_max == 0)
        return launch_topk_t<512>(b, mode, s, pdl);
    if (a.max_pages <= TOPK_SMALL_MAX) return launch_topk_t<256>(b, mode, s, pdl);
    return launch_topk_t<1024>(b, mode, s, pdl);
}

}  // namespace vx
