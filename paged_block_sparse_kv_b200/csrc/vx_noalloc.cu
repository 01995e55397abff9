// vx_noalloc.cu -- sparse decode for callers that cannot allocate device memory.
//
// Some callers of this library cannot call cudaMalloc: an inference engine that hands
// all free HBM to its KV-cache pool at start-up and routes every later allocation
// through its own planner, a plugin interface that passes tensors but no workspace, or
// code that must not risk the device synchronisation cudaMalloc / cudaFree can cause.
// vx_sparse_decode needs a workspace for its split partials; this entry point supplies
// one from a fixed array in the library's own device memory instead.
//
// The array lives at file scope; every GPU that loads this part of the library holds
// VX_NOALLOC_SCRATCH_BYTES of it until the process exits.  In host code `g_scratch` is
// only a host-side stand-in for the symbol, never a device address: the address a
// kernel may use is looked up with cudaGetSymbolAddress, once per device, with that
// device current (the first call on each device does it).
#include <cstdio>
#include <mutex>

#include "vx_internal.h"

namespace {

__device__ __align__(256) unsigned char g_scratch[VX_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void *g_scratch_dev[64] = {nullptr};  // per device ordinal, filled at first use

}  // namespace

extern "C" vx_status vx_sparse_decode_noalloc(const vx_geometry *geo, const vx_page_table *table, const void *q,
                                              const void *k_cache, const void *v_cache, const int32_t *sel,
                                              int32_t k, float sm_scale, int32_t num_splits, void *out, float *lse,
                                              int32_t *err, void *stream) {
    if (!table) return vx::set_error(VX_ERR_INVALID_ARG, "page table is NULL");
    size_t need = 0;
    vx_status st = vx::decode_partial_bytes(geo, table->max_pages, k, num_splits, &need);
    if (st != VX_OK) return st;
    if (need > VX_NOALLOC_SCRATCH_BYTES) {
        char msg[256];
        snprintf(msg, sizeof msg,
                 "this problem needs %zu bytes of split-partial scratch, more than the %zu bytes "
                 "vx_sparse_decode_noalloc holds; use fewer splits or vx_sparse_decode with a workspace",
                 need, (size_t)VX_NOALLOC_SCRATCH_BYTES);
        return vx::set_error(VX_ERR_WORKSPACE, msg);
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return vx::set_error(VX_ERR_CUDA, "cudaGetDevice failed");
    if (dev < 0 || dev >= 64) return vx::set_error(VX_ERR_UNSUPPORTED, "device ordinal >= 64");
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        if (!g_scratch_dev[dev]) {
            void *p = nullptr;
            e = cudaGetSymbolAddress(&p, g_scratch);  // on the current device
            if (e != cudaSuccess || !p) {
                char msg[160];
                snprintf(msg, sizeof msg, "cudaGetSymbolAddress of the scratch array failed: %s",
                         cudaGetErrorString(e));
                return vx::set_error(VX_ERR_CUDA, msg);
            }
            g_scratch_dev[dev] = p;
        }
        scratch = g_scratch_dev[dev];
    }
    return vx_sparse_decode(geo, table, q, k_cache, v_cache, sel, k, sm_scale, num_splits, out, lse, scratch,
                            VX_NOALLOC_SCRATCH_BYTES, err, stream);
}
