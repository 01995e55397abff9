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
// VX_NOALLOC_SCRATCH_BYTES of it until the process exits.  It is placed in device
// memory when the CUDA module of this file is loaded: with lazy module loading (the
// default since CUDA 12.2) that happens at the first call on a device, so that call
// needs 16 MiB of free device memory.  In host code `g_scratch` is only a host-side
// stand-in for the symbol, never a device address: the address a kernel may use is
// looked up with cudaGetSymbolAddress, with the device current, once per device and
// CUDA context (a device reset makes a new context, whose array may sit elsewhere).
#include <cudaTypedefs.h>

#include <cstdio>
#include <mutex>

#include "vx_internal.h"

namespace {

__device__ __align__(256) unsigned char g_scratch[VX_NOALLOC_SCRATCH_BYTES];

struct ScratchEntry {
    unsigned long long ctx_id;  // the context the address belongs to (0: none yet)
    void *ptr;
};
std::mutex g_scratch_mu;
ScratchEntry g_scratch_dev[64] = {};  // per device ordinal

// Driver entry points for the current context's unique id (fetched through the runtime;
// the library links the runtime statically and does not link the driver library).
struct CtxFns {
    PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
    PFN_cuCtxGetId_v12000 get_id = nullptr;
};
const CtxFns &ctx_fns() {
    static CtxFns f;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void *p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            f.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            f.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
    });
    return f;
}

// unique id of the calling thread's current context, 0 if there is none or it cannot be read
unsigned long long current_ctx_id() {
    const CtxFns &f = ctx_fns();
    if (!f.get_current || !f.get_id) return 0;
    CUcontext ctx = nullptr;
    if (f.get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
    unsigned long long id = 0;
    if (f.get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

}  // namespace

extern "C" vx_status vx_sparse_decode_noalloc(const vx_geometry *geo, const vx_page_table *table, const void *q,
                                              const void *k_cache, const void *v_cache, const int32_t *sel,
                                              int32_t k, float sm_scale, int32_t num_splits, void *out, float *lse,
                                              int32_t *err, void *stream) {
    if (!table) return vx::set_error(VX_ERR_INVALID_ARG, "page table is NULL");
    size_t need = 0;
    vx_status st = vx::compact_partial_bytes(geo, table->max_pages, k, num_splits, &need);
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
        const unsigned long long id = current_ctx_id();
        ScratchEntry &ent = g_scratch_dev[dev];
        if (!ent.ptr || id == 0 || ent.ctx_id != id) {
            void *p = nullptr;
            e = cudaGetSymbolAddress(&p, g_scratch);  // on the current device; loads the module if needed
            if (e != cudaSuccess || !p) {
                char msg[160];
                snprintf(msg, sizeof msg, "cudaGetSymbolAddress of the scratch array failed: %s",
                         cudaGetErrorString(e));
                return vx::set_error(VX_ERR_CUDA, msg);
            }
            ent.ptr = p;
            ent.ctx_id = current_ctx_id();  // the context exists now, whatever it was before the lookup
        }
        scratch = ent.ptr;
    }
    return vx::sparse_decode_compact(geo, table, q, k_cache, v_cache, sel, k, sm_scale, num_splits, out, lse,
                                     scratch, VX_NOALLOC_SCRATCH_BYTES, err, static_cast<cudaStream_t>(stream));
}
