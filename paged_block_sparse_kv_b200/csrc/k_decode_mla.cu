// k_decode_mla.cu -- exact attention over the selected pages for the MLA geometry.
#include "vx_internal.h"

namespace vx {

cudaError_t launch_decode_mla(const DecodeArgs &, const CUtensorMap &, int, cudaStream_t, bool) {
    return cudaErrorNotSupported;
}

}  // namespace vx
