// Persistent whole-stack decode kernel.
#include "spffn_fused.cuh"

namespace spffn {
bool fused_decode_supported(spffn_ctx* const*, int, int) { return false; }
cudaError_t launch_fused_decode(spffn_ctx* const*, int, const void*, int, void*, float*, int32_t*, cudaStream_t) {
    return cudaErrorNotSupported;
}
}  // namespace spffn
