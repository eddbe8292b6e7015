// Decode-sized M path (placeholder: not yet specialised; the general kernel serves these M).
#include "ss1_internal.cuh"

namespace ss1 {
bool smallm_supported(const ss1_layer&, int64_t) { return false; }
cudaError_t launch_smallm(const ss1_layer&, const void*, const void*, void*, int64_t, cudaStream_t) {
    return cudaErrorNotSupported;
}
}  // namespace ss1
