// Tensor-core (tcgen05 + TMEM + TMA) selection+local attention: not yet built.
#include "bsa_internal.cuh"

namespace bsa {
cudaError_t launch_attend_tc(const Problem &, const void *, const void *, const void *, const float *,
                             const float *, const int32_t *, void *, uint32_t *, cudaStream_t) {
    return cudaErrorNotSupported;
}
}  // namespace bsa
