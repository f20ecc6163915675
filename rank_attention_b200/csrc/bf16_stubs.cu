// Placeholders for the bf16 tensor-core kernels until they land.
#include "la_internal.cuh"

namespace la {
bool bf16_prefill_supported(const AttnParams&) { return false; }
cudaError_t launch_prefill_bf16(const AttnParams&, la_dtype, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace la
