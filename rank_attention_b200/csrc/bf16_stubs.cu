// Placeholders for the bf16 tensor-core kernels until they land.
#include "la_internal.cuh"

namespace la {
bool bf16_decode_supported(const AttnParams&) { return false; }
void bf16_decode_plan(const AttnParams&, int* n_splits, int64_t* split_len, int* rows) {
  *n_splits = 1; *split_len = 0; *rows = 0;
}
cudaError_t launch_decode_bf16(const AttnParams&, la_dtype, cudaStream_t) { return cudaErrorNotSupported; }
bool bf16_prefill_supported(const AttnParams&) { return false; }
cudaError_t launch_prefill_bf16(const AttnParams&, la_dtype, cudaStream_t) { return cudaErrorNotSupported; }
bool bf16_append_supported(int64_t, int) { return false; }
cudaError_t launch_append_bf16_mma(const void*, int64_t, int64_t, int64_t, const void*, int, void*,
                                   int64_t, int, int64_t, int64_t, cudaStream_t) {
  return cudaErrorNotSupported;
}
}  // namespace la
