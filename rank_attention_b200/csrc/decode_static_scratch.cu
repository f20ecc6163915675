// lora_attn_decode_static_scratch: lora_attn_decode without a caller workspace.
//
// Some callers cannot hand the library device memory: a plugin inside a
// serving runtime whose arena allocator owns every device allocation, or a
// process that plans its device memory once up front and may not grow it.
// For them the decode's split-K scratch (per-split partial results and the
// arrival counters) lives in one file-scope device array of kStaticScratchBytes
// instead of a workspace.  The caller still passes every input and output.
#include "la_internal.cuh"

namespace la {
bool decode_counter_range(const la_attn_args* a, size_t* offset, size_t* bytes);
la_status decode_args_status(const la_attn_args* a);
namespace {

constexpr size_t kStaticScratchBytes = LA_STATIC_SCRATCH_BYTES;  // held on every device using the library

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of the array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up on
// every call (a host-side query, cheap): nothing cached can go stale when a
// context is torn down and rebuilt.
void* scratch_on_current_device() {
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return ptr;
}

}  // namespace
}  // namespace la

extern "C" la_status lora_attn_decode_static_scratch(const la_attn_args* args, la_stream_t stream) {
  const size_t need = lora_attn_decode_workspace_bytes(args);
  // no scratch needed: invalid arguments (reported as lora_attn_decode would),
  // an empty batch, or a decode that needs no workspace (run as it is)
  if (need == 0) {
    const la_status st = la::decode_args_status(args);
    return st != LA_OK ? st : lora_attn_decode(args, nullptr, 0, stream);
  }
  if (need > la::kStaticScratchBytes) return LA_ERR_SCRATCH_LIMIT;
  void* ptr = la::scratch_on_current_device();
  if (!ptr) return LA_ERR_CUDA;
  // The array keeps whatever the previous call left in it, which may have had
  // other shapes: clear the arrival counters this decode relies on.  The
  // partials need no clearing (every split writes its own before any reads).
  size_t off = 0, bytes = 0;
  if (!la::decode_counter_range(args, &off, &bytes)) return LA_ERR_INVALID_ARG;
  if (cudaMemsetAsync(static_cast<unsigned char*>(ptr) + off, 0, bytes,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return LA_ERR_CUDA;
  return lora_attn_decode(args, ptr, la::kStaticScratchBytes, stream);
}
