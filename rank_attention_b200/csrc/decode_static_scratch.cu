// lora_attn_decode_static_scratch: lora_attn_decode without a caller workspace.
//
// Some callers cannot hand the library device memory: a plugin inside a
// serving runtime whose arena allocator owns every device allocation, or a
// process that plans its device memory once up front and may not grow it.
// For them the decode's split-K scratch (per-split partial results and the
// arrival counters) lives in one file-scope device array of kStaticScratchBytes
// instead of a workspace.  The caller still passes every input and output.
#include <mutex>

#include "la_internal.cuh"

namespace la {
bool decode_counter_range(const la_attn_args* a, size_t* offset, size_t* bytes);
namespace {

constexpr size_t kStaticScratchBytes = LA_STATIC_SCRATCH_BYTES;  // held on every device using the library

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[64];  // device address of g_static_scratch, per device

// Device address of the array on the current device.  The first call on a
// device looks it up (the host-side name is only a stand-in, not a device
// address), clears the array and waits for the clear to finish.
void* scratch_on_current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev]) return g_scratch_addr[dev];
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_static_scratch) != cudaSuccess || !ptr) return nullptr;
  if (cudaMemset(ptr, 0, kStaticScratchBytes) != cudaSuccess) return nullptr;
  if (cudaDeviceSynchronize() != cudaSuccess) return nullptr;
  g_scratch_addr[dev] = ptr;
  return ptr;
}

}  // namespace
}  // namespace la

extern "C" la_status lora_attn_decode_static_scratch(const la_attn_args* args, la_stream_t stream) {
  const size_t need = lora_attn_decode_workspace_bytes(args);
  if (need == 0) return lora_attn_decode(args, nullptr, 0, stream);  // reports the argument error
  if (need > la::kStaticScratchBytes) return LA_ERR_SCRATCH_LIMIT;
  void* ptr = la::scratch_on_current_device();
  if (!ptr) return LA_ERR_CUDA;
  // The array keeps whatever the previous call left in it, which may have had
  // other shapes: clear the arrival counters this decode relies on.
  size_t off = 0, bytes = 0;
  if (!la::decode_counter_range(args, &off, &bytes)) return LA_ERR_INVALID_ARG;
  if (cudaMemsetAsync(static_cast<unsigned char*>(ptr) + off, 0, bytes,
                      static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return LA_ERR_CUDA;
  return lora_attn_decode(args, ptr, la::kStaticScratchBytes, stream);
}
