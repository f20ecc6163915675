// lora_attn_decode_combine: the split-K combine of the decode taken across
// devices (the sequence-sharded decode).  Each of n_parts key slices of the
// same queries was decoded on its own (lora_attn_decode with row_stats), so
// every output row has, per slice p, the normalised output out_p and the
// slice's (M_p, L_p): M_p its largest scaled score in log2 units, L_p the sum
// of 2^(score - M_p) over its keys.  The attention over all the keys is then
//   out = sum_p w_p out_p / sum_p w_p,   w_p = 2^(M_p - M*) L_p,  M* = max_p M_p,
// the online-softmax rescale that merges partial results (the decode's own
// split merge does the same over the splits of one launch).  One warp per
// row, four columns a lane; memory-bound and small (n_parts x rows x d).
#include <cuda_bf16.h>

#include "la_internal.cuh"

namespace la {
namespace {

constexpr int kWarps = 8;   // rows per CTA

template <bool BF16>
__global__ void __launch_bounds__(32 * kWarps) combine_kernel(const void* __restrict__ outs,
                                                              const float2* __restrict__ stats,
                                                              int n_parts, int64_t rows, int d,
                                                              void* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  // the row's largest M over the parts
  float mx = -INFINITY;
  for (int pp = lane; pp < n_parts; pp += 32) mx = fmaxf(mx, stats[(int64_t)pp * rows + row].x);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float tot = 0.f;
  for (int pp = lane; pp < n_parts; pp += 32) {
    const float2 ml = stats[(int64_t)pp * rows + row];
    tot += (ml.y > 0.f && ml.x != -INFINITY) ? exp2f(ml.x - mx) * ml.y : 0.f;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  const float inv = tot > 0.f ? 1.f / tot : 0.f;
  for (int c = 4 * lane; c < d; c += 128) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int pp = 0; pp < n_parts; ++pp) {
      const float2 ml = stats[(int64_t)pp * rows + row];
      if (!(ml.y > 0.f) || ml.x == -INFINITY) continue;   // a slice with no keys for this row
      const float wp = exp2f(ml.x - mx) * ml.y * inv;
      const int64_t off = ((int64_t)pp * rows + row) * d + c;
      float4 v;
      if constexpr (BF16) {
        const uint2 u = *reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(outs) + off);
        const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
        const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
        v = make_float4(a.x, a.y, b.x, b.y);
      } else {
        v = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(outs) + off);
      }
      acc.x = fmaf(wp, v.x, acc.x); acc.y = fmaf(wp, v.y, acc.y);
      acc.z = fmaf(wp, v.z, acc.z); acc.w = fmaf(wp, v.w, acc.w);
    }
    const int64_t oi = row * d + c;
    if constexpr (BF16) {
      const __nv_bfloat162 a = __floats2bfloat162_rn(acc.x, acc.y), b = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 u;
      u.x = *reinterpret_cast<const uint32_t*>(&a);
      u.y = *reinterpret_cast<const uint32_t*>(&b);
      *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(out) + oi) = u;
    } else {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + oi) = acc;
    }
  }
}

bool aligned(const void* ptr, uintptr_t a) { return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) == 0; }

}  // namespace
}  // namespace la

extern "C" la_status lora_attn_decode_combine(const void* outs, const float* stats, int32_t n_parts,
                                              int64_t rows, int32_t d, la_dtype out_dtype, void* out,
                                              la_stream_t stream) {
  using namespace la;
  if (!outs || !stats || !out || n_parts < 1 || rows < 0 || d < 4 || d % 4 != 0)
    return LA_ERR_INVALID_ARG;
  if (out_dtype != LA_F32 && out_dtype != LA_BF16) return LA_ERR_INVALID_ARG;
  const uintptr_t va = out_dtype == LA_F32 ? 16 : 8;   // a lane's four elements in one access
  if (!aligned(outs, va) || !aligned(out, va) || !aligned(stats, 8)) return LA_ERR_INVALID_ARG;
  if (rows == 0) return LA_OK;
  const int64_t blocks = (rows + kWarps - 1) / kWarps;
  if (blocks > 0x7fffffffLL) return LA_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float2* s2 = reinterpret_cast<const float2*>(stats);
  if (out_dtype == LA_BF16)
    combine_kernel<true><<<(unsigned)blocks, 32 * kWarps, 0, st>>>(outs, s2, n_parts, rows, d, out);
  else
    combine_kernel<false><<<(unsigned)blocks, 32 * kWarps, 0, st>>>(outs, s2, n_parts, rows, d, out);
  return cudaGetLastError() == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}
