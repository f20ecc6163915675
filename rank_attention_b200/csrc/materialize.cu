// The non-shared baseline's cache: every agent's full keys and values,
//   K^a_t = K_base,t + RoPE_t(s LRk_t B_k^a),   V^a_t = V_base,t + s LRv_t B_v^a,
// written to memory (what a system without cache sharing keeps per agent;
// LRAgent summary §3, the Non-Shared and FullShared baselines).  Attention over
// these caches reads n_agents times the base cache; the shared path never
// writes them.
//
// One thread per (sequence, position, frequency pair): the RoPE angle is
// reduced once in fp64 and reused for every agent and KV head; B^a rows are
// read coalesced across the pair index and stay in L1 across the block's
// positions.
#include <cmath>

#include <cuda_bf16.h>

#include "bf16_common.cuh"
#include "la_internal.cuh"

namespace la {
namespace {

template <typename IO>
__device__ __forceinline__ float ld_io(const IO* p);
template <>
__device__ __forceinline__ float ld_io<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ld_io<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }
template <typename IO>
__device__ __forceinline__ IO st_cvt(float x);
template <>
__device__ __forceinline__ float st_cvt<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 st_cvt<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

constexpr int kMatThreads = 256;

template <typename IO, int R>
__global__ void __launch_bounds__(kMatThreads) materialize_kernel(AttnParams p, RopeTheta rt, IO* kout,
                                                                   IO* vout) {
  const int D = p.d, H2 = D / 2;
  const int tok_per_block = kMatThreads / H2;
  const int seq = blockIdx.y;
  const int64_t t = (int64_t)blockIdx.x * tok_per_block + threadIdx.x / H2;
  const int i = threadIdx.x % H2;
  if (t >= p.max_kv_len) return;
  const float2 cs = rope_cs_exact(t, rt.theta[i]);
  const IO* lr = reinterpret_cast<const IO*>(p.lr) + seq * p.lr_seq + t * 2 * R;
  float lk[R], lv[R];
  const int64_t ldB = (int64_t)p.n_kv * D;
  const IO* Bk = reinterpret_cast<const IO*>(p.B_k);
  const IO* Bv = reinterpret_cast<const IO*>(p.B_v);
  for (int a = 0; a < p.n_agents; ++a) {
    if (a == 0 || p.lr_agent) {  // the shared LR row, or agent a's own
#pragma unroll
      for (int m = 0; m < R; ++m) {
        lk[m] = ld_io(lr + a * p.lr_agent + m);
        lv[m] = ld_io(lr + a * p.lr_agent + R + m);
      }
    }
    for (int j = 0; j < p.n_kv; ++j) {
      const IO* bk = Bk + (int64_t)a * R * ldB + j * D + i;
      const IO* bv = Bv + (int64_t)a * R * ldB + j * D + i;
      float x1 = 0.f, x2 = 0.f, w1 = 0.f, w2 = 0.f;
#pragma unroll
      for (int m = 0; m < R; ++m) {
        x1 = fmaf(lk[m], ld_io(bk + m * ldB), x1);
        x2 = fmaf(lk[m], ld_io(bk + m * ldB + H2), x2);
        w1 = fmaf(lv[m], ld_io(bv + m * ldB), w1);
        w2 = fmaf(lv[m], ld_io(bv + m * ldB + H2), w2);
      }
      const IO* kb = reinterpret_cast<const IO*>(p.k_base) + seq * p.kv_seq + j * p.kv_head + t * p.kv_tok;
      const IO* vb = reinterpret_cast<const IO*>(p.v_base) + seq * p.kv_seq + j * p.kv_head + t * p.kv_tok;
      const int64_t o = ((((int64_t)seq * p.n_agents + a) * p.n_kv + j) * p.L_max + t) * D;
      kout[o + i] = st_cvt<IO>(ld_io(kb + i) + p.s * (x1 * cs.x - x2 * cs.y));
      kout[o + i + H2] = st_cvt<IO>(ld_io(kb + i + H2) + p.s * (x2 * cs.x + x1 * cs.y));
      vout[o + i] = st_cvt<IO>(ld_io(vb + i) + p.s * w1);
      vout[o + i + H2] = st_cvt<IO>(ld_io(vb + i + H2) + p.s * w2);
    }
  }
}

template <typename IO, int R>
cudaError_t launch_r(const AttnParams& p, void* kout, void* vout, cudaStream_t st) {
  RopeTheta rt;
  for (int i = 0; i < 64; ++i) {
    rt.theta[i] = i < p.d / 2 ? std::pow(p.rope_base, -2.0 * i / p.d) : 0.0;
    rt.thetaf[i] = (float)rt.theta[i];
  }
  const int tok_per_block = kMatThreads / (p.d / 2);
  dim3 grid((unsigned)((p.max_kv_len + tok_per_block - 1) / tok_per_block), p.n_seqs);
  materialize_kernel<IO, R><<<grid, kMatThreads, 0, st>>>(p, rt, static_cast<IO*>(kout),
                                                           static_cast<IO*>(vout));
  return cudaGetLastError();
}

template <typename IO>
cudaError_t launch_io(const AttnParams& p, void* kout, void* vout, cudaStream_t st) {
  switch (p.r) {
    case 8: return launch_r<IO, 8>(p, kout, vout, st);
    case 16: return launch_r<IO, 16>(p, kout, vout, st);
    case 32: return launch_r<IO, 32>(p, kout, vout, st);
    default: return launch_r<IO, 64>(p, kout, vout, st);
  }
}

}  // namespace

cudaError_t launch_materialize(const AttnParams& p, la_dtype io, void* kout, void* vout, cudaStream_t st) {
  return io == LA_BF16 ? launch_io<__nv_bfloat16>(p, kout, vout, st) : launch_io<float>(p, kout, vout, st);
}

}  // namespace la
