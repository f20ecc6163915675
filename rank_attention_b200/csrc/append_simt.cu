// lr_cache_append on the CUDA cores: LR[pos0 + i] = X_i [A_k | A_v].
//
// PreLRShared precompute: the low-rank rows of a new context chunk are
// computed once, through the A shared by every agent, and appended to the one
// LR cache all agents read (PReCache abstract and blog; LRAgent summary §3
// BaseLRShared).  Rows are stored unscaled and unrotated, K part first.
//
// This generic kernel accumulates in fp32 and serves fp32 inputs and every
// rank; the bf16 tensor-core kernel covers the large bf16 chunks.
#include "la_internal.cuh"

namespace la {
namespace {

constexpr int NT = 256;
constexpr int TOK = 64;  // chunk rows per CTA
constexpr int HC = 32;   // hidden columns per staged slice

template <typename T, int R>
__global__ void __launch_bounds__(NT) append_simt_kernel(const T* __restrict__ X, int64_t ldx,
                                                          int64_t n, int64_t H,
                                                          const T* __restrict__ A,
                                                          T* __restrict__ lr, int64_t pos0,
                                                          int64_t sx, int64_t slr) {
  constexpr int C = 2 * R;            // output columns
  constexpr int RSTEP = NT / C;       // rows between a thread's outputs
  constexpr int NO = TOK / RSTEP;     // outputs per thread
  __shared__ float Xs[TOK][HC + 1];
  __shared__ float As[HC][C];
  const int seq = blockIdx.y;
  const int64_t t0 = (int64_t)blockIdx.x * TOK;
  const int tid = threadIdx.x;
  const int col = tid % C, r0 = tid / C;
  const T* Xq = X + seq * sx;
  float acc[NO];
#pragma unroll
  for (int k = 0; k < NO; ++k) acc[k] = 0.f;

  for (int64_t h0 = 0; h0 < H; h0 += HC) {
    for (int i = tid; i < TOK * HC; i += NT) {
      const int t = i / HC, h = i % HC;
      float v = 0.f;
      if (t0 + t < n && h0 + h < H) v = to_f32(Xq[(t0 + t) * ldx + h0 + h]);
      Xs[t][h] = v;
    }
    for (int i = tid; i < HC * C; i += NT) {
      const int h = i / C, c = i % C;
      As[h][c] = (h0 + h < H) ? to_f32(A[(h0 + h) * C + c]) : 0.f;
    }
    __syncthreads();
#pragma unroll 4
    for (int h = 0; h < HC; ++h) {
      const float a = As[h][col];
#pragma unroll
      for (int k = 0; k < NO; ++k) acc[k] = fmaf(Xs[r0 + k * RSTEP][h], a, acc[k]);
    }
    __syncthreads();
  }
  T* out = lr + seq * slr + pos0 * C;
#pragma unroll
  for (int k = 0; k < NO; ++k) {
    const int64_t t = t0 + r0 + k * RSTEP;
    if (t < n) out[t * C + col] = from_f32<T>(acc[k]);
  }
}

template <typename T>
cudaError_t launch_r(const void* X, int64_t ldx, int64_t n, int64_t H, const void* A, int r,
                     void* lr, int64_t pos0, int n_seqs, int64_t sx, int64_t slr,
                     cudaStream_t st) {
  dim3 grid((unsigned)((n + TOK - 1) / TOK), n_seqs);
  const T* x = static_cast<const T*>(X);
  const T* a = static_cast<const T*>(A);
  T* o = static_cast<T*>(lr);
  switch (r) {
    case 8: append_simt_kernel<T, 8><<<grid, NT, 0, st>>>(x, ldx, n, H, a, o, pos0, sx, slr); break;
    case 16: append_simt_kernel<T, 16><<<grid, NT, 0, st>>>(x, ldx, n, H, a, o, pos0, sx, slr); break;
    case 32: append_simt_kernel<T, 32><<<grid, NT, 0, st>>>(x, ldx, n, H, a, o, pos0, sx, slr); break;
    case 64: append_simt_kernel<T, 64><<<grid, NT, 0, st>>>(x, ldx, n, H, a, o, pos0, sx, slr); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_append_simt(const void* X, int64_t ldx, int64_t n, int64_t H, const void* A,
                               int r, void* lr, int64_t pos0, int n_seqs, int64_t sx,
                               int64_t slr, la_dtype dt, cudaStream_t st) {
  if (dt == LA_F32) return launch_r<float>(X, ldx, n, H, A, r, lr, pos0, n_seqs, sx, slr, st);
  return launch_r<__nv_bfloat16>(X, ldx, n, H, A, r, lr, pos0, n_seqs, sx, slr, st);
}

}  // namespace la
