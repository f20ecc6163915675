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

// The one new row of a decode step for every sequence q, at row kv_len[q] - 1
// of every LR cache l (one shared, or one per agent with its own A):
// lr[l][q][kv_len[q] - 1] = x[q] A[l].  One CTA per (q, l) streams A[l] in
// 16-byte vectors, every load of a pass issued before the first is used (the
// row is a few hundred kilobytes of A against one SM's memory pipe): a thread
// keeps one vector column of A and every RP-th row; lanes of one column meet by
// shuffles, warps in shared memory.  A kv_len[q] outside [1, max_kv_len] is
// reported, nothing written.
constexpr int RA_NT = 512;   // threads of the row append
constexpr int RA_U = 16;     // vectors in flight per thread

template <typename T>
__global__ void __launch_bounds__(RA_NT) append_row_at_len_kernel(
    const T* __restrict__ x, const T* __restrict__ A, int64_t a_stride, T* __restrict__ lr,
    int64_t lr_seq, int64_t lr_agent, const int32_t* __restrict__ kv_len, int64_t max_kv_len,
    int64_t H, int C, int* err) {
  // the decode that follows is a programmatic dependent: its set-up may start
  // now (it reads nothing before waiting for this grid)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  constexpr int VE = 16 / (int)sizeof(T);   // elements of a 16-byte vector
  __shared__ float red[RA_NT / 32][128];
  const int q = blockIdx.x, l = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int64_t len = kv_len[q];
  if (len < 1 || len > max_kv_len) {
    if (tid == 0) atomicOr(err, 1);
    return;
  }
  const int VR = C / VE;            // vectors of an A row (divides 32)
  const int RP = RA_NT / VR;        // rows of one pass over the CTA
  const int cv = tid % VR;
  const T* xq = x + (int64_t)q * H;
  const uint4* Av = reinterpret_cast<const uint4*>(A + (int64_t)l * a_stride);
  float acc[VE];
#pragma unroll
  for (int e = 0; e < VE; ++e) acc[e] = 0.f;
  for (int64_t h0 = tid / VR; h0 < H; h0 += (int64_t)RP * RA_U) {
    uint4 av[RA_U];
    float xv[RA_U];
#pragma unroll
    for (int u = 0; u < RA_U; ++u) {
      const int64_t h = h0 + (int64_t)u * RP;
      av[u] = h < H ? __ldg(Av + h * VR + cv) : make_uint4(0, 0, 0, 0);
      xv[u] = h < H ? to_f32(xq[h]) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < RA_U; ++u) {
      const T* e8 = reinterpret_cast<const T*>(&av[u]);
#pragma unroll
      for (int e = 0; e < VE; ++e) acc[e] = fmaf(xv[u], to_f32(e8[e]), acc[e]);
    }
  }
  // lanes lane, lane ^ VR, ... hold the same column vector
  for (int o = VR; o < 32; o <<= 1)
#pragma unroll
    for (int e = 0; e < VE; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
  if (lane < VR)
#pragma unroll
    for (int e = 0; e < VE; ++e) red[w][cv * VE + e] = acc[e];
  __syncthreads();
  if (tid < C) {
    float v = 0.f;
#pragma unroll
    for (int ww = 0; ww < RA_NT / 32; ++ww) v += red[ww][tid];
    lr[(int64_t)l * lr_agent + (int64_t)q * lr_seq + (len - 1) * C + tid] = from_f32<T>(v);
  }
}

}  // namespace

cudaError_t launch_append_row_at_len(const void* x, const void* A, int64_t a_stride, void* lr,
                                     int64_t lr_seq, int64_t lr_agent, int n_lr,
                                     const int32_t* kv_len, int64_t max_kv_len, int n_seqs,
                                     int64_t H, int r, la_dtype dt, int* err, cudaStream_t st) {
  const int ve = dt == LA_F32 ? 4 : 8;
  if (2 * r > 128 || (2 * r) % ve != 0 || 32 % ((2 * r) / ve) != 0 || n_seqs < 1 || n_lr < 1)
    return cudaErrorInvalidValue;
  dim3 grid(n_seqs, n_lr);
  if (dt == LA_F32)
    append_row_at_len_kernel<float><<<grid, RA_NT, 0, st>>>(
        static_cast<const float*>(x), static_cast<const float*>(A), a_stride, static_cast<float*>(lr),
        lr_seq, lr_agent, kv_len, max_kv_len, H, 2 * r, err);
  else
    append_row_at_len_kernel<__nv_bfloat16><<<grid, RA_NT, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(A), a_stride,
        static_cast<__nv_bfloat16*>(lr), lr_seq, lr_agent, kv_len, max_kv_len, H, 2 * r, err);
  return cudaGetLastError();
}

cudaError_t launch_append_simt(const void* X, int64_t ldx, int64_t n, int64_t H, const void* A,
                               int r, void* lr, int64_t pos0, int n_seqs, int64_t sx,
                               int64_t slr, la_dtype dt, cudaStream_t st) {
  if (dt == LA_F32) return launch_r<float>(X, ldx, n, H, A, r, lr, pos0, n_seqs, sx, slr, st);
  return launch_r<__nv_bfloat16>(X, ldx, n, H, A, r, lr, pos0, n_seqs, sx, slr, st);
}

}  // namespace la
