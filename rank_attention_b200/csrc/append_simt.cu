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
#include "ptx.cuh"

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
// lr[l][q][kv_len[q] - 1] = x[q] A[l].  A cluster of 16 (else 8) CTAs per (q, l)
// splits the hidden rows (one SM alone cannot keep enough of A in flight);
// in a CTA a thread keeps one 16-byte column vector of A and every RP-th row,
// all loads of a pass issued before the first is used; lanes of one column
// meet by shuffles, warps in shared memory, the CTAs over distributed shared
// memory, where rank 0 writes the row.  A kv_len[q] outside [1, max_kv_len] is
// reported, nothing written.
constexpr int RA_NT = 256;   // threads of a row-append CTA
constexpr int RA_U = 8;      // vectors in flight per thread

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
  __shared__ float part[128];               // this CTA's sums, read by rank 0
  const int rank = blockIdx.x, ncl = gridDim.x, q = blockIdx.y, l = blockIdx.z;   // one cluster in x
  const int64_t len = kv_len[q];   // requested now, first used at the end
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int VR = C / VE;            // vectors of an A row (divides 32)
  const int RP = RA_NT / VR;        // rows of one pass over the CTA
  const int cv = tid % VR;
  const int64_t hb = rank * H / ncl, he = (rank + 1) * H / ncl;
  float acc[VE];
#pragma unroll
  for (int e = 0; e < VE; ++e) acc[e] = 0.f;
  {   // A's rows do not depend on the sequence's length: read before it arrives
    const T* xq = x + (int64_t)q * H;
    const uint4* Av = reinterpret_cast<const uint4*>(A + (int64_t)l * a_stride);
    for (int64_t h0 = hb + tid / VR; h0 < he; h0 += (int64_t)RP * RA_U) {
      uint4 av[RA_U];
      float xv[RA_U];
#pragma unroll
      for (int u = 0; u < RA_U; ++u) {
        const int64_t h = h0 + (int64_t)u * RP;
        av[u] = h < he ? __ldg(Av + h * VR + cv) : make_uint4(0, 0, 0, 0);
        xv[u] = h < he ? to_f32(xq[h]) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < RA_U; ++u) {
        const T* e8 = reinterpret_cast<const T*>(&av[u]);
#pragma unroll
        for (int e = 0; e < VE; ++e) acc[e] = fmaf(xv[u], to_f32(e8[e]), acc[e]);
      }
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
    part[tid] = v;
  }
  ptx::cluster_sync_all();   // every CTA's sums are in place
  const bool bad = len < 1 || len > max_kv_len;
  if (rank == 0 && tid < C && !bad) {
    // every CTA's sum requested before the first is added
    float pv[16];
    const uint32_t pa = ptx::smem_u32(part + tid);
#pragma unroll
    for (int k = 0; k < 16; ++k) pv[k] = k < ncl ? ptx::dsmem_ld(ptx::dsmem_addr(pa, k)) : 0.f;
    float v = 0.f;
#pragma unroll
    for (int k = 0; k < 16; ++k) v += pv[k];
    lr[(int64_t)l * lr_agent + (int64_t)q * lr_seq + (len - 1) * C + tid] = from_f32<T>(v);
  }
  if (rank == 0 && tid == 0 && bad) atomicOr(err, 1);
  ptx::cluster_sync_all();   // no CTA leaves while rank 0 reads its sums
}

}  // namespace

cudaError_t launch_append_row_at_len(const void* x, const void* A, int64_t a_stride, void* lr,
                                     int64_t lr_seq, int64_t lr_agent, int n_lr,
                                     const int32_t* kv_len, int64_t max_kv_len, int n_seqs,
                                     int64_t H, int r, la_dtype dt, int* err, cudaStream_t st) {
  const int ve = dt == LA_F32 ? 4 : 8;
  if (2 * r > 128 || (2 * r) % ve != 0 || 32 % ((2 * r) / ve) != 0 || n_seqs < 1 || n_lr < 1)
    return cudaErrorInvalidValue;
  // 16 CTAs a cluster (a non-portable size) where the device takes it, else 8;
  // decided once by an occupancy query, so that no launch is tried and refused
  // (a refused launch would break a stream capture)
  static int ncl_of[2] = {0, 0};
  int& ncl = ncl_of[dt == LA_F32 ? 0 : 1];
  const void* kfn = dt == LA_F32 ? reinterpret_cast<const void*>(append_row_at_len_kernel<float>)
                                 : reinterpret_cast<const void*>(append_row_at_len_kernel<__nv_bfloat16>);
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(RA_NT);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (ncl == 0) {
    int n = 0;
    cfg.gridDim = dim3(16, 1, 1);
    attr[0].val.clusterDim.x = 16;
    const bool ok16 = cudaFuncSetAttribute(kfn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess &&
                      cudaOccupancyMaxActiveClusters(&n, kfn, &cfg) == cudaSuccess && n >= 1;
    cudaGetLastError();
    ncl = ok16 ? 16 : 8;
  }
  cfg.gridDim = dim3((unsigned)ncl, (unsigned)n_seqs, (unsigned)n_lr);
  attr[0].val.clusterDim.x = (unsigned)ncl;
  cudaError_t e;
  if (dt == LA_F32)
    e = cudaLaunchKernelEx(&cfg, append_row_at_len_kernel<float>, static_cast<const float*>(x),
                           static_cast<const float*>(A), a_stride, static_cast<float*>(lr), lr_seq,
                           lr_agent, kv_len, max_kv_len, H, 2 * r, err);
  else
    e = cudaLaunchKernelEx(&cfg, append_row_at_len_kernel<__nv_bfloat16>,
                           static_cast<const __nv_bfloat16*>(x), static_cast<const __nv_bfloat16*>(A),
                           a_stride, static_cast<__nv_bfloat16*>(lr), lr_seq, lr_agent, kv_len,
                           max_kv_len, H, 2 * r, err);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_append_simt(const void* X, int64_t ldx, int64_t n, int64_t H, const void* A,
                               int r, void* lr, int64_t pos0, int n_seqs, int64_t sx,
                               int64_t slr, la_dtype dt, cudaStream_t st) {
  if (dt == LA_F32) return launch_r<float>(X, ldx, n, H, A, r, lr, pos0, n_seqs, sx, slr, st);
  return launch_r<__nv_bfloat16>(X, ldx, n, H, A, r, lr, pos0, n_seqs, sx, slr, st);
}

}  // namespace la
