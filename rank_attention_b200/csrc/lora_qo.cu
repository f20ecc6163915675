// LoRA on the query and output projections (the qkvo setting: LoRA on the
// query, key, value and output projections; LRAgent summary App. D.1
// "Ablation on LoRA Application"), around the attention, with the cache
// decomposition Y = X W_0 + (X A) B of App. A.3:
//
//   query side   q^a_t = RoPE_t( X^a_t W_q + s (X^a_t A_q) B_q^a )
//   output side  y^a   = O^a W_o + s (O^a A_o) B_o^a
//
// The base products X W_q and O W_o are the base model's; these kernels take
// them as inputs and add the rank-r parts.  Both are HBM-bound: every input
// element is read once and every output element written once, the r-wide
// rows X A_q and O A_o stay in shared memory, the up-projections B^a are read
// coalesced and reused from L1 / L2 across a CTA's tokens.
#include <cmath>

#include <cuda_bf16.h>

#include "bf16_common.cuh"
#include "la_internal.cuh"
#include "ptx.cuh"

namespace la {
namespace {

using ptx::pack_bf16;

template <typename IO>
__device__ __forceinline__ float ldf(const IO* p);
template <>
__device__ __forceinline__ float ldf<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ldf<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }
template <typename IO>
__device__ __forceinline__ IO stf(float x);
template <>
__device__ __forceinline__ float stf<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 stf<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

constexpr int kQThreads = 256;
constexpr int kQTok = 8;      // tokens per CTA: each B_q^a value is loaded once for them
constexpr int kQF = 4;        // adjacent frequencies per thread (one 8-byte bf16 access)

template <typename IO>
struct Vec4 {
  float v[4];
};
template <typename IO>
__device__ __forceinline__ Vec4<IO> ld4(const IO* p);
template <>
__device__ __forceinline__ Vec4<__nv_bfloat16> ld4<__nv_bfloat16>(const __nv_bfloat16* p) {
  Vec4<__nv_bfloat16> r;
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  r.v[0] = __uint_as_float(u.x << 16);
  r.v[1] = __uint_as_float(u.x & 0xffff0000u);
  r.v[2] = __uint_as_float(u.y << 16);
  r.v[3] = __uint_as_float(u.y & 0xffff0000u);
  return r;
}
template <>
__device__ __forceinline__ Vec4<float> ld4<float>(const float* p) {
  Vec4<float> r;
  const float4 a = *reinterpret_cast<const float4*>(p);
  r.v[0] = a.x; r.v[1] = a.y; r.v[2] = a.z; r.v[3] = a.w;
  return r;
}
__device__ __forceinline__ void st4(__nv_bfloat16* p, const float (&v)[4]) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]));
}
__device__ __forceinline__ void st4(float* p, const float (&v)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}

// One CTA per (8 tokens x a block of heads, agent, sequence); a thread owns
// 4 adjacent frequencies i of one head -- elements i and i + d/2, the RoPE
// pairs -- for all the CTA's tokens: it loads its slices of the r rows of
// B_q^a once, accumulates every token's delta, then adds the token's base
// projection and rotates (the delta joins before the rotation; every element
// is written once, so q_out may alias q_base).  (cos, sin) per (token,
// frequency) are formed once per CTA, angle reduced in fp64.
template <typename IO>
__global__ void __launch_bounds__(kQThreads) query_expand_kernel(
    const IO* __restrict__ q_base, const IO* __restrict__ lr_q, const IO* __restrict__ B_q,
    IO* q_out, int n_agents, int n_tok, int n_q, int d, int r, float s, RopeTheta rt,
    const int32_t* __restrict__ pos_end) {
  __shared__ float lr[kQTok][64];
  __shared__ float2 cs[kQTok][64];
  const int h2 = d / 2, ld = n_q * d;
  const int tph = h2 / kQF;                           // threads per head
  const int hpb = kQThreads / tph;                    // heads per CTA (16 at d = 128)
  const int hblocks = (n_q + hpb - 1) / hpb;
  const int tb = (blockIdx.x / hblocks) * kQTok, h0 = (blockIdx.x % hblocks) * hpb;
  const int agent = blockIdx.y, seq = blockIdx.z;
  const int nt = min(kQTok, n_tok - tb);
  const int64_t row0 = ((int64_t)seq * n_agents + agent) * n_tok + tb;
  const int64_t pos0 = (int64_t)pos_end[seq] - n_tok + tb;
  for (int u = threadIdx.x; u < nt * r; u += kQThreads)
    lr[u / r][u % r] = ldf(lr_q + (row0 + u / r) * r + u % r);
  for (int u = threadIdx.x; u < nt * h2; u += kQThreads)
    cs[u / h2][u % h2] = rope_cs_exact(pos0 + u / h2, rt.theta[u % h2]);
  __syncthreads();
  const int h = h0 + threadIdx.x / tph, i0 = (threadIdx.x % tph) * kQF;
  if (h >= n_q) return;
  const int c1 = h * d + i0, c2 = c1 + h2;
  const IO* B = B_q + (int64_t)agent * r * ld;
  float x1[kQTok][kQF], x2[kQTok][kQF];
#pragma unroll
  for (int tt = 0; tt < kQTok; ++tt)
#pragma unroll
    for (int j = 0; j < kQF; ++j) x1[tt][j] = x2[tt][j] = 0.f;
#pragma unroll 4
  for (int m = 0; m < r; ++m) {
    const Vec4<IO> b1 = ld4<IO>(B + (int64_t)m * ld + c1), b2 = ld4<IO>(B + (int64_t)m * ld + c2);
#pragma unroll
    for (int tt = 0; tt < kQTok; ++tt) {
      const float l = lr[tt][m];
#pragma unroll
      for (int j = 0; j < kQF; ++j) {
        x1[tt][j] = fmaf(l, b1.v[j], x1[tt][j]);
        x2[tt][j] = fmaf(l, b2.v[j], x2[tt][j]);
      }
    }
  }
#pragma unroll
  for (int tt = 0; tt < kQTok; ++tt) {
    if (tt < nt) {
      const IO* qb = q_base + (row0 + tt) * ld;
      IO* qo = q_out + (row0 + tt) * ld;
      const Vec4<IO> a1 = ld4<IO>(qb + c1), a2 = ld4<IO>(qb + c2);
      float o1[kQF], o2[kQF];
#pragma unroll
      for (int j = 0; j < kQF; ++j) {
        const float y1 = fmaf(s, x1[tt][j], a1.v[j]), y2 = fmaf(s, x2[tt][j], a2.v[j]);
        const float2 c = cs[tt][i0 + j];
        o1[j] = y1 * c.x - y2 * c.y;
        o2[j] = y2 * c.x + y1 * c.y;
      }
      st4(qo + c1, o1);
      st4(qo + c2, o2);
    }
  }
}

constexpr int kOThreads = 256;
constexpr int kOWarps = kOThreads / 32;
constexpr int kOTok = 4;      // tokens per CTA: A_o and B_o^a are read once for them
constexpr int kOCols = 8;     // output columns per thread (one 16-byte load of bf16)
constexpr int kOColBlock = kOThreads * kOCols;

template <typename IO>
struct Vec8 {
  float v[8];
};
template <typename IO>
__device__ __forceinline__ Vec8<IO> ld8(const IO* p);
template <>
__device__ __forceinline__ Vec8<__nv_bfloat16> ld8<__nv_bfloat16>(const __nv_bfloat16* p) {
  Vec8<__nv_bfloat16> r;
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    r.v[2 * j] = __uint_as_float(w[j] << 16);
    r.v[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
  }
  return r;
}
template <>
__device__ __forceinline__ Vec8<float> ld8<float>(const float* p) {
  Vec8<float> r;
  const float4 a = *reinterpret_cast<const float4*>(p), b = *reinterpret_cast<const float4*>(p + 4);
  r.v[0] = a.x; r.v[1] = a.y; r.v[2] = a.z; r.v[3] = a.w;
  r.v[4] = b.x; r.v[5] = b.y; r.v[6] = b.z; r.v[7] = b.w;
  return r;
}

// One CTA per (4 tokens x 2048 output columns, agent, sequence).  Shrink
// t = O A_o for the CTA's tokens (each column block recomputes it: O(D_in r)
// per token, small against the expand): thread j takes rows j, j + 256, ...
// of A_o, 16 columns at a time as two 16-byte vectors, multiplies them by
// the tokens' o values of the same rows, and the block sums the partials
// (warp shuffles, then shared memory).  Expand y += s t B_o^a: a thread owns
// 8 consecutive output columns, read as one 16-byte vector per row of B_o^a.
template <typename IO>
__global__ void __launch_bounds__(kOThreads) output_delta_kernel(
    const IO* __restrict__ o, const IO* __restrict__ A_o, int64_t a_agent_stride,
    const IO* __restrict__ B_o, IO* y, int n_agents, int n_tok, int d_in, int d_out, int r,
    float s) {
  __shared__ float part[kOWarps][kOTok][16];
  __shared__ float t[kOTok][64];
  const int cblocks = (d_out + kOColBlock - 1) / kOColBlock;
  const int tb = (blockIdx.x / cblocks) * kOTok, cb = blockIdx.x % cblocks;
  const int agent = blockIdx.y, seq = blockIdx.z;
  const int nt = min(kOTok, n_tok - tb);
  const int64_t row0 = ((int64_t)seq * n_agents + agent) * n_tok + tb;
  const IO* A = A_o + agent * a_agent_stride;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int m0 = 0; m0 < r; m0 += 16) {     // 16 columns of A_o per pass
    const int mw = min(16, r - m0);          // 8 at r = 8
    float acc[kOTok][16];
#pragma unroll
    for (int tt = 0; tt < kOTok; ++tt)
#pragma unroll
      for (int m = 0; m < 16; ++m) acc[tt][m] = 0.f;
#pragma unroll 4
    for (int k = threadIdx.x; k < d_in; k += kOThreads) {
      const Vec8<IO> a0 = ld8<IO>(A + (int64_t)k * r + m0);
      Vec8<IO> a1;
      if (mw > 8) a1 = ld8<IO>(A + (int64_t)k * r + m0 + 8);
      else
#pragma unroll
        for (int j = 0; j < 8; ++j) a1.v[j] = 0.f;
#pragma unroll
      for (int tt = 0; tt < kOTok; ++tt) {
        const float x = tt < nt ? ldf(o + (row0 + tt) * d_in + k) : 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          acc[tt][j] = fmaf(x, a0.v[j], acc[tt][j]);
          acc[tt][8 + j] = fmaf(x, a1.v[j], acc[tt][8 + j]);
        }
      }
    }
#pragma unroll
    for (int tt = 0; tt < kOTok; ++tt) {
      if (tt >= nt) break;   // the block's last tokens (one in a decode step)
#pragma unroll
      for (int m = 0; m < 16; ++m) {
        float v = acc[tt][m];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (lane == 0) part[w][tt][m] = v;
      }
    }
    __syncthreads();
    if (threadIdx.x < kOTok * 16) {
      const int tt = threadIdx.x / 16, m = threadIdx.x % 16;
      float v = 0.f;
#pragma unroll
      for (int ww = 0; ww < kOWarps; ++ww) v += part[ww][tt][m];
      if (m < mw) t[tt][m0 + m] = v;
    }
    __syncthreads();
  }
  const int c0 = cb * kOColBlock + threadIdx.x * kOCols;
  if (c0 >= d_out) return;
  const IO* B = B_o + (int64_t)agent * r * d_out + c0;
  float z[kOTok][kOCols];
#pragma unroll
  for (int tt = 0; tt < kOTok; ++tt)
#pragma unroll
    for (int j = 0; j < kOCols; ++j) z[tt][j] = 0.f;
#pragma unroll 4
  for (int m = 0; m < r; ++m) {
    const Vec8<IO> b = ld8<IO>(B + (int64_t)m * d_out);
#pragma unroll
    for (int tt = 0; tt < kOTok; ++tt)
#pragma unroll
      for (int j = 0; j < kOCols; ++j) z[tt][j] = fmaf(t[tt][m], b.v[j], z[tt][j]);
  }
#pragma unroll
  for (int tt = 0; tt < kOTok; ++tt) {
    if (tt < nt) {
      IO* yp = y + (row0 + tt) * d_out + c0;
      const Vec8<IO> y0 = ld8<IO>(yp);
      float o[kOCols];
#pragma unroll
      for (int j = 0; j < kOCols; ++j) o[j] = fmaf(s, z[tt][j], y0.v[j]);
      st4(yp, *reinterpret_cast<const float(*)[4]>(o));
      st4(yp + 4, *reinterpret_cast<const float(*)[4]>(o + 4));
    }
  }
}

// bf16 query side, 16 tokens a CTA: a thread owns 8 adjacent frequencies of
// one head (16-byte vectors at columns i and i + d/2, the RoPE pairs) and
// forms their deltas for 4 tokens at a time from one 16-byte read of each
// B_q^a row; the base projections are read and the rotated queries written in
// 16-byte vectors.  (cos, sin) of the CTA's positions are formed once (angle
// reduced in fp64) in shared memory, with the tokens' LR rows.
constexpr int kQ2Threads = 256;
constexpr int kQ2Tok = 16;

template <int R>
__global__ void __launch_bounds__(kQ2Threads, 2) query_expand_v_kernel(
    const __nv_bfloat16* __restrict__ q_base, const __nv_bfloat16* __restrict__ lr_q,
    const __nv_bfloat16* __restrict__ B_q, __nv_bfloat16* q_out, int n_agents, int n_tok, int n_q,
    int d, float s, RopeTheta rt, const int32_t* __restrict__ pos_end) {
  __shared__ float lr[kQ2Tok][R];
  __shared__ float2 cs[kQ2Tok][64];
  const int h2 = d / 2, ld = n_q * d;
  const int tb = blockIdx.x * kQ2Tok, agent = blockIdx.y, seq = blockIdx.z;
  const int nt = min(kQ2Tok, n_tok - tb);
  const int64_t row0 = ((int64_t)seq * n_agents + agent) * n_tok + tb;
  const int64_t pos0 = (int64_t)pos_end[seq] - n_tok + tb;
  for (int u = threadIdx.x; u < nt * R; u += kQ2Threads)
    lr[u / R][u % R] = __bfloat162float(lr_q[(row0 + u / R) * R + u % R]);
  for (int u = threadIdx.x; u < nt * h2; u += kQ2Threads)
    cs[u / h2][u % h2] = rope_cs_exact(pos0 + u / h2, rt.theta[u % h2]);
  __syncthreads();
  const __nv_bfloat16* B = B_q + (int64_t)agent * R * ld;
  const int cph = h2 / 8;                       // 8-frequency chunks of a head
  for (int item = threadIdx.x; item < n_q * cph; item += kQ2Threads) {
    const int h = item / cph, i0 = (item % cph) * 8;
    const int c1 = h * d + i0, c2 = c1 + h2;
#pragma unroll 1
    for (int g0 = 0; g0 < nt; g0 += 4) {
      // the group's base projections requested before the deltas are formed
      uint4 qa[4][2];
#pragma unroll
      for (int tt = 0; tt < 4; ++tt) {
        const __nv_bfloat16* qb = q_base + (row0 + g0 + tt) * ld;
        qa[tt][0] = g0 + tt < nt ? *reinterpret_cast<const uint4*>(qb + c1) : make_uint4(0, 0, 0, 0);
        qa[tt][1] = g0 + tt < nt ? *reinterpret_cast<const uint4*>(qb + c2) : make_uint4(0, 0, 0, 0);
      }
      float x1[4][8], x2[4][8];
#pragma unroll
      for (int tt = 0; tt < 4; ++tt)
#pragma unroll
        for (int j = 0; j < 8; ++j) x1[tt][j] = x2[tt][j] = 0.f;
#pragma unroll 2
      for (int m = 0; m < R; ++m) {
        const Vec8<__nv_bfloat16> b1 = ld8<__nv_bfloat16>(B + (int64_t)m * ld + c1);
        const Vec8<__nv_bfloat16> b2 = ld8<__nv_bfloat16>(B + (int64_t)m * ld + c2);
#pragma unroll
        for (int tt = 0; tt < 4; ++tt) {
          const float l = lr[(g0 + tt) & (kQ2Tok - 1)][m];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            x1[tt][j] = fmaf(l, b1.v[j], x1[tt][j]);
            x2[tt][j] = fmaf(l, b2.v[j], x2[tt][j]);
          }
        }
      }
#pragma unroll
      for (int tt = 0; tt < 4; ++tt) {
        const int tok = g0 + tt;
        if (tok < nt) {
          const Vec8<__nv_bfloat16> a1 = ld8<__nv_bfloat16>(reinterpret_cast<const __nv_bfloat16*>(&qa[tt][0]));
          const Vec8<__nv_bfloat16> a2 = ld8<__nv_bfloat16>(reinterpret_cast<const __nv_bfloat16*>(&qa[tt][1]));
          uint32_t o1[4], o2[4];
#pragma unroll
          for (int j = 0; j < 8; j += 2) {
            const float2 ca = cs[tok][i0 + j], cb = cs[tok][i0 + j + 1];
            const float y1a = fmaf(s, x1[tt][j], a1.v[j]), y2a = fmaf(s, x2[tt][j], a2.v[j]);
            const float y1b = fmaf(s, x1[tt][j + 1], a1.v[j + 1]), y2b = fmaf(s, x2[tt][j + 1], a2.v[j + 1]);
            o1[j / 2] = pack_bf16(y1a * ca.x - y2a * ca.y, y1b * cb.x - y2b * cb.y);
            o2[j / 2] = pack_bf16(y2a * ca.x + y1a * ca.y, y2b * cb.x + y1b * cb.y);
          }
          __nv_bfloat16* qo = q_out + (row0 + tok) * ld;
          *reinterpret_cast<uint4*>(qo + c1) = make_uint4(o1[0], o1[1], o1[2], o1[3]);
          *reinterpret_cast<uint4*>(qo + c2) = make_uint4(o2[0], o2[1], o2[2], o2[3]);
        }
      }
    }
  }
}

// bf16 query side on the tensor cores (r >= 16): one CTA per (16 tokens,
// agent, sequence).  The deltas D = lr_q B_q^a (16 tokens x 8 columns a tile)
// are warp MMAs (m16n8k16, fp32 accumulation; bf16 x bf16 products are exact
// in fp32, as on the CUDA cores): the A operand is the tokens' LR rows, the B
// operand B_q^a's 8 x 8 blocks read as rows and transposed in registers
// (movmatrix), so that B_q^a is read once per 16 tokens.  A warp takes the
// column tiles c and c + d/2 of a head together, so each thread holds both
// elements of its RoPE pairs, adds them to the base projection and rotates.
template <int R>
__global__ void __launch_bounds__(kQ2Threads) query_expand_tc_kernel(
    const __nv_bfloat16* q_base, const __nv_bfloat16* __restrict__ lr_q,
    const __nv_bfloat16* __restrict__ B_q, __nv_bfloat16* q_out, int n_agents, int n_tok, int n_q,
    int d, float s, RopeTheta rt, const int32_t* __restrict__ pos_end) {
  constexpr int KS = R / 16;                   // k-steps of the MMA
  __shared__ __align__(16) uint32_t lrs[kQ2Tok][R / 2 + 4];   // bf16 pairs, padded rows
  __shared__ float2 cs[kQ2Tok][64];
  const int h2 = d / 2, ld = n_q * d;
  const int tb = blockIdx.x * kQ2Tok, agent = blockIdx.y, seq = blockIdx.z;
  const int nt = min(kQ2Tok, n_tok - tb);
  const int64_t row0 = ((int64_t)seq * n_agents + agent) * n_tok + tb;
  const int64_t pos0 = (int64_t)pos_end[seq] - n_tok + tb;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, gq = lane >> 2, t4 = lane & 3;
  for (int u = tid; u < kQ2Tok * (R / 2); u += kQ2Threads) {
    const int tt = u / (R / 2), c = u % (R / 2);
    lrs[tt][c] = tt < nt ? *reinterpret_cast<const uint32_t*>(lr_q + (row0 + tt) * R + 2 * c) : 0u;
  }
  for (int u = tid; u < nt * h2; u += kQ2Threads)
    cs[u / h2][u % h2] = rope_cs_exact(pos0 + u / h2, rt.theta[u % h2]);
  __syncthreads();
  // A fragments (tokens x r), the same for every column tile
  uint32_t a[KS][4];
#pragma unroll
  for (int k = 0; k < KS; ++k) {
    a[k][0] = lrs[gq][8 * k + t4];
    a[k][1] = lrs[gq + 8][8 * k + t4];
    a[k][2] = lrs[gq][8 * k + 4 + t4];
    a[k][3] = lrs[gq + 8][8 * k + 4 + t4];
  }
  const __nv_bfloat16* B = B_q + (int64_t)agent * R * ld;
  const bool v0 = gq < nt, v1 = gq + 8 < nt;
  const int tph = h2 / 8;                       // column-tile pairs of a head
  for (int pr = w; pr < n_q * tph; pr += kQ2Threads / 32) {
    const int h = pr / tph, c = 8 * (pr % tph) + 2 * t4;   // this thread's columns c, c + 1 (and + d/2)
    const int64_t col1 = (int64_t)h * d + c, col2 = col1 + h2;
    // the base projections, requested before the MMAs
    const uint32_t* qb0 = reinterpret_cast<const uint32_t*>(q_base + (row0 + gq) * ld);
    const uint32_t* qb1 = reinterpret_cast<const uint32_t*>(q_base + (row0 + gq + 8) * ld);
    const uint32_t b00 = v0 ? qb0[col1 >> 1] : 0u, b01 = v0 ? qb0[col2 >> 1] : 0u;
    const uint32_t b10 = v1 ? qb1[col1 >> 1] : 0u, b11 = v1 ? qb1[col2 >> 1] : 0u;
    float d1[4] = {0.f, 0.f, 0.f, 0.f}, d2[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k = 0; k < KS; ++k) {
      const __nv_bfloat16* Bk = B + (int64_t)(16 * k + gq) * ld + (int64_t)h * d + 8 * (pr % tph) + 2 * t4;
      const uint32_t m10 = __ldg(reinterpret_cast<const uint32_t*>(Bk));
      const uint32_t m11 = __ldg(reinterpret_cast<const uint32_t*>(Bk + 8 * (int64_t)ld));
      const uint32_t m20 = __ldg(reinterpret_cast<const uint32_t*>(Bk + h2));
      const uint32_t m21 = __ldg(reinterpret_cast<const uint32_t*>(Bk + 8 * (int64_t)ld + h2));
      ptx::mma16816(d1, a[k], ptx::movmatrix_t(m10), ptx::movmatrix_t(m11));
      ptx::mma16816(d2, a[k], ptx::movmatrix_t(m20), ptx::movmatrix_t(m21));
    }
    // rows gq (d[0], d[1]) and gq + 8 (d[2], d[3]); columns c, c + 1
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int tok = gq + 8 * hr;
      if (tok >= nt) continue;
      const uint32_t u1 = hr ? b10 : b00, u2 = hr ? b11 : b01;
      const float2 ca = cs[tok][c], cb = cs[tok][c + 1];
      const float y1a = fmaf(s, d1[2 * hr], __uint_as_float(u1 << 16));
      const float y1b = fmaf(s, d1[2 * hr + 1], __uint_as_float(u1 & 0xffff0000u));
      const float y2a = fmaf(s, d2[2 * hr], __uint_as_float(u2 << 16));
      const float y2b = fmaf(s, d2[2 * hr + 1], __uint_as_float(u2 & 0xffff0000u));
      uint32_t* qo = reinterpret_cast<uint32_t*>(q_out + (row0 + tok) * ld);
      qo[col1 >> 1] = pack_bf16(y1a * ca.x - y2a * ca.y, y1b * cb.x - y2b * cb.y);
      qo[col2 >> 1] = pack_bf16(y2a * ca.x + y1a * ca.y, y2b * cb.x + y1b * cb.y);
    }
  }
}

// bf16 output side on the tensor cores: one CTA per (16 tokens, agent,
// sequence).  The shrink t = O A_o (16 tokens x r) runs as warp MMAs
// (m16n8k16, fp32 accumulation): warp w takes every 8th 16-wide slice of d_in,
// its A operand is the tokens' o rows read straight from memory, its B operand
// A_o's 8 x 8 blocks read as rows and transposed in registers (movmatrix); the
// warps' partial sums meet in shared memory.  The expand y += s t B_o^a stays
// on the CUDA cores in fp32: a thread owns 8 consecutive output columns, reads
// each row of B_o^a once as a 16-byte vector for 8 tokens, and updates y in
// 16-byte vectors.  A_o and B_o^a are read once per 16 tokens.
constexpr int kO2Threads = 256;
constexpr int kO2Tok = 16;

template <int R>
__global__ void __launch_bounds__(kO2Threads, 2) output_delta_tc_kernel(
    const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ A_o, int64_t a_agent_stride,
    const __nv_bfloat16* __restrict__ B_o, __nv_bfloat16* y, int n_agents, int n_tok, int d_in,
    int d_out, float s) {
  constexpr int NTN = R / 8;   // 8-column tiles of t
  __shared__ float part[kO2Threads / 32][kO2Tok][R + 1];
  __shared__ float t[kO2Tok][R];
  const int tb = blockIdx.x * kO2Tok, agent = blockIdx.y, seq = blockIdx.z;
  const int nt = min(kO2Tok, n_tok - tb);
  const int64_t row0 = ((int64_t)seq * n_agents + agent) * n_tok + tb;
  const __nv_bfloat16* A = A_o + agent * a_agent_stride;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5, gq = lane >> 2, t4 = lane & 3;

  // ---- shrink: t = O A_o on the tensor cores
  float D[NTN][4];
#pragma unroll
  for (int n = 0; n < NTN; ++n) D[n][0] = D[n][1] = D[n][2] = D[n][3] = 0.f;
  const uint32_t* olo = reinterpret_cast<const uint32_t*>(o + (row0 + gq) * d_in);
  const uint32_t* ohi = reinterpret_cast<const uint32_t*>(o + (row0 + gq + 8) * d_in);
  const bool vlo = gq < nt, vhi = gq + 8 < nt;
  for (int k0 = 16 * w; k0 < d_in; k0 += 16 * (kO2Threads / 32)) {
    uint32_t a[4];
    a[0] = vlo ? __ldg(olo + (k0 >> 1) + t4) : 0u;
    a[1] = vhi ? __ldg(ohi + (k0 >> 1) + t4) : 0u;
    a[2] = vlo ? __ldg(olo + (k0 >> 1) + 4 + t4) : 0u;
    a[3] = vhi ? __ldg(ohi + (k0 >> 1) + 4 + t4) : 0u;
#pragma unroll
    for (int n = 0; n < NTN; ++n) {
      const uint32_t m0 = __ldg(reinterpret_cast<const uint32_t*>(A + (int64_t)(k0 + gq) * R + 8 * n + 2 * t4));
      const uint32_t m1 = __ldg(reinterpret_cast<const uint32_t*>(A + (int64_t)(k0 + 8 + gq) * R + 8 * n + 2 * t4));
      ptx::mma16816(D[n], a, ptx::movmatrix_t(m0), ptx::movmatrix_t(m1));
    }
  }
#pragma unroll
  for (int n = 0; n < NTN; ++n) {
    part[w][gq][8 * n + 2 * t4] = D[n][0];
    part[w][gq][8 * n + 2 * t4 + 1] = D[n][1];
    if (gq + 8 < kO2Tok) {   // the MMA's rows 8 .. 15 exist only with 16 tokens a CTA
      part[w][gq + 8][8 * n + 2 * t4] = D[n][2];
      part[w][gq + 8][8 * n + 2 * t4 + 1] = D[n][3];
    }
  }
  __syncthreads();
  for (int i = tid; i < kO2Tok * R; i += kO2Threads) {
    const int tt = i / R, m = i % R;
    float v = 0.f;
#pragma unroll
    for (int ww = 0; ww < kO2Threads / 32; ++ww) v += part[ww][tt][m];
    t[tt][m] = v;
  }
  __syncthreads();

  // ---- expand: y += s t B_o^a, 8 columns a thread, 8 tokens at a time
  const __nv_bfloat16* B = B_o + (int64_t)agent * R * d_out;
  for (int c = tid * 8; c < d_out; c += kO2Threads * 8) {
#pragma unroll 1
    for (int h = 0; h < kO2Tok / 8; ++h) {
      if (8 * h >= nt) break;
      float z[8][8];
#pragma unroll
      for (int tt = 0; tt < 8; ++tt)
#pragma unroll
        for (int j = 0; j < 8; ++j) z[tt][j] = 0.f;
#pragma unroll 2
      for (int m = 0; m < R; ++m) {
        const Vec8<__nv_bfloat16> b = ld8<__nv_bfloat16>(B + (int64_t)m * d_out + c);
#pragma unroll
        for (int tt = 0; tt < 8; ++tt) {
          const float tv = t[8 * h + tt][m];
#pragma unroll
          for (int j = 0; j < 8; ++j) z[tt][j] = fmaf(tv, b.v[j], z[tt][j]);
        }
      }
#pragma unroll
      for (int tt = 0; tt < 8; ++tt) {
        if (8 * h + tt < nt) {
          const uint4 yv = *reinterpret_cast<const uint4*>(y + (row0 + 8 * h + tt) * d_out + c);
          const uint32_t yw[4] = {yv.x, yv.y, yv.z, yv.w};
          uint32_t ow[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float y0 = __uint_as_float(yw[j] << 16), y1 = __uint_as_float(yw[j] & 0xffff0000u);
            ow[j] = pack_bf16(fmaf(s, z[tt][2 * j], y0), fmaf(s, z[tt][2 * j + 1], y1));
          }
          *reinterpret_cast<uint4*>(y + (row0 + 8 * h + tt) * d_out + c) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
        }
      }
    }
  }
}

}  // namespace

cudaError_t launch_query_expand(const void* q_base, const void* lr_q, const void* B_q, void* q_out,
                                int n_seqs, int n_agents, int n_tok, int n_q, int d, int r, float s,
                                double rope_base, const int32_t* pos_end, la_dtype dt,
                                cudaStream_t st) {
  RopeTheta rt;
  for (int i = 0; i < 64; ++i) {
    rt.theta[i] = i < d / 2 ? std::pow(rope_base, -2.0 * i / d) : 0.0;
    rt.thetaf[i] = (float)rt.theta[i];
  }
  // bf16 with 16-byte aligned rows: 16 tokens a CTA, 16-byte vectors
  if (dt == LA_BF16 && ((int64_t)n_q * d) % 8 == 0 && (reinterpret_cast<uintptr_t>(q_base) & 15) == 0 &&
      (reinterpret_cast<uintptr_t>(q_out) & 15) == 0 && (reinterpret_cast<uintptr_t>(B_q) & 15) == 0) {
    const dim3 g2((unsigned)((n_tok + kQ2Tok - 1) / kQ2Tok), (unsigned)n_agents, (unsigned)n_seqs);
    auto qb = static_cast<const __nv_bfloat16*>(q_base);
    auto lq = static_cast<const __nv_bfloat16*>(lr_q);
    auto bq = static_cast<const __nv_bfloat16*>(B_q);
    auto qo = static_cast<__nv_bfloat16*>(q_out);
    switch (r) {   // r = 8: the CUDA-core kernel (the MMA's k is 16)
      case 8: query_expand_v_kernel<8><<<g2, kQ2Threads, 0, st>>>(qb, lq, bq, qo, n_agents, n_tok, n_q, d, s, rt, pos_end); break;
      case 16: query_expand_tc_kernel<16><<<g2, kQ2Threads, 0, st>>>(qb, lq, bq, qo, n_agents, n_tok, n_q, d, s, rt, pos_end); break;
      case 32: query_expand_tc_kernel<32><<<g2, kQ2Threads, 0, st>>>(qb, lq, bq, qo, n_agents, n_tok, n_q, d, s, rt, pos_end); break;
      default: query_expand_tc_kernel<64><<<g2, kQ2Threads, 0, st>>>(qb, lq, bq, qo, n_agents, n_tok, n_q, d, s, rt, pos_end); break;
    }
    return cudaGetLastError();
  }
  const int hpb = kQThreads / (d / 2 / kQF);
  const int hblocks = (n_q + hpb - 1) / hpb;
  const dim3 grid((unsigned)(((int64_t)n_tok + kQTok - 1) / kQTok * hblocks), (unsigned)n_agents,
                  (unsigned)n_seqs);
  if (dt == LA_BF16)
    query_expand_kernel<__nv_bfloat16><<<grid, kQThreads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(q_base), static_cast<const __nv_bfloat16*>(lr_q),
        static_cast<const __nv_bfloat16*>(B_q), static_cast<__nv_bfloat16*>(q_out), n_agents, n_tok,
        n_q, d, r, s, rt, pos_end);
  else
    query_expand_kernel<float><<<grid, kQThreads, 0, st>>>(
        static_cast<const float*>(q_base), static_cast<const float*>(lr_q),
        static_cast<const float*>(B_q), static_cast<float*>(q_out), n_agents, n_tok, n_q, d, r, s, rt,
        pos_end);
  return cudaGetLastError();
}

cudaError_t launch_output_delta(const void* o, const void* A_o, int64_t a_agent_stride,
                                const void* B_o, void* y, int n_seqs, int n_agents, int n_tok,
                                int d_in, int d_out, int r, float s, la_dtype dt, cudaStream_t st) {
  // bf16 with d_in a multiple of 16 (the MMA's k) and 16-byte aligned rows: the
  // tensor-core shrink
  const bool tc = dt == LA_BF16 && d_in % 16 == 0 && d_out % 8 == 0 &&
                  (reinterpret_cast<uintptr_t>(o) & 15) == 0 && (reinterpret_cast<uintptr_t>(y) & 15) == 0 &&
                  (reinterpret_cast<uintptr_t>(B_o) & 15) == 0 && (reinterpret_cast<uintptr_t>(A_o) & 3) == 0 &&
                  (a_agent_stride & 1) == 0;
  if (tc) {
    const dim3 g2((unsigned)((n_tok + kO2Tok - 1) / kO2Tok), (unsigned)n_agents, (unsigned)n_seqs);
    auto o2 = static_cast<const __nv_bfloat16*>(o);
    auto a2 = static_cast<const __nv_bfloat16*>(A_o);
    auto b2 = static_cast<const __nv_bfloat16*>(B_o);
    auto y2 = static_cast<__nv_bfloat16*>(y);
    switch (r) {
      case 8: output_delta_tc_kernel<8><<<g2, kO2Threads, 0, st>>>(o2, a2, a_agent_stride, b2, y2, n_agents, n_tok, d_in, d_out, s); break;
      case 16: output_delta_tc_kernel<16><<<g2, kO2Threads, 0, st>>>(o2, a2, a_agent_stride, b2, y2, n_agents, n_tok, d_in, d_out, s); break;
      case 32: output_delta_tc_kernel<32><<<g2, kO2Threads, 0, st>>>(o2, a2, a_agent_stride, b2, y2, n_agents, n_tok, d_in, d_out, s); break;
      default: output_delta_tc_kernel<64><<<g2, kO2Threads, 0, st>>>(o2, a2, a_agent_stride, b2, y2, n_agents, n_tok, d_in, d_out, s); break;
    }
    return cudaGetLastError();
  }
  const int cblocks = (d_out + kOColBlock - 1) / kOColBlock;
  const dim3 grid((unsigned)((int64_t)(n_tok + kOTok - 1) / kOTok * cblocks), (unsigned)n_agents,
                  (unsigned)n_seqs);
  if (dt == LA_BF16)
    output_delta_kernel<__nv_bfloat16><<<grid, kOThreads, 0, st>>>(
        static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(A_o), a_agent_stride,
        static_cast<const __nv_bfloat16*>(B_o), static_cast<__nv_bfloat16*>(y), n_agents, n_tok,
        d_in, d_out, r, s);
  else
    output_delta_kernel<float><<<grid, kOThreads, 0, st>>>(
        static_cast<const float*>(o), static_cast<const float*>(A_o), a_agent_stride,
        static_cast<const float*>(B_o), static_cast<float*>(y), n_agents, n_tok, d_in, d_out, r, s);
  return cudaGetLastError();
}

}  // namespace la
