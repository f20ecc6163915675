// Flash-LoRA-Attention decode on the tensor cores (bf16 storage, fp32 accumulate).
//
// One CTA = one (sequence, KV head, split of the keys); the splits of a
// (sequence, KV head) form one thread-block cluster.  A CTA's rows are every
// agent x every query head of the GQA group, so each base and LR tile is read
// from HBM once for all agents (LRAgent summary §3 BaseLRShared: one base and
// one LR cache shared by the whole system).  128-key tiles of K_base, V_base
// and the LR rows are staged in shared memory by TMA (128/64/32-byte swizzle,
// no multicast) through a two-stage full/empty mbarrier pipeline.
//
// Warp roles (320 threads):
//  * 8 score warps, 16 keys each.  Key side (LRAgent summary App. D.1: RoPE
//    blocks the reordering, so the delta is rebuilt in head dimension).  A key
//    at position t = k0 + j of a tile starting at k0 is rotated by
//    R(t) = R(k0) R(j), so
//      q . K^a_t = q . K_base,t + (s R(-k0) q) . R(j) (LRk_t B_k^a):
//    the base scores are one MMA over all agents' rows, the delta dK = LRk B_k^a
//    is an MMA per agent (M = 16 keys, N = d, K = r) turned in registers by
//    R(j) -- whose cos / sin are per-thread constants, j being fixed per
//    thread -- and scored against the tile's rotated queries Q' = s R(-k0) Q.
//    Two agents are interleaved for ILP.  The tile's row maxima meet in
//    shared memory; the warps write P^T (bf16) and the rescale factors.
//  * 2 value warps own O_base^T (half of d each) and O_lr^T: value side
//    reordered (LRAgent explainer, Metodologia 3; summary App. B),
//    O_base^T += V_base^T P^T and O_lr^T += LRv^T P^T, so the LoRA value path
//    stays r wide inside the loop.  They also rotate the queries for the next
//    tile and refill the pipeline.
// Epilogue: each CTA applies B_v^a once per row to its partial,
// Z = O_base + s O_lr B_v^a (linear, so it commutes with the merge).  With one
// split the CTA writes out = Z / l; otherwise it writes (Z, m, l) to the
// workspace and a small merge kernel, chained by programmatic dependent launch,
// forms out = sum_k w_k Z_k / sum_k w_k l_k with w_k = 2^(m_k - max m).
#include <cudaTypedefs.h>

#include <cmath>

#include "la_internal.cuh"
#include "ptx.cuh"

namespace la {
namespace {

using namespace ptx;

constexpr int ST = 2;               // pipeline stages
constexpr int KT = 128;             // keys per tile
constexpr int NES = 8;              // score warps (16 keys each)
constexpr int NPV = 2;              // value warps
constexpr int NTHR = 32 * (NES + NPV);
constexpr int kMaxSplits = 32;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int kSMs = 148;
// named barriers (0 is __syncthreads)
constexpr int BAR_MAX = 1, BAR_P = 2, BAR_PFREE = 4, BAR_QP = 6, BAR_END = 8;

constexpr int align1k(int x) { return (x + 1023) / 1024 * 1024; }

// RoPE frequencies theta_i = base^(-2i/d), formed in fp64 on the host
struct RopeTheta {
  double theta[64];
};
constexpr int imax(int a, int b) { return a > b ? a : b; }

template <int D, int R, int NT>
struct Cfg {
  static constexpr int ROWS = NT * 8;                   // padded query rows
  static constexpr int W = D + R + 4;                   // Z | O_lr | m | l | pad (16-byte rows)
  static constexpr int KV_TILE = KT * D * 2;            // bytes of a K or V tile
  static constexpr int LR_TILE = align1k(KT * 2 * R * 2);
  static constexpr int STAGE = 2 * KV_TILE + LR_TILE;
  static constexpr int AREA = imax(ST * STAGE, align1k(ROWS * W * 4));
  static constexpr int P_TILE = align1k(ROWS * KT * 2);
  static constexpr int SMALL = 2 * NES * ROWS * 4 + 2 * ROWS * 4 + NES * ROWS * 4 + 64 * 8;
  static constexpr int Q_BYTES = align1k(ROWS * D * 2);   // Q, and each of the two Q' buffers
  static constexpr int BK_BYTES = R * D * 2;            // one agent's B_k (or B_v) slice
  static constexpr int KS = R >= 16 ? R / 16 : 1;        // k-steps of the expansion
  static constexpr int MR = R >= 16 ? R / 16 : 1;        // m-tiles of O_lr^T
  static constexpr int NG = D / 32;                      // column groups
  static constexpr int MT = D / 2 / 16;                  // m-tiles of O^T per value warp
  static size_t smem(int n_agents) {
    return 1024 + AREA + 2 * P_TILE + align1k(SMALL) + 3 * Q_BYTES +
           (size_t)align1k(BK_BYTES) * n_agents + (size_t)BK_BYTES * n_agents + 64;
  }
};

// (cos, sin) of t * theta, the angle formed and reduced modulo 2 pi in fp64
__device__ __forceinline__ float2 rope_cs_exact(int64_t t, double theta) {
  const double two_pi = 6.283185307179586476925286766559;
  const double ang = (double)t * theta;
  const float red = (float)fma(-two_pi, rint(ang * 0.15915494309189533577), ang);
  float s, c;
  sincosf(red, &s, &c);
  return make_float2(c, s);
}

// (cos, sin) of a small angle (|ang| < ~200 rad): Cody-Waite reduction with a
// two-constant split of 2 pi, then the SFU (about 2^-21 absolute on [-pi, pi])
__device__ __forceinline__ float2 sincos_small(float ang) {
  const float k = rintf(ang * 0.15915494309189535f);
  float red = fmaf(-k, 6.28318548202514648f, ang);
  red = fmaf(-k, -1.7484556000744083e-07f, red);
  float s, c;
  __sincosf(red, &s, &c);
  return make_float2(c, s);
}

// Q'[row] = s R(-t) Q[row] for every row, frequencies i = lane .. of this warp
// (nw_off: first frequency handled by the calling warp, step 32 per warp)
template <int D, int ROWS>
__device__ __forceinline__ void rotate_queries(uint32_t qs_u, uint32_t qp_u, const double* theta,
                                               int64_t t, float s, int i) {
  const float2 cs = rope_cs_exact(t, theta[i]);
  const float c = cs.x * s, sn = cs.y * s;
#pragma unroll 4
  for (int row = 0; row < ROWS; ++row) {
    uint16_t a, b;
    const uint32_t oa = tile_off<D, ROWS>(row, i), ob = tile_off<D, ROWS>(row, i + D / 2);
    asm volatile("ld.shared.b16 %0, [%1];" : "=h"(a) : "r"(qs_u + oa));
    asm volatile("ld.shared.b16 %0, [%1];" : "=h"(b) : "r"(qs_u + ob));
    const float x1 = __uint_as_float((uint32_t)a << 16), x2 = __uint_as_float((uint32_t)b << 16);
    const __nv_bfloat16 y1 = __float2bfloat16_rn(fmaf(x1, c, x2 * sn));
    const __nv_bfloat16 y2 = __float2bfloat16_rn(fmaf(x2, c, -x1 * sn));
    sts16(qp_u + oa, *reinterpret_cast<const uint16_t*>(&y1));
    sts16(qp_u + ob, *reinterpret_cast<const uint16_t*>(&y2));
  }
}

template <int D, int R, int NT>
__global__ void __launch_bounds__(NTHR, 1)
    decode_bf16_kernel(const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV,
                       const __grid_constant__ CUtensorMap tmL, const AttnParams p,
                       const __grid_constant__ RopeTheta rt) {
  using C = Cfg<D, R, NT>;
  constexpr int W = C::W, ROWS = C::ROWS;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* area = smem;
  unsigned char* ptile = area + C::AREA;                        // [2][ROWS][KT] bf16
  float* Mx = reinterpret_cast<float*>(ptile + 2 * C::P_TILE);  // [2][NES][ROWS]
  float* Corr = Mx + 2 * NES * ROWS;                             // [2][ROWS]
  float* Lw = Corr + 2 * ROWS;                                   // [NES][ROWS]
  double* theta = reinterpret_cast<double*>(Lw + NES * ROWS);    // [64]
  unsigned char* qs = ptile + 2 * C::P_TILE + align1k(C::SMALL); // Q, then Q'[2]
  unsigned char* bks = qs + 3 * C::Q_BYTES;
  unsigned char* bvs = bks + (size_t)align1k(C::BK_BYTES) * p.n_agents;
  uint64_t* bars = reinterpret_cast<uint64_t*>(bvs + (size_t)C::BK_BYTES * p.n_agents);
  __shared__ int s_fail;

  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int gq = lane >> 2, t4 = lane & 3;
  const int mi = lane >> 3, rr = lane & 7;
  const int unit = blockIdx.y;
  const int seq = unit / p.n_kv, kvh = unit % p.n_kv;
  const int split = blockIdx.x;
  const int ns = p.n_splits;
  const int g = p.g, na = p.n_agents, n_rows = na * g;

  // ---- key range of this split
  const int64_t kvl = p.kv_len[seq];
  if (kvl < 1 || kvl > p.max_kv_len) {
    if (tid == 0 && split == 0) atomicOr(p.err, 1);
    return;
  }
  const int64_t total_tiles = (p.max_kv_len + KT - 1) / KT;
  const int64_t tb = split * total_tiles / ns;
  const int64_t te = (split + 1) * total_tiles / ns;
  const int64_t k_lo = tb * KT;
  const int64_t k_hi = min(te * KT, kvl);
  const int n_tiles = k_hi > k_lo ? (int)((k_hi - k_lo + KT - 1) / KT) : 0;

  const uint32_t area_u = smem_u32(area);
  const uint32_t ptile_u = smem_u32(ptile);
  const uint32_t qs_u = smem_u32(qs);
  const uint32_t qp_u = qs_u + C::Q_BYTES;     // Q'[pb] at qp_u + pb * Q_BYTES
  const uint32_t bks_u = smem_u32(bks);
  const uint32_t bvs_u = smem_u32(bvs);
  const uint32_t full_u = smem_u32(bars);        // [ST]
  const uint32_t empty_u = full_u + 8 * ST;      // [ST]
  const uint32_t bvbar = full_u + 16 * ST;
  const int64_t ldB = (int64_t)p.n_kv * D;

  if (tid == 0) {
    s_fail = 0;
    for (int s = 0; s < ST; ++s) {
      mbar_init(full_u + 8 * s, 1);
      mbar_init(empty_u + 8 * s, NES + NPV);
    }
    mbar_init(bvbar, 1);
    fence_mbar_init();
    tma_prefetch(&tmK);
    tma_prefetch(&tmV);
    tma_prefetch(&tmL);
  }
  __syncthreads();
  pdl_launch_dependents();  // the split merge may be scheduled; it waits for this grid

  auto issue = [&](int n) {  // TMA of tile n into stage n % ST (one thread)
    const int s = n % ST;
    const uint32_t sb = area_u + s * C::STAGE;
    const uint32_t bar = full_u + 8 * s;
    const int key0 = (int)(k_lo + (int64_t)n * KT);
    mbar_expect_tx(bar, 2 * C::KV_TILE + KT * 2 * R * 2);
#pragma unroll
    for (int b = 0; b < D / 64; ++b) {
      tma_load_4d(sb + b * KT * 128, &tmK, bar, 64 * b, key0, kvh, seq);
      tma_load_4d(sb + C::KV_TILE + b * KT * 128, &tmV, bar, 64 * b, key0, kvh, seq);
    }
    constexpr int LB = (2 * R) < 64 ? 2 * R : 64;
#pragma unroll
    for (int b = 0; b < (2 * R) / LB; ++b)
      tma_load_3d(sb + 2 * C::KV_TILE + b * KT * LB * 2, &tmL, bar, LB * b, key0, seq);
  };
  if (tid == 0) {
    for (int n = 0; n < ST && n < n_tiles; ++n) issue(n);
    // B_v^a head slices for the epilogue, row by row, land while the loop runs
    const __nv_bfloat16* Bv = reinterpret_cast<const __nv_bfloat16*>(p.B_v);
    mbar_expect_tx(bvbar, (uint32_t)(na * C::BK_BYTES));
    for (int i = 0; i < na * R; ++i)
      bulk_load(bvs_u + i * D * 2, Bv + (int64_t)i * ldB + kvh * D, D * 2, bvbar);
  }

  // ---- per-CTA constants: B_k^a slices, queries, RoPE frequencies
  {
    const __nv_bfloat16* Bk = reinterpret_cast<const __nv_bfloat16*>(p.B_k);
    const int chunks = na * R * (D / 8);
    for (int i = tid; i < chunks; i += NTHR) {
      const int a = i / (R * (D / 8)), rem = i % (R * (D / 8));
      const int j = rem / (D / 8), c = rem % (D / 8);
      const uint4 v = *reinterpret_cast<const uint4*>(Bk + ((int64_t)a * R + j) * ldB + kvh * D + c * 8);
      *reinterpret_cast<uint4*>(bks + (size_t)a * align1k(C::BK_BYTES) + tile_off<D, R>(j, c * 8)) = v;
    }
    const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(p.q);
    for (int i = tid; i < ROWS * (D / 8); i += NTHR) {
      const int row = i / (D / 8), c = i % (D / 8);
      uint4 v = make_uint4(0, 0, 0, 0);
      if (row < n_rows) {
        const int a = row / g, gi = row % g;
        v = *reinterpret_cast<const uint4*>(Q + (((int64_t)seq * na + a) * p.n_q + kvh * g + gi) * D + c * 8);
      }
      *reinterpret_cast<uint4*>(qs + tile_off<D, ROWS>(row, c * 8)) = v;
    }
    if (tid < D / 2) theta[tid] = rt.theta[tid];
  }
  __syncthreads();
  if (tid < D / 2) rotate_queries<D, ROWS>(qs_u, qp_u, theta, k_lo, p.s, tid);
  __syncthreads();

  const float sl2 = p.scale * kLog2e;
  int fail = 0;

  if (w < NES) {
    // ======================================================== score warps
    // R(j) for this thread's keys j = 16w+gq (+8) and its 16 frequencies
    float2 cj[C::NG][2][4];
#pragma unroll
    for (int grp = 0; grp < C::NG; ++grp)
#pragma unroll
      for (int f = 0; f < 4; ++f) {
        const int i = 16 * grp + 8 * (f >> 1) + 2 * t4 + (f & 1);
#pragma unroll
        for (int kr = 0; kr < 2; ++kr) cj[grp][kr][f] = sincos_small((float)(16 * w + gq + 8 * kr) * (float)rt.theta[i]);
      }
    float m_st[NT][2], l_st[NT][2];
#pragma unroll
    for (int pt = 0; pt < NT; ++pt) {
      m_st[pt][0] = m_st[pt][1] = -INFINITY;
      l_st[pt][0] = l_st[pt][1] = 0.f;
    }
    for (int n = 0; n < n_tiles; ++n) {
      const int s = n % ST, pb = n & 1;
      const uint32_t sK = area_u + s * C::STAGE;
      const uint32_t sL = sK + 2 * C::KV_TILE;
      const uint32_t qpb = qp_u + pb * C::Q_BYTES;
      const int64_t k0 = k_lo + (int64_t)n * KT;
      const int64_t kw0 = k0 + 16 * w;
      if (!mbar_wait(full_u + 8 * s, (n / ST) & 1)) fail = 1;
      bar_sync(BAR_QP + pb, NTHR);  // the tile's rotated queries are ready

      float S[NT][4];
#pragma unroll
      for (int pt = 0; pt < NT; ++pt)
#pragma unroll
        for (int e = 0; e < 4; ++e) S[pt][e] = 0.f;

      if (kw0 < k_hi) {
        // base scores for every agent's rows: S^T += K_base Q^T
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          uint32_t aK[4];
          ldsm_x4(aK, sK + tile_off<D, KT>(16 * w + rr + (mi & 1) * 8, 16 * kk + (mi >> 1) * 8));
#pragma unroll
          for (int pt = 0; pt < NT; pt += 2) {
            if (pt + 1 < NT) {
              uint32_t bq[4];
              ldsm_x4(bq, qs_u + tile_off<D, ROWS>(8 * pt + rr + (mi >> 1) * 8, 16 * kk + (mi & 1) * 8));
              mma16816(S[pt], aK, bq[0], bq[1]);
              mma16816(S[pt + 1], aK, bq[2], bq[3]);
            } else {
              uint32_t b0, b1;
              ldsm_x2(b0, b1, qs_u + tile_off<D, ROWS>(8 * pt + rr, 16 * kk + ((lane >> 3) & 1) * 8));
              mma16816(S[pt], aK, b0, b1);
            }
          }
        }
        // LoRA key deltas, agent by agent (two at a time)
        uint32_t aL[C::KS][4];
        if constexpr (R >= 16) {
#pragma unroll
          for (int ks = 0; ks < C::KS; ++ks)
            ldsm_x4(aL[ks], sL + tile_off<2 * R, KT>(16 * w + rr + (mi & 1) * 8, 16 * ks + (mi >> 1) * 8));
        } else {
          ldsm_x2(aL[0][0], aL[0][1], sL + tile_off<2 * R, KT>(16 * w + (lane & 15), 0));
        }
#pragma unroll
        for (int grp = 0; grp < C::NG; ++grp) {
          // n-tiles q=0,1 -> 2grp, 2grp+1 (columns < d/2); q=2,3 -> their RoPE partners
          const int ntq[4] = {2 * grp, 2 * grp + 1, 2 * grp + D / 16, 2 * grp + 1 + D / 16};
          for (int a0 = 0; a0 < na; a0 += 2) {
            const bool two = a0 + 1 < na;
            float acc[2][4][4];
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
              for (int q = 0; q < 4; ++q)
#pragma unroll
                for (int e = 0; e < 4; ++e) acc[u][q][e] = 0.f;
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              if (u == 1 && !two) break;
              const uint32_t bk_a = bks_u + (a0 + u) * align1k(C::BK_BYTES);
              if constexpr (R >= 16) {
#pragma unroll
                for (int ks = 0; ks < C::KS; ++ks)
#pragma unroll
                  for (int h = 0; h < 2; ++h) {
                    uint32_t b[4];
                    ldsm_x4_t(b, bk_a + tile_off<D, R>(16 * ks + rr + (mi & 1) * 8,
                                                       8 * (mi < 2 ? ntq[2 * h] : ntq[2 * h + 1])));
                    mma16816(acc[u][2 * h], aL[ks], b[0], b[1]);
                    mma16816(acc[u][2 * h + 1], aL[ks], b[2], b[3]);
                  }
              } else {
                uint32_t b[4];
                ldsm_x4_t(b, bk_a + tile_off<D, R>(rr, 8 * (2 * grp + (mi & 1) + (mi >> 1) * (D / 16))));
#pragma unroll
                for (int q = 0; q < 4; ++q) mma1688(acc[u][q], aL[0][0], aL[0][1], b[q]);
              }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              if (u == 1 && !two) break;
              const int a = a0 + u;
              // R(j) of the delta, in the A layout of the score MMA
              uint32_t A_lo[4], A_hi[4];
#pragma unroll
              for (int q = 0; q < 2; ++q)
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                  float lo2[2], hi2[2];
#pragma unroll
                  for (int x = 0; x < 2; ++x) {
                    const int e = 2 * hh + x;
                    const float2 c = cj[grp][hh][2 * q + x];
                    const float x1 = acc[u][q][e], x2 = acc[u][q + 2][e];
                    lo2[x] = fmaf(-x2, c.y, x1 * c.x);
                    hi2[x] = fmaf(x1, c.y, x2 * c.x);
                  }
                  A_lo[2 * q + hh] = pack_bf16(lo2[0], lo2[1]);
                  A_hi[2 * q + hh] = pack_bf16(hi2[0], hi2[1]);
                }
              // this agent's rotated query rows live in n-tile pa; other rows are zeroed
              const int pa = (a * g) >> 3;
              uint32_t bq[4];
              ldsm_x4(bq, qpb + tile_off<D, ROWS>(8 * pa + rr, 16 * grp + (mi & 1) * 8 + (mi >> 1) * (D / 2)));
              if ((8 * pa + gq) / g != a) bq[0] = bq[1] = bq[2] = bq[3] = 0u;
#pragma unroll
              for (int pt = 0; pt < NT; ++pt)
                if (pt == pa) {
                  mma16816(S[pt], A_lo, bq[0], bq[1]);
                  mma16816(S[pt], A_hi, bq[2], bq[3]);
                }
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty_u + 8 * s);  // done with K and LRk of this stage

      // tile row maxima over all score warps
      const bool v0 = kw0 + gq < k_hi, v1 = kw0 + gq + 8 < k_hi;
      float x[NT][4];
      float* mxw = Mx + (pb * NES + w) * ROWS;
#pragma unroll
      for (int pt = 0; pt < NT; ++pt) {
        x[pt][0] = v0 ? S[pt][0] * sl2 : -INFINITY;
        x[pt][1] = v0 ? S[pt][1] * sl2 : -INFINITY;
        x[pt][2] = v1 ? S[pt][2] * sl2 : -INFINITY;
        x[pt][3] = v1 ? S[pt][3] * sl2 : -INFINITY;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float mt = fmaxf(x[pt][e], x[pt][e + 2]);
          mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 4));
          mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 8));
          mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16));
          if (gq == 0) mxw[8 * pt + 2 * t4 + e] = mt;
        }
      }
      bar_sync(BAR_MAX, 32 * NES);
#pragma unroll
      for (int pt = 0; pt < NT; ++pt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int row = 8 * pt + 2 * t4 + e;
          float mt = -INFINITY;
#pragma unroll
          for (int ww = 0; ww < NES; ++ww) mt = fmaxf(mt, Mx[(pb * NES + ww) * ROWS + row]);
          const float mo = m_st[pt][e];
          const float mn = fmaxf(mo, mt);
          const float corr = (mo == -INFINITY) ? 0.f : fast_exp2(mo - mn);
          const float p0 = (mn == -INFINITY) ? 0.f : fast_exp2(x[pt][e] - mn);
          const float p1 = (mn == -INFINITY) ? 0.f : fast_exp2(x[pt][e + 2] - mn);
          x[pt][e] = p0;
          x[pt][e + 2] = p1;
          l_st[pt][e] = l_st[pt][e] * corr + p0 + p1;
          m_st[pt][e] = mn;
          if (w == 0 && gq == 0) Corr[pb * ROWS + row] = corr;
        }
      // hand P^T to the value warps (buffer pb is free once they finished tile n-2)
      bar_sync(BAR_PFREE + pb, NTHR);
      const uint32_t pt_u = ptile_u + pb * C::P_TILE;
#pragma unroll
      for (int pt = 0; pt < NT; ++pt) {
        const uint32_t b0 = movmatrix_t(pack_bf16(x[pt][0], x[pt][1]));
        const uint32_t b1 = movmatrix_t(pack_bf16(x[pt][2], x[pt][3]));
        // b0 holds row 8pt+gq, keys 16w+2t4.. ; b1 the keys 8 further
        sts32(pt_u + tile_off<KT, ROWS>(8 * pt + gq, 16 * w + 2 * t4), b0);
        sts32(pt_u + tile_off<KT, ROWS>(8 * pt + gq, 16 * w + 8 + 2 * t4), b1);
      }
      bar_arrive(BAR_P + pb, NTHR);
    }
    // row sums of this warp's keys -> shared memory; warp 0 also keeps m
#pragma unroll
    for (int pt = 0; pt < NT; ++pt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float l = l_st[pt][e];
        l += __shfl_xor_sync(0xffffffffu, l, 4);
        l += __shfl_xor_sync(0xffffffffu, l, 8);
        l += __shfl_xor_sync(0xffffffffu, l, 16);
        if (gq == 0) Lw[w * ROWS + 8 * pt + 2 * t4 + e] = l;
      }
    bar_sync(BAR_END, NTHR);  // loop done everywhere; the stage area may be reused
    float* Mo = reinterpret_cast<float*>(area);
    if (w == 0 && gq == 0) {
#pragma unroll
      for (int pt = 0; pt < NT; ++pt)
#pragma unroll
        for (int e = 0; e < 2; ++e) Mo[(8 * pt + 2 * t4 + e) * W + D + R] = m_st[pt][e];
    }
  } else {
    // ======================================================== value warps
    const int pv = w - NES;
    float O[C::MT][NT][4];
    float Olr[C::MR][NT][4];
#pragma unroll
    for (int mt = 0; mt < C::MT; ++mt)
#pragma unroll
      for (int pt = 0; pt < NT; ++pt)
#pragma unroll
        for (int e = 0; e < 4; ++e) O[mt][pt][e] = 0.f;
#pragma unroll
    for (int mr = 0; mr < C::MR; ++mr)
#pragma unroll
      for (int pt = 0; pt < NT; ++pt)
#pragma unroll
        for (int e = 0; e < 4; ++e) Olr[mr][pt][e] = 0.f;
    if (n_tiles > 0) {
      bar_arrive(BAR_QP + 0, NTHR);
      bar_arrive(BAR_PFREE + 0, NTHR);
    }
    if (n_tiles > 1) bar_arrive(BAR_PFREE + 1, NTHR);
    const int d0 = pv * (D / 2);
    for (int n = 0; n < n_tiles; ++n) {
      const int s = n % ST, pb = n & 1;
      const uint32_t sV = area_u + s * C::STAGE + C::KV_TILE;
      const uint32_t sL = area_u + s * C::STAGE + 2 * C::KV_TILE;
      const int64_t k0 = k_lo + (int64_t)n * KT;
      // rotated queries for the next tile (its buffer was last read in tile n-1)
      if (n + 1 < n_tiles) {
        const int i = pv * 32 + lane;
        if (i < D / 2)
          rotate_queries<D, ROWS>(qs_u, qp_u + ((n + 1) & 1) * C::Q_BYTES, theta, k0 + KT, p.s, i);
        bar_arrive(BAR_QP + ((n + 1) & 1), NTHR);
      }
      if (!mbar_wait(full_u + 8 * s, (n / ST) & 1)) fail = 1;
      if (k0 + KT > k_hi) {
        // rows at or past k_hi may hold anything: zero the V and LRv rows this
        // warp multiplies so that P = 0 never meets a non-finite value
        unsigned char* vb = area + s * C::STAGE + C::KV_TILE;
        unsigned char* lb = area + s * C::STAGE + 2 * C::KV_TILE;
        const int first = (int)(k_hi - k0);
        for (int i = lane; i < (KT - first) * (D / 4); i += 32) {
          const int row = first + i / (D / 4), c = d0 + 2 * (i % (D / 4));
          *reinterpret_cast<uint32_t*>(vb + tile_off<D, KT>(row, c)) = 0u;
        }
        if (pv == 0)
          for (int i = lane; i < (KT - first) * (R / 2); i += 32) {
            const int row = first + i / (R / 2), c = R + 2 * (i % (R / 2));
            *reinterpret_cast<uint32_t*>(lb + tile_off<2 * R, KT>(row, c)) = 0u;
          }
        fence_proxy_async_smem();
        __syncwarp();
      }
      bar_sync(BAR_P + pb, NTHR);
#pragma unroll
      for (int pt = 0; pt < NT; ++pt) {
        const float c0 = Corr[pb * ROWS + 8 * pt + 2 * t4];
        const float c1 = Corr[pb * ROWS + 8 * pt + 2 * t4 + 1];
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) {
          O[mt][pt][0] *= c0; O[mt][pt][2] *= c0;
          O[mt][pt][1] *= c1; O[mt][pt][3] *= c1;
        }
#pragma unroll
        for (int mr = 0; mr < C::MR; ++mr) {
          Olr[mr][pt][0] *= c0; Olr[mr][pt][2] *= c0;
          Olr[mr][pt][1] *= c1; Olr[mr][pt][3] *= c1;
        }
      }
      const uint32_t pt_u = ptile_u + pb * C::P_TILE;
#pragma unroll 2
      for (int ks = 0; ks < KT / 16; ++ks) {
        // P^T as the B operand: rows 8pt.. (N) x keys 16ks.. (K)
        uint32_t bP[NT][2];
#pragma unroll
        for (int pt = 0; pt < NT; ++pt)
          ldsm_x2(bP[pt][0], bP[pt][1], pt_u + tile_off<KT, ROWS>(8 * pt + rr, 16 * ks + ((lane >> 3) & 1) * 8));
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) {
          uint32_t aV[4];
          ldsm_x4_t(aV, sV + tile_off<D, KT>(16 * ks + rr + (mi >> 1) * 8, d0 + 16 * mt + (mi & 1) * 8));
#pragma unroll
          for (int pt = 0; pt < NT; ++pt) mma16816(O[mt][pt], aV, bP[pt][0], bP[pt][1]);
        }
        if (pv == 0) {
#pragma unroll
          for (int mr = 0; mr < C::MR; ++mr) {
            uint32_t aV[4];
            if constexpr (R >= 16) {
              ldsm_x4_t(aV, sL + tile_off<2 * R, KT>(16 * ks + rr + (mi >> 1) * 8, R + 16 * mr + (mi & 1) * 8));
            } else {
              ldsm_x4_t(aV, sL + tile_off<2 * R, KT>(16 * ks + rr + (mi >> 1) * 8, R));
              aV[1] = aV[3] = 0u;  // rows r >= 8 do not exist
            }
#pragma unroll
            for (int pt = 0; pt < NT; ++pt) mma16816(Olr[mr][pt], aV, bP[pt][0], bP[pt][1]);
          }
        }
      }
      __syncwarp();
      if (n + 2 < n_tiles) bar_arrive(BAR_PFREE + pb, NTHR);
      if (lane == 0) mbar_arrive(empty_u + 8 * s);
      if (pv == 0 && lane == 0 && n + ST < n_tiles) {
        if (!mbar_wait(empty_u + 8 * s, (n / ST) & 1)) fail = 1;
        issue(n + ST);
      }
      __syncwarp();
    }
    bar_sync(BAR_END, NTHR);
    float* Mo = reinterpret_cast<float*>(area);
#pragma unroll
    for (int pt = 0; pt < NT; ++pt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = 8 * pt + 2 * t4 + (e & 1);
        const int dd = gq + (e >> 1) * 8;
#pragma unroll
        for (int mt = 0; mt < C::MT; ++mt) Mo[row * W + d0 + 16 * mt + dd] = O[mt][pt][e];
        if (pv == 0) {
#pragma unroll
          for (int mr = 0; mr < C::MR; ++mr)
            if (16 * mr + dd < R) Mo[row * W + D + 16 * mr + dd] = Olr[mr][pt][e];
        }
      }
  }
  if (fail) s_fail = 1;
  if (!mbar_wait(bvbar, 0)) s_fail = 1;
  __syncthreads();
  float* Mo = reinterpret_cast<float*>(area);
  for (int row = tid; row < n_rows; row += NTHR) {
    float l = 0.f;
#pragma unroll
    for (int ww = 0; ww < NES; ++ww) l += Lw[ww * ROWS + row];
    Mo[row * W + D + R + 1] = l;
  }
  // Z = O_base + s O_lr B_v^a for this CTA's partial (B_v staged by the bulk copy)
  {
    const __nv_bfloat16* bv = reinterpret_cast<const __nv_bfloat16*>(bvs);
    for (int i = tid; i < n_rows * (D / 4); i += NTHR) {
      const int row = i / (D / 4), c = 4 * (i % (D / 4));
      const __nv_bfloat16* b = bv + (size_t)(row / g) * R * D + c;
      float z0 = 0.f, z1 = 0.f, z2 = 0.f, z3 = 0.f;
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const float o = Mo[row * W + D + j];
        const uint2 bb = *reinterpret_cast<const uint2*>(b + j * D);
        const float2 f01 = unpack_bf16(bb.x), f23 = unpack_bf16(bb.y);
        z0 = fmaf(o, f01.x, z0); z1 = fmaf(o, f01.y, z1);
        z2 = fmaf(o, f23.x, z2); z3 = fmaf(o, f23.y, z3);
      }
      float4* zp = reinterpret_cast<float4*>(Mo + row * W + c);
      float4 zo = *zp;
      zo.x = fmaf(p.s, z0, zo.x); zo.y = fmaf(p.s, z1, zo.y);
      zo.z = fmaf(p.s, z2, zo.z); zo.w = fmaf(p.s, z3, zo.w);
      *zp = zo;
    }
  }
  __syncthreads();
  if (s_fail) {
    if (tid == 0) atomicOr(p.err, 2);
    return;
  }
  if (ns == 1) {
    for (int i = tid; i < n_rows * D; i += NTHR) {
      const int row = i / D, c = i % D;
      const int a = row / g, gi = row % g;
      const float l = Mo[row * W + D + R + 1];
      const float val = l > 0.f ? Mo[row * W + c] / l : 0.f;
      const int64_t oi = (((int64_t)seq * na + a) * p.n_q + kvh * g + gi) * D + c;
      if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(val);
      else reinterpret_cast<float*>(p.out)[oi] = val;
    }
  } else {
    // partial (Z, m, l) of this split -> workspace [unit][split][row][D + 4]
    constexpr int WP = D + 4;
    float* part = p.partials + ((size_t)unit * ns + split) * n_rows * WP;
    for (int i = tid; i < n_rows * (WP / 4); i += NTHR) {
      const int row = i / (WP / 4), c = 4 * (i % (WP / 4));
      float4 v;
      if (c < D) v = *reinterpret_cast<const float4*>(Mo + row * W + c);
      else v = make_float4(Mo[row * W + D + R], Mo[row * W + D + R + 1], 0.f, 0.f);
      *reinterpret_cast<float4*>(part + row * WP + c) = v;
    }
  }
}

// Merge of a unit's splits: one CTA per (row, unit), one thread per column.
// out = sum_k 2^(m_k - M) Z_k / sum_k 2^(m_k - M) l_k, M = max_k m_k.
template <int D>
__global__ void __launch_bounds__(D) decode_merge_kernel(const AttnParams p) {
  pdl_wait();  // the partials of the preceding decode grid are complete and visible
  constexpr int WP = D + 4;
  const int row = blockIdx.x, unit = blockIdx.y, c = threadIdx.x;
  {
    const int64_t kvl = p.kv_len[unit / p.n_kv];
    if (kvl < 1 || kvl > p.max_kv_len) return;  // reported by the decode grid
  }
  const int ns = p.n_splits, n_rows = p.n_agents * p.g;
  const float* base = p.partials + (size_t)unit * ns * n_rows * WP + (size_t)row * WP;
  const size_t kstr = (size_t)n_rows * WP;
  float mx = -INFINITY;
  for (int k = 0; k < ns; ++k) mx = fmaxf(mx, __ldcg(base + k * kstr + D));
  float l = 0.f, acc = 0.f;
#pragma unroll 4
  for (int k = 0; k < ns; ++k) {
    const float mk = __ldcg(base + k * kstr + D);
    const float wk = mk == -INFINITY ? 0.f : exp2f(mk - mx);
    l = fmaf(wk, __ldcg(base + k * kstr + D + 1), l);
    acc = fmaf(wk, __ldcg(base + k * kstr + c), acc);
  }
  const int seq = unit / p.n_kv, kvh = unit % p.n_kv;
  const int a = row / p.g, gi = row % p.g;
  const int64_t oi = (((int64_t)seq * p.n_agents + a) * p.n_q + kvh * p.g + gi) * D + c;
  const float val = l > 0.f ? acc / l : 0.f;
  if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(val);
  else reinterpret_cast<float*>(p.out)[oi] = val;
}

// -------------------------------------------------------------------- host
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

CUtensorMapSwizzle swizzle_for(int row_bytes) {
  return row_bytes >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : (row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
}

bool make_maps(const AttnParams& p, CUtensorMap* mk, CUtensorMap* mv, CUtensorMap* ml) {
  auto enc = encode_fn();
  if (!enc) return false;
  const int D = p.d, R = p.r;
  cuuint64_t kdims[4] = {(cuuint64_t)D, (cuuint64_t)p.L_max, (cuuint64_t)p.n_kv, (cuuint64_t)p.n_seqs};
  cuuint64_t kstr[3] = {(cuuint64_t)p.kv_tok * 2, (cuuint64_t)p.kv_head * 2, (cuuint64_t)p.kv_seq * 2};
  cuuint32_t kbox[4] = {64, (cuuint32_t)KT, 1, 1};
  cuuint32_t one[4] = {1, 1, 1, 1};
  if (enc(mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(p.k_base), kdims, kstr, kbox,
          one, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  if (enc(mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(p.v_base), kdims, kstr, kbox,
          one, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  const int lb = 2 * R < 64 ? 2 * R : 64;
  cuuint64_t ldims[3] = {(cuuint64_t)(2 * R), (cuuint64_t)p.L_max, (cuuint64_t)p.n_seqs};
  cuuint64_t lstr[2] = {(cuuint64_t)(2 * R * 2), (cuuint64_t)p.lr_seq * 2};
  cuuint32_t lbox[3] = {(cuuint32_t)lb, (cuuint32_t)KT, 1};
  if (enc(ml, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(p.lr), ldims, lstr, lbox, one,
          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_for(lb * 2), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  return true;
}

int n_rowtiles(const AttnParams& p) { return (p.n_agents * p.g + 7) / 8; }

size_t smem_for(const AttnParams& p) {
  const int NT = n_rowtiles(p), na = p.n_agents;
  switch (p.r) {
    case 8: return NT == 1 ? Cfg<128, 8, 1>::smem(na) : NT == 2 ? Cfg<128, 8, 2>::smem(na) : Cfg<128, 8, 3>::smem(na);
    case 16: return NT == 1 ? Cfg<128, 16, 1>::smem(na) : NT == 2 ? Cfg<128, 16, 2>::smem(na) : Cfg<128, 16, 3>::smem(na);
    case 32: return NT == 1 ? Cfg<128, 32, 1>::smem(na) : NT == 2 ? Cfg<128, 32, 2>::smem(na) : Cfg<128, 32, 3>::smem(na);
    default: return NT == 1 ? Cfg<128, 64, 1>::smem(na) : Cfg<128, 64, 2>::smem(na);
  }
}

// Splits per (sequence, KV head): enough CTAs for one CTA per SM.
int n_splits_for(const AttnParams& p) {
  const int units = p.n_seqs * p.n_kv;
  const int64_t total_tiles = (p.max_kv_len + KT - 1) / KT;
  int64_t ns = units >= kSMs ? 1 : kSMs / units;
  if (ns > kMaxSplits) ns = kMaxSplits;
  if (ns > total_tiles) ns = total_tiles;
  if (ns < 1) ns = 1;
  return (int)ns;
}

template <int D, int R, int NT>
cudaError_t launch_t(const AttnParams& p, cudaStream_t st) {
  using C = Cfg<D, R, NT>;
  RopeTheta rt;
  for (int i = 0; i < 64; ++i) rt.theta[i] = i < D / 2 ? std::pow(p.rope_base, -2.0 * i / D) : 0.0;
  CUtensorMap mk, mv, ml;
  if (!make_maps(p, &mk, &mv, &ml)) return cudaErrorInvalidValue;
  const size_t sm = C::smem(p.n_agents);
  auto kern = decode_bf16_kernel<D, R, NT>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_splits, p.n_seqs * p.n_kv);
  kern<<<grid, NTHR, sm, st>>>(mk, mv, ml, p, rt);
  e = cudaGetLastError();
  if (e != cudaSuccess || p.n_splits == 1) return e;
  // merge of the splits, launched early (programmatic dependent launch)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.n_agents * p.g, p.n_seqs * p.n_kv);
  cfg.blockDim = dim3(D);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, decode_merge_kernel<D>, p);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool bf16_decode_supported(const AttnParams& p) {
  if (p.d != 128) return false;
  if (!(p.g == 1 || p.g == 2 || p.g == 4 || p.g == 8)) return false;
  const int NT = n_rowtiles(p);
  if (NT > 3) return false;
  if (NT == 3 && p.r == 64) return false;
  if (p.L_max >= (1ll << 31)) return false;
  if (smem_for(p) > 227 * 1024) return false;
  return true;
}

void bf16_decode_plan(const AttnParams& p, int* n_splits, int64_t* split_len, int* rows) {
  *n_splits = n_splits_for(p);
  *split_len = KT;
  *rows = p.n_agents * p.g;
}

size_t bf16_decode_partial_bytes(const AttnParams& p) {
  const int ns = n_splits_for(p);
  if (ns == 1) return 0;
  return (size_t)p.n_seqs * p.n_kv * ns * (p.n_agents * p.g) * (p.d + 4) * sizeof(float);
}

cudaError_t launch_decode_bf16(const AttnParams& pin, la_dtype out, cudaStream_t st) {
  AttnParams p = pin;
  p.out_bf16 = out == LA_BF16;
  const int NT = n_rowtiles(p);
  switch (p.r) {
    case 8: return NT == 1 ? launch_t<128, 8, 1>(p, st) : NT == 2 ? launch_t<128, 8, 2>(p, st) : launch_t<128, 8, 3>(p, st);
    case 16: return NT == 1 ? launch_t<128, 16, 1>(p, st) : NT == 2 ? launch_t<128, 16, 2>(p, st) : launch_t<128, 16, 3>(p, st);
    case 32: return NT == 1 ? launch_t<128, 32, 1>(p, st) : NT == 2 ? launch_t<128, 32, 2>(p, st) : launch_t<128, 32, 3>(p, st);
    default: return NT == 1 ? launch_t<128, 64, 1>(p, st) : launch_t<128, 64, 2>(p, st);
  }
}

}  // namespace la
