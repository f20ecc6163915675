// Flash-LoRA-Attention decode on the tensor cores (bf16 storage, fp32 accumulate).
//
// Two kernels share this file.
//
// decode_tc_kernel (the main path).  One CTA = one (sequence, KV head, agent
// group, split of the keys).  Its rows are the group's agents x the query
// heads of the GQA group, so each base and LR tile is read from HBM once for
// all of them (LRAgent summary §3 BaseLRShared: one base and one LR cache
// shared by the whole system; with one LR cache per agent -- BaseShared --
// each stage holds every agent's own LR tile).  128-key tiles of K_base,
// V_base and the LR rows are staged in shared memory by TMA (128/64/32-byte
// swizzle, no multicast) through a two-stage full/empty mbarrier pipeline,
// with a window of later tiles requested into L2.
//  * Warp 10 issues the TMA loads and, per tile, the tcgen05 MMAs (M = 128
//    keys): the base scores S_base^T = K_base Q^T for every row and each
//    agent's key delta dK^a = LRk B_k^a (N = d, K = r), into TMEM; then the
//    previous tile's O_base^T += V_base^T P^T (M = d, N = the query rows).
//  * 8 score warps, 16 keys each (LRAgent summary App. D.1: RoPE blocks the
//    reordering, so the delta is rebuilt in head dimension).  A key at
//    position t = k0 + j of a tile starting at k0 is rotated by
//    R(t) = R(k0) R(j), so
//      q . K^a_t = q . K_base,t + (s R(-k0) q) . R(j) (LRk_t B_k^a):
//    dK^a comes out of TMEM in the mma.sync fragment layout, is turned by
//    R(j) -- whose cos / sin are per-thread constants, j being fixed per
//    thread; the turn runs on f16 pairs -- and scored (f16 mma.sync) against
//    the tile's rotated queries
//    Q' = s R(-k0) Q.  The tile's row maxima meet in shared memory; the warps
//    write P (bf16) and rescale O_base^T in TMEM when a row's maximum moved.
//  * 2 value warps: the value side reordered (LRAgent explainer, Metodologia
//    3; summary App. B) keeps the LoRA path r wide inside the loop, O_lr^T +=
//    LRv^T P^T (mma.sync); they also rotate the next tile's queries and zero
//    the rows of a tile past the sequence's end.
//  Split keys merge inside the same launch: each CTA writes (O_base, O_lr, m,
//  l), the unit's CTAs wait for one another (cooperative launch, bounded
//  wait), and each merges a share of the unit's rows, applying B_v^a once per
//  row: out = (sum_k w_k O_base,k + s (sum_k w_k O_lr,k) B_v^a) with
//  w_k = 2^(m_k - M) / sum_k 2^(m_k - M) l_k.  The launch is a programmatic
//  dependent of the kernel before it (the step's LR append): the set-up runs
//  while that kernel finishes, every input is read after griddepcontrol.wait
//  -- in a decode step every input but the LR rows (the append's output) is
//  read at once, and only the LR loads wait.
//
// decode_bf16_kernel + decode_merge_kernel (shapes the first kernel does not
// take: d = 64, r = 8).  The same tiling with mma.sync for every product and a
// second kernel, chained by programmatic dependent launch, for the merge.
#include <cudaTypedefs.h>

#include <cmath>

#include <cuda_fp16.h>

#include "bf16_common.cuh"
#include "la_internal.cuh"
#include "ptx.cuh"

namespace la {
namespace {

using namespace ptx;

constexpr int ST = 2;               // pipeline stages
// tiles requested into L2 ahead of the stage loads: enough to keep HBM busy
// between refills, few enough that 148 CTAs' windows stay resident in L2
constexpr int kL2Ahead = 4;
constexpr int KT = 128;             // keys per tile
constexpr int NES = 8;              // score warps (16 keys each)
constexpr int NPV = 2;              // value warps
constexpr int NTHR = 32 * (NES + NPV);
constexpr int kMaxSplits = 32;
constexpr int kSMs = 148;
// named barriers (0 is __syncthreads)
constexpr int BAR_MAX = 1, BAR_P = 2, BAR_PFREE = 4, BAR_QP = 6, BAR_END = 8;


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
      tma_load_4d(sb + 2 * C::KV_TILE + b * KT * LB * 2, &tmL, bar, LB * b, key0, seq, 0);
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
// out = sum_k 2^(m_k - M) Z_k / sum_k 2^(m_k - M) l_k, M = max_k m_k.  The
// split weights are formed once per CTA; every thread then issues its column's
// loads of all splits before using them, so the merge costs a couple of L2
// round trips, not one per split.
template <int D>
__global__ void __launch_bounds__(D) decode_merge_kernel(const AttnParams p) {
  constexpr int WP = D + 4;
  __shared__ float wts[kMaxSplits];
  const int row = blockIdx.x, unit = blockIdx.y, c = threadIdx.x;
  const int64_t kvl = p.kv_len[unit / p.n_kv];  // an input: read before the wait
  pdl_wait();  // the partials of the preceding decode grid are complete and visible
  if (kvl < 1 || kvl > p.max_kv_len) return;  // reported by the decode grid
  const int ns = p.n_splits, n_rows = p.n_agents * p.g;
  const float* base = p.partials + (size_t)unit * ns * n_rows * WP + (size_t)row * WP;
  const size_t kstr = (size_t)n_rows * WP;
  // every load of this thread is issued before any of them is used
  float z[kMaxSplits];
#pragma unroll
  for (int k = 0; k < kMaxSplits; ++k) z[k] = k < ns ? __ldcg(base + k * kstr + c) : 0.f;
  float2 ml = make_float2(-INFINITY, 0.f);
  if (c < ns) ml = __ldcg(reinterpret_cast<const float2*>(base + c * kstr + D));
  if (c < 32) {
    float mx = ml.x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float wk = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - mx);
    float l = wk * ml.y;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (c < ns) wts[c] = l > 0.f ? wk / l : 0.f;
  }
  __syncthreads();
  float acc = 0.f;
#pragma unroll
  for (int k = 0; k < kMaxSplits; ++k)
    if (k < ns) acc = fmaf(wts[k], z[k], acc);
  const int seq = unit / p.n_kv, kvh = unit % p.n_kv;
  const int a = row / p.g, gi = row % p.g;
  const int64_t oi = (((int64_t)seq * p.n_agents + a) * p.n_q + kvh * p.g + gi) * D + c;
  if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(acc);
  else reinterpret_cast<float*>(p.out)[oi] = acc;
}

// ============================================================================
// Decode with the 5th-generation tensor cores (tcgen05 / TMEM).
//
// The agent-shared GEMMs of a 128-key tile run as single-thread-issued
// tcgen05 MMAs (M = 128 keys) whose operands are read from shared memory once
// per CTA: the base scores S_base^T = K_base Q^T (N = the query rows, padded to
// 16 / 32) and every agent's key delta dK^a = LRk B_k^a (N = d, K = r), all
// accumulated in TMEM, and O_base^T += V_base^T P^T.  Eight score warps --
// two per 32-lane TMEM sub-partition, 16 keys each -- read dK^a straight into
// the mma.sync accumulator layout (tcgen05.ld 16x256b), turn it by R(j), score
// it against the tile's rotated queries and run the softmax; two value warps
// keep the r-wide O_lr; warp 10 stages B_k and the tiles (TMA) and issues the
// MMAs.
// ============================================================================
constexpr int TC_NES = 8;                          // score warps (16 keys each)
constexpr int TC_NTHR = 32 * (TC_NES + NPV + 1);   // + value warps + TMA / MMA warp
constexpr int TC_COLS = 512;                        // TMEM columns allocated
constexpr int TC_SCOL = 384;                        // TMEM column of S_base
constexpr int TC_OCOL = 448;                        // TMEM column of O_base^T (d lanes x query rows)

// PA: one LR cache per agent with several agents per CTA -- every stage holds
// each agent's LR tile beside the shared base tiles (r = 16: up to 3 agents)
template <int D, int R, int NT, bool PA = false>
struct TCfg {
  static constexpr int ROWS = NT * 8;
  static constexpr int NLR = PA ? 3 : 1;               // LR tiles per stage
  static constexpr int QPAD = NT <= 2 ? 16 : 32;        // N of the base-score MMA
  static constexpr int W = D + R + 4;
  static constexpr int KV_TILE = KT * D * 2;
  static constexpr int LR_TILE = align1k(KT * 2 * R * 2);
  static constexpr int STAGE = 2 * KV_TILE + NLR * LR_TILE;
  static constexpr int AREA = imax(ST * STAGE, align1k(ROWS * W * 4));
  static constexpr int P_TILE = align1k(ROWS * KT * 2);
  static constexpr int SMALL = 2 * TC_NES * ROWS * 4 + 2 * ROWS * 4 + TC_NES * ROWS * 4 + 64 * 8 + 16 + 64 * 8;
  static constexpr int QU_BYTES = align1k(QPAD * D * 2);   // Q as the MMA operand
  static constexpr int QP_BYTES = align1k(ROWS * D * 2);   // each Q' buffer
  static constexpr int BK_BYTES = R * D * 2;
  static constexpr int KS = R / 16;
  static constexpr int MR = R / 16;
  static constexpr int NG = D / 32;
  // LR tile: rows of 2r bf16 in boxes of min(2r, 64); its swizzle span
  static constexpr int LR_ROWB = (2 * R < 64 ? 2 * R : 64) * 2;
  static constexpr uint32_t LR_LAYOUT = LR_ROWB == 128 ? 2u : (LR_ROWB == 64 ? 4u : 6u);
  static size_t smem(int n_agents) {  // n_agents: the agents of one CTA
    return 1024 + AREA + 2 * P_TILE + align1k(SMALL) + QU_BYTES + 2 * QP_BYTES +
           (size_t)align1k(BK_BYTES) * n_agents + 128;
  }
};

// Q' = R(-k0) Q scaled by s for one frequency i of every row, from the
// scaled (cos, sin)(k0 theta_i) (bf16 in, f16 out; swizzled 64-column boxes).
template <int D, int SRC_ROWS, int DST_ROWS>
__device__ __forceinline__ void rotate_queries_cs(uint32_t qs_u, uint32_t qp_u, float c, float sn, int i) {
#pragma unroll 4
  for (int row = 0; row < DST_ROWS; ++row) {
    uint16_t a, b;
    asm volatile("ld.shared.b16 %0, [%1];" : "=h"(a) : "r"(qs_u + tile_off<D, SRC_ROWS>(row, i)));
    asm volatile("ld.shared.b16 %0, [%1];" : "=h"(b) : "r"(qs_u + tile_off<D, SRC_ROWS>(row, i + D / 2)));
    const float x1 = __uint_as_float((uint32_t)a << 16), x2 = __uint_as_float((uint32_t)b << 16);
    const __half y1 = __float2half_rn(fmaf(x1, c, x2 * sn));
    const __half y2 = __float2half_rn(fmaf(x2, c, -x1 * sn));
    sts16(qp_u + tile_off<D, DST_ROWS>(row, i), *reinterpret_cast<const uint16_t*>(&y1));
    sts16(qp_u + tile_off<D, DST_ROWS>(row, i + D / 2), *reinterpret_cast<const uint16_t*>(&y2));
  }
}

__device__ __forceinline__ uint32_t pack_half2(float2 v) {
  __half2 h = __floats2half2_rn(v.x, v.y);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ float2 unpack_half2(uint32_t v) {
  return __half22float2(*reinterpret_cast<const __half2*>(&v));
}

template <int D, int R, int NT, bool PA>
__global__ void __launch_bounds__(TC_NTHR, 1)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                     const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmL,
                     const __grid_constant__ CUtensorMap tmB, const AttnParams p,
                     const __grid_constant__ RopeTheta rt) {
  using C = TCfg<D, R, NT, PA>;
  constexpr int W = C::W, ROWS = C::ROWS, QPAD = C::QPAD;
  constexpr int NB = 32 * (TC_NES + NPV);   // threads in the score / value barriers
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* area = smem;
  unsigned char* ptile = area + C::AREA;
  float* Mx = reinterpret_cast<float*>(ptile + 2 * C::P_TILE);   // [2][ROWS][NES]
  static_assert(TC_NES == 8, "a row's maxima are read as two float4");
  float* Corr = Mx + 2 * TC_NES * ROWS;                          // [2][ROWS]
  float* Lw = Corr + 2 * ROWS;                                   // [NES][ROWS]
  double* theta = reinterpret_cast<double*>(Lw + TC_NES * ROWS); // [64]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(theta + 64);
  float2* cs0 = reinterpret_cast<float2*>(tslot + 4);             // [64] s (cos, sin)(k_lo theta_i)
  unsigned char* qu = ptile + 2 * C::P_TILE + align1k(C::SMALL);  // Q (MMA operand)
  unsigned char* qpb0 = qu + C::QU_BYTES;                          // Q'[2]
  unsigned char* bks = qpb0 + 2 * C::QP_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(bks + (size_t)align1k(C::BK_BYTES) * p.agent_group);
  __shared__ int s_fail;

  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int gq = lane >> 2, t4 = lane & 3;
  const int mi = lane >> 3, rr = lane & 7;
  const int unit = blockIdx.z;
  const int seq = unit / p.n_kv, kvh = unit % p.n_kv;
  const int split = blockIdx.x;
  const int ns = p.n_splits;
  // this CTA's agents: group blockIdx.y of p.agent_group agents (the groups of a
  // unit are adjacent in launch order, so its cache tiles are read from HBM once
  // and are L2 hits for the other groups)
  const int agent0 = blockIdx.y * p.agent_group;
  const int lra = p.lr_agent ? agent0 : 0;   // LR cache of the CTA's agent (one per CTA then)
  const int g = p.g, na = min(p.agent_group, p.n_agents - agent0), n_rows = na * g;
  const int na_tot = p.n_agents;
  const int unitg = blockIdx.y * (p.n_seqs * p.n_kv) + unit;   // (agent group, unit)

  const int64_t total_tiles = (p.max_kv_len + KT - 1) / KT;
  const int64_t tb = split * total_tiles / ns;
  const int64_t te = (split + 1) * total_tiles / ns;
  const int64_t k_lo = tb * KT;

  const uint32_t area_u = smem_u32(area);
  const uint32_t ptile_u = smem_u32(ptile);
  const uint32_t qu_u = smem_u32(qu);
  const uint32_t qp_u = smem_u32(qpb0);
  const uint32_t bks_u = smem_u32(bks);
  const uint32_t full_u = smem_u32(bars);          // [ST]
  const uint32_t empty_u = full_u + 8 * ST;        // [ST]: MMA commit + value warps
  const uint32_t tfull = full_u + 16 * ST;         // MMA results of a tile are in TMEM
  const uint32_t tempty = tfull + 8;               // score warps are done reading TMEM
  const uint32_t bkbar = tfull + 24;              // B_k^a slices have landed
  const uint32_t qbar = tfull + 32;               // the queries have landed (staged unswizzled)
  const uint32_t pfull = tfull + 40;              // P of a tile is written, its V rows are final
  const uint32_t pvdone = tfull + 48;             // the P V_base MMA of a tile has completed
  const int64_t ldB = (int64_t)p.n_kv * D;

  // TMA of tile n into stage n % ST (one thread): the base tiles (and the
  // stage's whole byte count), then the LR rows
  auto issue_kv = [&](int n) {
    const int s = n % ST;
    const uint32_t sb = area_u + s * C::STAGE;
    const uint32_t bar = full_u + 8 * s;
    const int key0 = (int)(k_lo + (int64_t)n * KT);
    const int nlr = PA ? na : 1;   // the agents' own LR tiles, or the shared one
    mbar_expect_tx(bar, 2 * C::KV_TILE + nlr * KT * 2 * R * 2);
#pragma unroll
    for (int b = 0; b < D / 64; ++b) {
      tma_load_4d(sb + b * KT * 128, &tmK, bar, 64 * b, key0, kvh, seq);
      tma_load_4d(sb + C::KV_TILE + b * KT * 128, &tmV, bar, 64 * b, key0, kvh, seq);
    }
  };
  auto issue_lr = [&](int n) {
    const int s = n % ST;
    const uint32_t sb = area_u + s * C::STAGE;
    const uint32_t bar = full_u + 8 * s;
    const int key0 = (int)(k_lo + (int64_t)n * KT);
    const int nlr = PA ? na : 1;
    constexpr int LB = (2 * R) < 64 ? 2 * R : 64;
    for (int al = 0; al < nlr; ++al)
#pragma unroll
      for (int b = 0; b < (2 * R) / LB; ++b)
        tma_load_4d(sb + 2 * C::KV_TILE + al * C::LR_TILE + b * KT * LB * 2, &tmL, bar, LB * b, key0, seq,
                    PA ? agent0 + al : lra);
  };
  auto issue = [&](int n) {
    issue_kv(n);
    issue_lr(n);
  };

  // ---- first loads (independent of kv_len): queries, B_k^a, the first tiles, B_v^a
  const int n_spec = (int)min((int64_t)ST, te - tb);
  if (w == TC_NES + NPV && lane == 0) {
    s_fail = 0;
    for (int s = 0; s < ST; ++s) {
      mbar_init(full_u + 8 * s, 1);
      mbar_init(empty_u + 8 * s, 1 + NPV);
    }
    mbar_init(tfull, 1);
    mbar_init(tempty, TC_NES);
    mbar_init(bkbar, 1);
    mbar_init(qbar, 1);
    mbar_init(pfull, TC_NES + NPV);
    mbar_init(pvdone, 1);
    fence_mbar_init();
    tma_prefetch(&tmB);
    tma_prefetch(&tmK);
    tma_prefetch(&tmV);
    tma_prefetch(&tmL);
    // launched as a programmatic dependent of the preceding kernel: everything
    // above overlaps its tail, and every read of an input comes after the wait
    // (a no-op without a preceding kernel) -- except in a decode step, whose
    // preceding kernel (the row append) writes only LR rows: there the
    // queries, B_k and the first base tiles are requested at once, and only
    // the LR rows wait
    if (!p.early) pdl_wait();
    // each agent's g query rows of this KV head are contiguous
    const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(p.q);
    mbar_expect_tx(qbar, (uint32_t)(n_rows * D * 2));
    for (int a = 0; a < na; ++a)
      bulk_load(ptile_u + a * g * D * 2, Q + (((int64_t)seq * na_tot + agent0 + a) * p.n_q + kvh * g) * D,
                (uint32_t)(g * D * 2), qbar);
    // B_k^a head slices (r rows x 64 d boxes, the MN-major MMA operand)
    mbar_expect_tx(bkbar, (uint32_t)(na * C::BK_BYTES));
    for (int a = 0; a < na; ++a)
#pragma unroll
      for (int b = 0; b < D / 64; ++b)
        tma_load_3d(bks_u + a * align1k(C::BK_BYTES) + b * R * 128, &tmB, bkbar, kvh * D + 64 * b, 0, agent0 + a);
    // the first stages before kv_len is known: tiles of this split's range
    // (by max_kv_len) past the sequence's length are loaded but never used
    if (p.early) {
      for (int n = 0; n < n_spec; ++n) issue_kv(n);
      pdl_wait();   // the append's LR rows are complete and visible
      for (int n = 0; n < n_spec; ++n) issue_lr(n);
    } else {
      for (int n = 0; n < n_spec; ++n) issue(n);
    }
  }
  // kv_len is written before the step's append, so a step reads it at once;
  // the LR rows (the append's output) are read only by the TMA thread's loads
  if (!p.early) pdl_wait();
  const int64_t kvl = p.kv_len[seq];  // in flight while the constants are computed
  const int sp = w & 3, kb = 32 * sp + 16 * (w >> 2);  // score warp: TMEM sub-partition, first key
  // R(j) for this thread's keys j = kb + gq + 8 hh and its frequencies
  // i = 16 grp + 8 q + 2 t4 (+1), as (cos, cos) and (sin, sin) f16 pairs over
  // the two adjacent frequencies: the operands of the packed f16x2 rotation
  uint32_t RC[C::NG][2][2], RS[C::NG][2][2];
  if (w < TC_NES) {
#pragma unroll
    for (int grp = 0; grp < C::NG; ++grp)
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int i = 16 * grp + 8 * q + 2 * t4;
        const float th0 = rt.thetaf[i], th1 = rt.thetaf[i + 1];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const float j = (float)(kb + gq + 8 * hh);
          const float2 a = sincos_small(j * th0), b = sincos_small(j * th1);
          RC[grp][hh][q] = pack_half2(make_float2(a.x, b.x));
          RS[grp][hh][q] = pack_half2(make_float2(a.y, b.y));
        }
      }
  }
  if (tid < D / 2) theta[tid] = rt.theta[tid];
  if (w >= TC_NES && w < TC_NES + NPV) {
    // the first tile's query rotation R(-k_lo), scaled by s (exact in fp64)
    for (int i = tid - 32 * TC_NES; i < D / 2; i += 32 * NPV) {
      const float2 cs = rope_cs_exact(k_lo + p.key_pos0, rt.theta[i]);
      cs0[i] = make_float2(cs.x * p.s, cs.y * p.s);
    }
  }
  // a sharded decode's slice may hold none of a sequence's keys (kv_len 0)
  if (kvl < (p.row_stats ? 0 : 1) || kvl > p.max_kv_len) {
    if (tid == 0 && split == 0) atomicOr(p.err, 1);
    if (w == TC_NES + NPV && lane == 0) {  // the copies in flight land before the CTA leaves
      mbar_wait(qbar, 0);
      mbar_wait(bkbar, 0);
      for (int n = 0; n < n_spec; ++n) mbar_wait(full_u + 8 * n, 0);
    }
    return;
  }
  const int64_t k_hi = min(te * KT, kvl);
  const int n_tiles = k_hi > k_lo ? (int)((k_hi - k_lo + KT - 1) / KT) : 0;
  if (w == TC_NES + NPV) tmem_alloc(smem_u32(tslot), TC_COLS);

  int fail = 0;
  __syncthreads();  // barriers initialised, cs0 ready
  if (!mbar_wait(qbar, 0)) fail = 1;
  // Q (swizzled: the base-score MMA operand) and Q' = s R(-k_lo) Q for the first tile
  for (int i = tid; i < QPAD * (D / 16); i += TC_NTHR) {
    const int row = i / (D / 16), c = i % (D / 16);
    uint4 v1 = make_uint4(0, 0, 0, 0), v2 = v1;
    if (row < n_rows) {
      v1 = *reinterpret_cast<const uint4*>(ptile + (size_t)row * D * 2 + c * 16);
      v2 = *reinterpret_cast<const uint4*>(ptile + (size_t)row * D * 2 + D + c * 16);
    }
    *reinterpret_cast<uint4*>(qu + tile_off<D, QPAD>(row, c * 8)) = v1;
    *reinterpret_cast<uint4*>(qu + tile_off<D, QPAD>(row, c * 8 + D / 2)) = v2;
    if (row < ROWS) {
      const uint32_t* x1 = reinterpret_cast<const uint32_t*>(&v1);
      const uint32_t* x2 = reinterpret_cast<const uint32_t*>(&v2);
      uint4 y1, y2;
      uint32_t* o1 = reinterpret_cast<uint32_t*>(&y1);
      uint32_t* o2 = reinterpret_cast<uint32_t*>(&y2);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 a = unpack_bf16(x1[e]), b = unpack_bf16(x2[e]);
        const float2 c0 = cs0[8 * c + 2 * e], c1 = cs0[8 * c + 2 * e + 1];
        o1[e] = pack_half2(make_float2(fmaf(a.x, c0.x, b.x * c0.y), fmaf(a.y, c1.x, b.y * c1.y)));
        o2[e] = pack_half2(make_float2(fmaf(b.x, c0.x, -a.x * c0.y), fmaf(b.y, c1.x, -a.y * c1.y)));
      }
      *reinterpret_cast<uint4*>(qpb0 + tile_off<D, ROWS>(row, c * 8)) = y1;
      *reinterpret_cast<uint4*>(qpb0 + tile_off<D, ROWS>(row, c * 8 + D / 2)) = y2;
    }
  }
  fence_proxy_async_smem();  // the MMA reads Q through the async proxy
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;

  const float sl2 = p.scale * kLog2e;

  if (w < TC_NES) {
    // ======================================================== score warps
    float m_st[NT][2], l_st[NT][2];
#pragma unroll
    for (int pt = 0; pt < NT; ++pt) {
      m_st[pt][0] = m_st[pt][1] = -INFINITY;
      l_st[pt][0] = l_st[pt][1] = 0.f;
    }
    const uint32_t tl = tmem + ((uint32_t)kb << 16);
    // per agent: the n-tile holding its query rows, and whether this lane's row is one of them
    int pa_of[3];
    bool mine[3];
#pragma unroll
    for (int a = 0; a < 3; ++a) {
      pa_of[a] = (a * g) >> 3;
      mine[a] = (8 * pa_of[a] + gq) / g == a;
    }
    for (int n = 0; n < n_tiles; ++n) {
      const int pb = n & 1;
      const uint32_t qpb = qp_u + pb * C::QP_BYTES;
      const int64_t k0 = k_lo + (int64_t)n * KT;
      const int64_t kw0 = k0 + kb;
      if (!mbar_wait(tfull, n & 1)) fail = 1;
      tc_fence_after();
      bar_sync(BAR_QP + pb, NB);

      float S[NT][4];
      {
        uint32_t r4[NT][4];
#pragma unroll
        for (int pt = 0; pt < NT; ++pt) tmem_ld16x256_x1(r4[pt], tl + TC_SCOL + 8 * pt);
        tmem_wait_ld();
#pragma unroll
        for (int pt = 0; pt < NT; ++pt)
#pragma unroll
          for (int e = 0; e < 4; ++e) S[pt][e] = __uint_as_float(r4[pt][e]);
      }
      if (kw0 < k_hi) {
        // agents outer, column groups inner; the TMEM load of the next (agent,
        // group) is in flight while the current one is turned and scored
        uint32_t xl[2][8], xh[2][8];   // delta columns i and i + d/2 of a group
        tmem_ld16x256_x2(xl[0], tl);
        tmem_ld16x256_x2(xh[0], tl + D / 2);
        for (int a = 0; a < na; ++a) {
          const int pa = a == 0 ? pa_of[0] : (a == 1 ? pa_of[1] : pa_of[2]);
          const bool mn = a == 0 ? mine[0] : (a == 1 ? mine[1] : mine[2]);
          float Sd[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int grp = 0; grp < C::NG; ++grp) {
            const int cb = grp & 1, nb = cb ^ 1;
            tmem_wait_ld_regs(xl[cb], xh[cb]);
            if (grp + 1 < C::NG) {
              const uint32_t ta = tl + 128 * a + 16 * (grp + 1);
              tmem_ld16x256_x2(xl[nb], ta);
              tmem_ld16x256_x2(xh[nb], ta + D / 2);
            } else if (a + 1 < na) {
              const uint32_t ta = tl + 128 * (a + 1);
              tmem_ld16x256_x2(xl[nb], ta);
              tmem_ld16x256_x2(xh[nb], ta + D / 2);
            }
            uint32_t A_lo[4], A_hi[4];
#pragma unroll
            for (int q = 0; q < 2; ++q)
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                // (x1, x2) = delta columns (i, i + d/2) at two adjacent i, as
                // f16 pairs; R(j) x in f16x2 arithmetic: the rotated delta is the
                // f16 A operand of the scoring MMA
                const __half2 x1 = __floats2half2_rn(__uint_as_float(xl[cb][4 * q + 2 * hh]), __uint_as_float(xl[cb][4 * q + 2 * hh + 1]));
                const __half2 x2 = __floats2half2_rn(__uint_as_float(xh[cb][4 * q + 2 * hh]), __uint_as_float(xh[cb][4 * q + 2 * hh + 1]));
                const __half2 c = *reinterpret_cast<const __half2*>(&RC[grp][hh][q]);
                const __half2 sn = *reinterpret_cast<const __half2*>(&RS[grp][hh][q]);
                const __half2 l2 = __hfma2(x1, c, __hneg2(__hmul2(x2, sn)));
                const __half2 h2 = __hfma2(x2, c, __hmul2(x1, sn));
                A_lo[2 * q + hh] = *reinterpret_cast<const uint32_t*>(&l2);
                A_hi[2 * q + hh] = *reinterpret_cast<const uint32_t*>(&h2);
              }
            uint32_t bq[4];
            ldsm_x4(bq, qpb + tile_off<D, ROWS>(8 * pa + rr, 16 * grp + (mi & 1) * 8 + (mi >> 1) * (D / 2)));
            if (!mn) bq[0] = bq[1] = bq[2] = bq[3] = 0u;
            mma16816_f16(Sd, A_lo, bq[0], bq[1]);
            mma16816_f16(Sd, A_hi, bq[2], bq[3]);
          }
#pragma unroll
          for (int pt = 0; pt < NT; ++pt)
            if (pt == pa) {
              S[pt][0] += Sd[0]; S[pt][1] += Sd[1];
              S[pt][2] += Sd[2]; S[pt][3] += Sd[3];
            }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty);  // TMEM of this tile may be overwritten

      // tile row maxima over all score warps
      const bool v0 = kw0 + gq < k_hi, v1 = kw0 + gq + 8 < k_hi;
      float x[NT][4];
#pragma unroll
      for (int pt = 0; pt < NT; ++pt) {
        x[pt][0] = v0 ? S[pt][0] * sl2 : -INFINITY;
        x[pt][1] = v0 ? S[pt][1] * sl2 : -INFINITY;
        x[pt][2] = v1 ? S[pt][2] * sl2 : -INFINITY;
        x[pt][3] = v1 ? S[pt][3] * sl2 : -INFINITY;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float mt_ = fmaxf(x[pt][e], x[pt][e + 2]);
          mt_ = fmaxf(mt_, __shfl_xor_sync(0xffffffffu, mt_, 4));
          mt_ = fmaxf(mt_, __shfl_xor_sync(0xffffffffu, mt_, 8));
          mt_ = fmaxf(mt_, __shfl_xor_sync(0xffffffffu, mt_, 16));
          if (gq == 0) Mx[(pb * ROWS + 8 * pt + 2 * t4 + e) * TC_NES + w] = mt_;
        }
      }
      bar_sync(BAR_MAX, 32 * TC_NES);
      bool moved = false;   // a running maximum of this lane's rows grew
#pragma unroll
      for (int pt = 0; pt < NT; ++pt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int row = 8 * pt + 2 * t4 + e;
          const float4 ma = *reinterpret_cast<const float4*>(Mx + (pb * ROWS + row) * TC_NES);
          const float4 mb = *reinterpret_cast<const float4*>(Mx + (pb * ROWS + row) * TC_NES + 4);
          const float mt_ = fmaxf(max3f(ma.x, ma.y, ma.z), max3f(ma.w, max3f(mb.x, mb.y, mb.z), mb.w));
          const float mo = m_st[pt][e];
          const float mn = fmaxf(mo, mt_);
          const float corr = (mo == -INFINITY) ? 0.f : fast_exp2(mo - mn);
          const float p0 = (mn == -INFINITY) ? 0.f : fast_exp2(x[pt][e] - mn);
          const float p1 = (mn == -INFINITY) ? 0.f : fast_exp2(x[pt][e + 2] - mn);
          x[pt][e] = p0;
          x[pt][e + 2] = p1;
          l_st[pt][e] = l_st[pt][e] * corr + p0 + p1;
          m_st[pt][e] = mn;
          moved |= corr != 1.f;
          if (w == 0 && gq == 0) Corr[pb * ROWS + row] = corr;
        }
      const bool any_moved = __any_sync(0xffffffffu, moved);   // over every row (the lanes' t4)
      bar_sync(BAR_PFREE + pb, NB);
      // O^T holds every tile before this one (and P buffer pb, last read by the
      // P V MMA of tile n-2, is free)
      if (n > 0 && !mbar_wait(pvdone, (n - 1) & 1)) fail = 1;
      const uint32_t pt_u = ptile_u + pb * C::P_TILE;
#pragma unroll
      for (int pt = 0; pt < NT; ++pt) {
        const uint32_t b0 = movmatrix_t(pack_bf16(x[pt][0], x[pt][1]));
        const uint32_t b1 = movmatrix_t(pack_bf16(x[pt][2], x[pt][3]));
        sts32(pt_u + tile_off<KT, ROWS>(8 * pt + gq, kb + 2 * t4), b0);
        sts32(pt_u + tile_off<KT, ROWS>(8 * pt + gq, kb + 8 + 2 * t4), b1);
      }
      bar_arrive(BAR_P + pb, NB);
      // the running maxima moved: O^T (TMEM lanes = d, columns = query rows)
      // times corr, by one warp per sub-partition
      if (n > 0 && w < 4) {
        if (any_moved) {
          tc_fence_after();
#pragma unroll
          for (int c0 = 0; c0 < QPAD; c0 += 16) {
            uint32_t ov[16];
            const uint32_t ta = tmem + TC_OCOL + c0 + ((uint32_t)(32 * w) << 16);
            tmem_ld32x32b_x16(ov, ta);
            tmem_wait_ld_r16(ov);
#pragma unroll
            for (int c = 0; c < 16; ++c)
              if (c0 + c < ROWS) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * Corr[pb * ROWS + c0 + c]);
            tmem_st32x32b_x16(ta, ov);
          }
          tmem_wait_st();
        }
      }
      fence_proxy_async_smem();  // the MMA reads P through the async proxy
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pfull);
    }
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
    if (n_tiles > 0 && !mbar_wait(pvdone, (n_tiles - 1) & 1)) fail = 1;  // O^T is complete
    tc_fence_before();
    bar_sync(BAR_END, TC_NTHR);
    float* Mo = reinterpret_cast<float*>(area);
    if (w == 0 && gq == 0) {
#pragma unroll
      for (int pt = 0; pt < NT; ++pt)
#pragma unroll
        for (int e = 0; e < 2; ++e) Mo[(8 * pt + 2 * t4 + e) * W + D + R] = m_st[pt][e];
    }
    if (w < 4) {  // O_base, this lane's d = 32 w + lane, every query row
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < QPAD; c0 += 16) {
        uint32_t ov[16];
        if (n_tiles > 0) {
          tmem_ld32x32b_x16(ov, tmem + TC_OCOL + c0 + ((uint32_t)(32 * w) << 16));
          tmem_wait_ld_r16(ov);
        } else {
#pragma unroll
          for (int c = 0; c < 16; ++c) ov[c] = 0u;
        }
#pragma unroll
        for (int c = 0; c < 16; ++c)
          if (c0 + c < ROWS) Mo[(c0 + c) * W + 32 * w + lane] = __uint_as_float(ov[c]);
      }
    }
  } else if (w < TC_NES + NPV) {
    // ======================================================== value warps
    // the next tile's rotated queries, the tail rows of a tile past the
    // sequence's end, and O_lr^T += LRv^T P^T (mma.sync; r columns)
    const int pv = w - TC_NES;
    float Olr[C::MR][NT][4];
#pragma unroll
    for (int mr = 0; mr < C::MR; ++mr)
#pragma unroll
      for (int pt = 0; pt < NT; ++pt)
#pragma unroll
        for (int e = 0; e < 4; ++e) Olr[mr][pt][e] = 0.f;
    if (n_tiles > 0) {
      bar_arrive(BAR_QP + 0, NB);
      bar_arrive(BAR_PFREE + 0, NB);
    }
    if (n_tiles > 1) bar_arrive(BAR_PFREE + 1, NB);
    const int d0 = pv * (D / 2);
    // this lane's frequency i: s (cos, sin)(k0 theta_i) of the tile being
    // rotated, advanced one tile at a time by the rotation through KT theta_i
    // in fp32 and taken exactly (fp64) again every 16 tiles
    const int qi = pv * 32 + lane;
    float2 qcs = make_float2(0.f, 0.f), qstep = qcs;
    if (qi < D / 2) {
      qcs = cs0[qi];
      qstep = rope_cs_exact(KT, theta[qi]);
    }
    for (int n = 0; n < n_tiles; ++n) {
      const int s = n % ST, pb = n & 1;
      const uint32_t sL = area_u + s * C::STAGE + 2 * C::KV_TILE;
      const int64_t k0 = k_lo + (int64_t)n * KT;
      if (n + 1 < n_tiles) {
        if (qi < D / 2) {
          if (((n + 1) & 15) == 0) {
            const float2 cs = rope_cs_exact(p.key_pos0 + k0 + KT, theta[qi]);
            qcs = make_float2(cs.x * p.s, cs.y * p.s);
          } else {
            qcs = make_float2(fmaf(qcs.x, qstep.x, -qcs.y * qstep.y), fmaf(qcs.y, qstep.x, qcs.x * qstep.y));
          }
          rotate_queries_cs<D, QPAD, ROWS>(qu_u, qp_u + ((n + 1) & 1) * C::QP_BYTES, qcs.x, qcs.y, qi);
        }
        bar_arrive(BAR_QP + ((n + 1) & 1), NB);
      }
      if (!mbar_wait(full_u + 8 * s, (n / ST) & 1)) fail = 1;
      if (k0 + KT > k_hi) {  // rows past the end: zero, so that P (0 there) meets no stale NaN
        unsigned char* vb = area + s * C::STAGE + C::KV_TILE;
        unsigned char* lb = area + s * C::STAGE + 2 * C::KV_TILE;
        const int first = (int)(k_hi - k0);
        for (int i = lane; i < (KT - first) * (D / 4); i += 32) {
          const int row = first + i / (D / 4), c = d0 + 2 * (i % (D / 4));
          *reinterpret_cast<uint32_t*>(vb + tile_off<D, KT>(row, c)) = 0u;
        }
        if (pv == 0)
          for (int al = 0; al < (PA ? na : 1); ++al)
            for (int i = lane; i < (KT - first) * (R / 2); i += 32) {
              const int row = first + i / (R / 2), c = R + 2 * (i % (R / 2));
              *reinterpret_cast<uint32_t*>(lb + al * C::LR_TILE + tile_off<2 * R, KT>(row, c)) = 0u;
            }
        fence_proxy_async_smem();  // the P V MMA reads V through the async proxy
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(pfull);
      bar_sync(BAR_P + pb, NB);
      if (pv == 0) {
#pragma unroll
        for (int pt = 0; pt < NT; ++pt) {
          const float c0 = Corr[pb * ROWS + 8 * pt + 2 * t4];
          const float c1 = Corr[pb * ROWS + 8 * pt + 2 * t4 + 1];
#pragma unroll
          for (int mr = 0; mr < C::MR; ++mr) {
            Olr[mr][pt][0] *= c0; Olr[mr][pt][2] *= c0;
            Olr[mr][pt][1] *= c1; Olr[mr][pt][3] *= c1;
          }
        }
        const uint32_t pt_u = ptile_u + pb * C::P_TILE;
#pragma unroll 2
        for (int ks = 0; ks < KT / 16; ++ks) {
          uint32_t bP[NT][2];
#pragma unroll
          for (int pt = 0; pt < NT; ++pt)
            ldsm_x2(bP[pt][0], bP[pt][1], pt_u + tile_off<KT, ROWS>(8 * pt + rr, 16 * ks + ((lane >> 3) & 1) * 8));
          if constexpr (PA) {
            // each agent's rows against its own LRv: the other agents' P
            // columns of the fragment (its query rows, n = lane / 4) are zeroed
            for (int al = 0; al < na; ++al) {
#pragma unroll
              for (int mr = 0; mr < C::MR; ++mr) {
                uint32_t aV[4];
                ldsm_x4_t(aV, sL + al * C::LR_TILE +
                                  tile_off<2 * R, KT>(16 * ks + rr + (mi >> 1) * 8, R + 16 * mr + (mi & 1) * 8));
#pragma unroll
                for (int pt = 0; pt < NT; ++pt) {
                  const bool mine = (8 * pt + gq) / g == al;
                  mma16816(Olr[mr][pt], aV, mine ? bP[pt][0] : 0u, mine ? bP[pt][1] : 0u);
                }
              }
            }
          } else {
#pragma unroll
            for (int mr = 0; mr < C::MR; ++mr) {
              uint32_t aV[4];
              ldsm_x4_t(aV, sL + tile_off<2 * R, KT>(16 * ks + rr + (mi >> 1) * 8, R + 16 * mr + (mi & 1) * 8));
#pragma unroll
              for (int pt = 0; pt < NT; ++pt) mma16816(Olr[mr][pt], aV, bP[pt][0], bP[pt][1]);
            }
          }
        }
      }
      __syncwarp();
      if (n + 2 < n_tiles) bar_arrive(BAR_PFREE + pb, NB);
      if (lane == 0) mbar_arrive(empty_u + 8 * s);
    }
    bar_sync(BAR_END, TC_NTHR);
    float* Mo = reinterpret_cast<float*>(area);
    if (pv == 0) {
#pragma unroll
      for (int pt = 0; pt < NT; ++pt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int row = 8 * pt + 2 * t4 + (e & 1);
          const int dd = gq + (e >> 1) * 8;
#pragma unroll
          for (int mr = 0; mr < C::MR; ++mr)
            if (16 * mr + dd < R) Mo[row * W + D + 16 * mr + dd] = Olr[mr][pt][e];
        }
    }
  } else {
    // ======================================================== TMA / MMA warp
    if (lane == 0) {
      constexpr uint32_t ID_S = umma_idesc_bf16(128, QPAD, 0, 0);
      constexpr uint32_t ID_E = umma_idesc_bf16(128, D, 0, 1);
      constexpr uint32_t ID_PV = umma_idesc_bf16(128, QPAD, 1, 0);   // O^T += V^T P^T, A = V MN-major
      const uint64_t dQ = umma_desc(qu_u, 16, 1024, 2);
      const uint64_t dBk = umma_desc(bks_u, R * 128, 1024, 2);
      if (n_tiles > 0 && !mbar_wait(bkbar, 0)) fail = 1;
      // the split's next tiles stream into L2 from here on (the queries and the
      // first stages were requested first), so that HBM stays busy between
      // stage refills; the window moves one tile per tile consumed
      auto prefetch = [&](int m) {
        const int key0 = (int)(k_lo + (int64_t)m * KT);
#pragma unroll
        for (int b = 0; b < D / 64; ++b) {
          tma_prefetch_l2_4d(&tmK, 64 * b, key0, kvh, seq);
          tma_prefetch_l2_4d(&tmV, 64 * b, key0, kvh, seq);
        }
        constexpr int LB = (2 * R) < 64 ? 2 * R : 64;
#pragma unroll
        for (int al = 0; al < (PA ? na : 1); ++al)
          for (int b = 0; b < (2 * R) / LB; ++b)
            tma_prefetch_l2_4d(&tmL, LB * b, key0, seq, PA ? agent0 + al : lra);
      };
      for (int m = ST; m < n_tiles && m < ST + kL2Ahead; ++m) prefetch(m);
      auto mma_pv = [&](int m) {  // O^T (d x query rows) += V_base^T P^T over the tile's keys
        const int sm = m % ST;
        if (!mbar_wait(pfull, m & 1)) fail = 1;
        tc_fence_after();
        // P^T as the K-major B operand: the P tile's ROWS rows in 64-key boxes
        // (ROWS * 128 bytes apart); with N = QPAD > ROWS the MMA also reads the
        // next rows' bytes (the next box, the next buffer or the softmax
        // scratch, all inside shared memory) into O^T columns that are never read
        const uint64_t dV = umma_desc(area_u + sm * C::STAGE + C::KV_TILE, KT * 128, 1024, 2);
        const uint64_t dP = umma_desc(ptile_u + (m & 1) * C::P_TILE, 16, 1024, 2);
#pragma unroll
        for (int kk = 0; kk < KT / 16; ++kk)
          umma_bf16(tmem + TC_OCOL, umma_desc_add(dV, kk * 16 * 128),
                    umma_desc_add(dP, (kk >> 2) * (ROWS * 128) + (kk & 3) * 32), ID_PV, (m > 0 || kk > 0) ? 1u : 0u);
        umma_commit(pvdone);
        umma_commit(empty_u + 8 * sm);  // the stage's K, LRk and V have been read
      };
      for (int n = 0; n < n_tiles; ++n) {
        const int s = n % ST;
        const uint32_t sK = area_u + s * C::STAGE;
        const uint32_t sL = sK + 2 * C::KV_TILE;
        if (!mbar_wait(full_u + 8 * s, (n / ST) & 1)) fail = 1;
        if (n > 0 && !mbar_wait(tempty, (n - 1) & 1)) fail = 1;
        tc_fence_after();
        // base scores for every agent's rows: S_base^T = K_base Q^T
        const uint64_t dK = umma_desc(sK, 16, 1024, 2);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_bf16(tmem + TC_SCOL, umma_desc_add(dK, (kk >> 2) * (KT * 128) + (kk & 3) * 32),
                    umma_desc_add(dQ, (kk >> 2) * (QPAD * 128) + (kk & 3) * 32), ID_S, kk > 0);
        // key deltas dK^a = LRk B_k^a (B_k^a stored r-major: the MN-major operand)
        const uint64_t dL = umma_desc(sL, 16, 8 * C::LR_ROWB, C::LR_LAYOUT);
        for (int a = 0; a < na; ++a) {
          const uint64_t dB = umma_desc_add(dBk, a * align1k(C::BK_BYTES));
          const uint64_t dLa = PA ? umma_desc_add(dL, a * C::LR_TILE) : dL;
#pragma unroll
          for (int ks = 0; ks < C::KS; ++ks)
            umma_bf16(tmem + 128 * a, umma_desc_add(dLa, ks * 32), umma_desc_add(dB, ks * 16 * 128), ID_E, ks > 0);
        }
        umma_commit(tfull);
        if (n > 0) mma_pv(n - 1);
        if (n >= 1 && n - 1 + ST < n_tiles) {
          const int sp = (n - 1) % ST;
          if (!mbar_wait(empty_u + 8 * sp, ((n - 1) / ST) & 1)) fail = 1;
          issue(n - 1 + ST);
          if (n - 1 + ST + kL2Ahead < n_tiles) prefetch(n - 1 + ST + kL2Ahead);
        }
      }
      if (n_tiles > 0) mma_pv(n_tiles - 1);
      for (int n = n_tiles; n < n_spec; ++n)  // loaded ahead of kv_len and not used
        if (!mbar_wait(full_u + 8 * n, 0)) fail = 1;
    }
    __syncwarp();
    bar_sync(BAR_END, TC_NTHR);
  }
  if (fail) s_fail = 1;
  if (!mbar_wait(bkbar, 0)) s_fail = 1;
  __syncthreads();
  if (w == TC_NES + NPV) {
    tc_fence_after();
    tmem_dealloc(tmem, TC_COLS);
  }
  float* Mo = reinterpret_cast<float*>(area);
  for (int row = tid; row < n_rows; row += TC_NTHR) {
    float l = 0.f;
#pragma unroll
    for (int ww = 0; ww < TC_NES; ++ww) l += Lw[ww * ROWS + row];
    Mo[row * W + D + R + 1] = l;
  }
  if (ns == 1) {  // Z = O_base + s O_lr B_v^a (with split keys the merge applies B_v^a once)
    const __nv_bfloat16* bv = reinterpret_cast<const __nv_bfloat16*>(p.B_v) + (int64_t)agent0 * R * ldB + kvh * D;
    for (int i = tid; i < n_rows * (D / 4); i += TC_NTHR) {
      const int row = i / (D / 4), c = 4 * (i % (D / 4));
      const __nv_bfloat16* b = bv + (size_t)(row / g) * R * ldB + c;
      float z0 = 0.f, z1 = 0.f, z2 = 0.f, z3 = 0.f;
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const float o = Mo[row * W + D + j];
        const uint2 bb = __ldg(reinterpret_cast<const uint2*>(b + j * ldB));
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
  if (s_fail && tid == 0) atomicOr(p.err, 2);
  if (ns == 1) {
    if (s_fail) return;
    if (p.row_stats)   // (M, L) of every row, for the combine of a sequence-sharded decode
      for (int row = tid; row < n_rows; row += TC_NTHR) {
        const int64_t ri = ((int64_t)seq * na_tot + agent0 + row / g) * p.n_q + kvh * g + row % g;
        reinterpret_cast<float2*>(p.row_stats)[ri] = make_float2(Mo[row * W + D + R], Mo[row * W + D + R + 1]);
      }
    for (int i = tid; i < n_rows * D; i += TC_NTHR) {
      const int row = i / D, c = i % D;
      const int a = row / g, gi = row % g;
      const float l = Mo[row * W + D + R + 1];
      const float val = l > 0.f ? Mo[row * W + c] / l : 0.f;
      const int64_t oi = (((int64_t)seq * na_tot + agent0 + a) * p.n_q + kvh * g + gi) * D + c;
      if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(val);
      else reinterpret_cast<float*>(p.out)[oi] = val;
    }
    return;
  }
  // ---- split merge, shared by the unit's CTAs.  Each writes its partial
  // (O_base, O_lr, m, l) to the workspace, waits until every split of the unit
  // has (the launch is cooperative, so all CTAs are resident; the wait is
  // bounded), then produces one contiguous share of the unit's output:
  //   w_k = 2^(m_k - M) / sum_k 2^(m_k - M) l_k,  M = max_k m_k,
  //   out = sum_k w_k O_base,k + s (sum_k w_k O_lr,k) B_v^a,
  // B_v^a applied once per row (it is linear, so it commutes with the merge).
  // A CTA that failed still arrives, so the others never wait for it.
  float* ws_unit = p.partials + (size_t)unitg * ns * (p.agent_group * g) * W;
  {
    float* part = ws_unit + (size_t)split * n_rows * W;
    for (int i = tid; i < n_rows * (W / 4); i += TC_NTHR)
      reinterpret_cast<float4*>(part)[i] = reinterpret_cast<const float4*>(Mo)[i];
  }
  int* arrive = p.counters + unitg;
  int* depart = p.counters + gridDim.y * (p.n_seqs * p.n_kv) + unitg;
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    atomicAdd(arrive, 1);
    int it = 0;
    while (ld_acquire_gpu(arrive) < ns) {
      if (++it > (1 << 22)) {
        atomicOr(p.err, 4);
        break;
      }
      __nanosleep(32);
    }
    __threadfence();
  }
  __syncthreads();
  constexpr int CH = D / 4;                        // float4 chunks per output row
  const int n_items = n_rows * CH;
  const int ib = (int)((int64_t)split * n_items / ns), ie = (int)((int64_t)(split + 1) * n_items / ns);
  const int ni = ie - ib;
  const int rb = ib / CH, nr = ni > 0 ? (ie - 1) / CH + 1 - rb : 0;
  const int ks = ni > 0 ? max(1, TC_NTHR / ni) : 1;   // subsets of the splits per item
  float* Wf = Mo;                                  // [nr][kMaxSplits] weights
  float* Ol = Wf + nr * kMaxSplits;                // [nr][R] merged O_lr
  float* T = Ol + nr * R;                          // [nr][ns][R] w_k O_lr,k
  float4* red = reinterpret_cast<float4*>(T + ((nr * ns * R + 3) & ~3));  // [ks][ni]
  auto part_at = [&](int k, int row, int c) {
    return reinterpret_cast<const float4*>(ws_unit + ((size_t)k * n_rows + row) * W + c);
  };
  // (a) this thread's partial loads, issued before the weights are known
  float4 v[2][4];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int u = tid + h * TC_NTHR;
    const int item = ib + u % max(ni, 1), sub = u / max(ni, 1);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int k = sub + j * ks;
      v[h][j] = (u < ni * ks && k < ns) ? __ldcg(part_at(k, item / CH, 4 * (item % CH)))
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  // (b) per row, one warp: lane k holds split k's (m, l) and O_lr
  for (int r = w; r < nr; r += TC_NTHR / 32) {
    const int row = rb + r;
    float2 ml = make_float2(-INFINITY, 0.f);
    float4 ol[R / 4];
    if (lane < ns) {
      ml = __ldcg(reinterpret_cast<const float2*>(ws_unit + ((size_t)lane * n_rows + row) * W + D + R));
#pragma unroll
      for (int j = 0; j < R / 4; ++j) ol[j] = __ldcg(part_at(lane, row, D + 4 * j));
    }
    float mx = ml.x;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    const float e = (lane < ns && ml.x != -INFINITY) ? fast_exp2(ml.x - mx) : 0.f;
    float lt = e * ml.y;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lt += __shfl_xor_sync(0xffffffffu, lt, o);
    const float wk = lt > 0.f ? e / lt : 0.f;
    if (p.row_stats && lane == 0) {   // (M, L) of the row over all its splits
      const int64_t ri = ((int64_t)seq * na_tot + agent0 + row / g) * p.n_q + kvh * g + row % g;
      reinterpret_cast<float2*>(p.row_stats)[ri] = make_float2(mx, lt);
    }
    if (lane < ns) {
      Wf[r * kMaxSplits + lane] = wk;
      float4* tr = reinterpret_cast<float4*>(T + ((size_t)r * ns + lane) * R);
#pragma unroll
      for (int j = 0; j < R / 4; ++j)
        tr[j] = make_float4(wk * ol[j].x, wk * ol[j].y, wk * ol[j].z, wk * ol[j].w);
    }
  }
  __syncthreads();
  // (c) merged O_lr per row; (d) weighted sums of this thread's loads
  for (int i = tid; i < nr * R; i += TC_NTHR) {
    const int r = i / R, j = i % R;
    float acc = 0.f;
    for (int k = 0; k < ns; ++k) acc += T[((size_t)r * ns + k) * R + j];
    Ol[i] = acc;
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int u = tid + h * TC_NTHR;
    if (u < ni * ks) {
      const int item = ib + u % ni, sub = u / ni;
      const int row = item / CH, c = 4 * (item % CH);
      const float* wr = Wf + (row - rb) * kMaxSplits;
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int k = sub + j * ks;
        const float wk = k < ns ? wr[k] : 0.f;
        acc.x = fmaf(wk, v[h][j].x, acc.x); acc.y = fmaf(wk, v[h][j].y, acc.y);
        acc.z = fmaf(wk, v[h][j].z, acc.z); acc.w = fmaf(wk, v[h][j].w, acc.w);
      }
      for (int k = sub + 4 * ks; k < ns; k += ks) {  // more splits than four per subset
        const float4 x = __ldcg(part_at(k, row, c));
        acc.x = fmaf(wr[k], x.x, acc.x); acc.y = fmaf(wr[k], x.y, acc.y);
        acc.z = fmaf(wr[k], x.z, acc.z); acc.w = fmaf(wr[k], x.w, acc.w);
      }
      red[u] = acc;
    }
  }
  __syncthreads();
  // (e) out = sum over subsets + s O_lr B_v^a
  {
    const __nv_bfloat16* bv = reinterpret_cast<const __nv_bfloat16*>(p.B_v) + (int64_t)agent0 * R * ldB + kvh * D;
    for (int i = tid; i < ni; i += TC_NTHR) {
      float4 acc = red[i];
      for (int sub = 1; sub < ks; ++sub) {
        const float4 x = red[sub * ni + i];
        acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
      }
      const int item = ib + i, row = item / CH, c = 4 * (item % CH);
      const int a = row / g, gi = row % g;
      const float* ol = Ol + (row - rb) * R;
      const __nv_bfloat16* bb = bv + (size_t)a * R * ldB + c;
      float z0 = 0.f, z1 = 0.f, z2 = 0.f, z3 = 0.f;
#pragma unroll
      for (int j = 0; j < R; ++j) {
        const float o = ol[j];
        const uint2 b2 = __ldg(reinterpret_cast<const uint2*>(bb + j * ldB));
        const float2 f01 = unpack_bf16(b2.x), f23 = unpack_bf16(b2.y);
        z0 = fmaf(o, f01.x, z0); z1 = fmaf(o, f01.y, z1);
        z2 = fmaf(o, f23.x, z2); z3 = fmaf(o, f23.y, z3);
      }
      acc.x = fmaf(p.s, z0, acc.x); acc.y = fmaf(p.s, z1, acc.y);
      acc.z = fmaf(p.s, z2, acc.z); acc.w = fmaf(p.s, z3, acc.w);
      const int64_t oi = (((int64_t)seq * na_tot + agent0 + a) * p.n_q + kvh * g + gi) * D + c;
      if (p.out_bf16) {
        uint2 o;
        o.x = pack_bf16(acc.x, acc.y);
        o.y = pack_bf16(acc.z, acc.w);
        *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p.out) + oi) = o;
      } else {
        *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + oi) = acc;
      }
    }
  }
  // the last CTA to leave resets the unit's counters for the next call
  __syncthreads();
  if (tid == 0 && atomicAdd(depart, 1) == ns - 1) {
    *arrive = 0;
    *depart = 0;
    __threadfence();
  }
}

// -------------------------------------------------------------------- host
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
  // LR caches [n_lr][n_seqs][L_max][2r]: one shared cache, or one per agent
  const int lb = 2 * R < 64 ? 2 * R : 64;
  const int64_t n_lr = p.lr_agent ? p.n_agents : 1;
  const int64_t lr_agent_b = p.lr_agent ? p.lr_agent * 2 : p.lr_seq * 2 * p.n_seqs;
  cuuint64_t ldims[4] = {(cuuint64_t)(2 * R), (cuuint64_t)p.L_max, (cuuint64_t)p.n_seqs, (cuuint64_t)n_lr};
  cuuint64_t lstr[3] = {(cuuint64_t)(2 * R * 2), (cuuint64_t)p.lr_seq * 2, (cuuint64_t)lr_agent_b};
  cuuint32_t lbox[4] = {(cuuint32_t)lb, (cuuint32_t)KT, 1, 1};
  if (enc(ml, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(p.lr), ldims, lstr, lbox, one,
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
// SMs of the current device (148 on B200; also the answer when no device is
// visible, so that workspace sizes can be planned on a host without a GPU)
int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
    cudaGetLastError();
    return kSMs;
  }
  return n;
}

bool tc_fits(const AttnParams& p, int G);
int tc_group_size(const AttnParams& p);

// agent groups of the tensor-core decode (each CTA holds one group), else 1
int decode_groups(const AttnParams& p) {
  const int G = tc_group_size(p);
  return G > 0 ? (p.n_agents + G - 1) / G : 1;
}

// splits of each (sequence, KV head, agent group) over the keys: enough CTAs
// to cover the SMs once (one CTA per SM), so that a split launch is always
// fully resident
int n_splits_for(const AttnParams& p) {
  const int units = p.n_seqs * p.n_kv * decode_groups(p);
  if (units < 1) return 1;   // an empty batch
  const int64_t total_tiles = (p.max_kv_len + KT - 1) / KT;
  const int sms = device_sms();
  int64_t ns = units >= sms ? 1 : sms / units;
  if (ns > kMaxSplits) ns = kMaxSplits;
  if (ns > total_tiles) ns = total_tiles;
  if (ns < 1) ns = 1;
  // as few splits as give the same longest split: the split with the most tiles
  // sets the time, fewer splits mean less to merge
  const int64_t per = (total_tiles + ns - 1) / ns;
  ns = (total_tiles + per - 1) / per;
  return (int)ns;
}

template <int D, int R, int NT>
cudaError_t launch_t(const AttnParams& p, cudaStream_t st) {
  using C = Cfg<D, R, NT>;
  RopeTheta rt;
  for (int i = 0; i < 64; ++i) {
    rt.theta[i] = i < D / 2 ? std::pow(p.rope_base, -2.0 * i / D) : 0.0;
    rt.thetaf[i] = (float)rt.theta[i];
  }
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

// the tensor-core decode with G agents per CTA: TMEM holds G key deltas of
// 128 columns and the scores; rows G g in at most three m16 row tiles; shared
// memory within 227 KB
bool tc_fits(const AttnParams& p, int G) {
  if (G < 1 || G > 3) return false;
  const int NT = (G * p.g + 7) / 8;
  if (NT > 3) return false;
  size_t sm = 0;
  if (p.lr_agent && G > 1) {   // per-agent LR tiles in every stage: r = 16 only
    if (p.r != 16) return false;
    sm = NT == 1 ? TCfg<128, 16, 1, true>::smem(G) : NT == 2 ? TCfg<128, 16, 2, true>::smem(G)
                                                    : TCfg<128, 16, 3, true>::smem(G);
    return sm <= 227 * 1024;
  }
  switch (p.r) {
    case 16: sm = NT == 1 ? TCfg<128, 16, 1>::smem(G) : NT == 2 ? TCfg<128, 16, 2>::smem(G) : TCfg<128, 16, 3>::smem(G); break;
    case 32: sm = NT == 1 ? TCfg<128, 32, 1>::smem(G) : NT == 2 ? TCfg<128, 32, 2>::smem(G) : TCfg<128, 32, 3>::smem(G); break;
    default: sm = NT == 1 ? TCfg<128, 64, 1>::smem(G) : NT == 2 ? TCfg<128, 64, 2>::smem(G) : TCfg<128, 64, 3>::smem(G); break;
  }
  return sm <= 227 * 1024;
}

// agents per CTA of the tensor-core decode (0: the shape does not run on it).
// The largest group that fits: more agents per CTA read the shared caches
// fewer times; the groups of a launch run side by side, so a cache tile read
// by one group is mostly an L2 hit for the others.
int tc_group_size(const AttnParams& p) {
  if (p.d != 128 || !(p.r == 16 || p.r == 32 || p.r == 64)) return 0;
  if (!(p.g == 1 || p.g == 2 || p.g == 4 || p.g == 8)) return 0;
  if (p.L_max >= (1ll << 31)) return 0;
  // with one LR cache per agent every stage holds each agent's LR tile: up to
  // three agents a CTA at r = 16 (shared memory), one at r = 32 and 64
  const int gmax = p.lr_agent && p.r != 16 ? 1 : 3;
  for (int G = p.n_agents < gmax ? p.n_agents : gmax; G >= 1; --G)
    if (tc_fits(p, G)) return G;
  return 0;
}

bool tc_supported(const AttnParams& p) { return tc_group_size(p) > 0; }

template <int D, int R, int NT, bool PA = false>
cudaError_t launch_tc(const AttnParams& p, cudaStream_t st) {
  using C = TCfg<D, R, NT, PA>;
  RopeTheta rt;
  for (int i = 0; i < 64; ++i) {
    rt.theta[i] = i < D / 2 ? std::pow(p.rope_base, -2.0 * i / D) : 0.0;
    rt.thetaf[i] = (float)rt.theta[i];
  }
  CUtensorMap mk, mv, ml, mb;
  if (!make_maps(p, &mk, &mv, &ml)) return cudaErrorInvalidValue;
  {
    // B_k as (n_kv*d, r, n_agents): a CTA loads its head's r x 64 slices
    cuuint64_t dims[3] = {(cuuint64_t)p.n_kv * D, (cuuint64_t)R, (cuuint64_t)p.n_agents};
    cuuint64_t str[2] = {(cuuint64_t)p.n_kv * D * 2, (cuuint64_t)R * p.n_kv * D * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)R, 1};
    cuuint32_t one[3] = {1, 1, 1};
    if (encode_fn()(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(p.B_k), dims, str, box,
                    one, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const size_t sm = C::smem(p.agent_group);
  auto kern = decode_tc_kernel<D, R, NT, PA>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_splits, (p.n_agents + p.agent_group - 1) / p.agent_group, p.n_seqs * p.n_kv);
  // with split keys the unit's CTAs wait for one another: all must be resident
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(TC_NTHR);
  cfg.dynamicSmemBytes = sm;
  cfg.stream = st;
  // the set-up may overlap the preceding kernel (programmatic dependent
  // launch; the kernel waits for it before reading any input)
  cudaLaunchAttribute attr[2];
  int na = 0;
  attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[na++].val.programmaticStreamSerializationAllowed = 1;
  if (p.n_splits > 1) {
    attr[na].id = cudaLaunchAttributeCooperative;
    attr[na++].val.cooperative = 1;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  e = cudaLaunchKernelEx(&cfg, kern, mk, mv, ml, mb, p, rt);
  if (e != cudaSuccess) {  // without the overlap where the runtime refuses the pair of attributes
    cudaGetLastError();
    cfg.attrs = attr + 1;
    cfg.numAttrs = na - 1;
    e = cudaLaunchKernelEx(&cfg, kern, mk, mv, ml, mb, p, rt);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace

bool bf16_decode_uses_tc(const AttnParams& p) { return tc_supported(p); }

bool bf16_decode_supported(const AttnParams& p) {
  if (tc_supported(p)) return true;
  if (p.lr_agent) return false;   // the generic kernel serves per-agent LR caches otherwise
  if (p.d != 128) return false;
  if (!(p.g == 1 || p.g == 2 || p.g == 4 || p.g == 8)) return false;
  const int NT = n_rowtiles(p);
  if (NT > 3) return false;
  if (NT == 3 && p.r == 64) return false;
  if (p.L_max >= (1ll << 31)) return false;
  if (smem_for(p) > 227 * 1024) return false;
  return true;
}

void bf16_decode_plan(const AttnParams& p, int* n_splits, int64_t* split_len, int* rows, int* groups) {
  const int G = tc_group_size(p);
  *n_splits = n_splits_for(p);
  *split_len = KT;
  *rows = (G > 0 ? G : p.n_agents) * p.g;
  *groups = decode_groups(p);
}

size_t bf16_decode_partial_bytes(const AttnParams& p) {
  const int ns = n_splits_for(p);
  if (ns == 1) return 0;
  const int G = tc_group_size(p);
  const int rows = (G > 0 ? G : p.n_agents) * p.g;
  return (size_t)p.n_seqs * p.n_kv * decode_groups(p) * ns * rows * (p.d + p.r + 4) * sizeof(float);
}

// arrival counters (and flags) of the split merge, in ints, per workspace
size_t bf16_decode_counter_ints(const AttnParams& p) {
  return (size_t)2 * p.n_seqs * p.n_kv * decode_groups(p);
}

cudaError_t launch_decode_bf16(const AttnParams& pin, la_dtype out, cudaStream_t st) {
  AttnParams p = pin;
  p.out_bf16 = out == LA_BF16;
  p.agent_group = tc_group_size(p);
  if (p.agent_group > 0) {
    const int NT = (p.agent_group * p.g + 7) / 8;
    if (p.lr_agent && p.agent_group > 1)   // r = 16 (tc_fits)
      return NT == 1 ? launch_tc<128, 16, 1, true>(p, st) : NT == 2 ? launch_tc<128, 16, 2, true>(p, st)
                                                         : launch_tc<128, 16, 3, true>(p, st);
    switch (p.r) {
      case 16: return NT == 1 ? launch_tc<128, 16, 1>(p, st) : NT == 2 ? launch_tc<128, 16, 2>(p, st) : launch_tc<128, 16, 3>(p, st);
      case 32: return NT == 1 ? launch_tc<128, 32, 1>(p, st) : NT == 2 ? launch_tc<128, 32, 2>(p, st) : launch_tc<128, 32, 3>(p, st);
      default: return NT == 1 ? launch_tc<128, 64, 1>(p, st) : NT == 2 ? launch_tc<128, 64, 2>(p, st) : launch_tc<128, 64, 3>(p, st);
    }
  }
  const int NT = n_rowtiles(p);
  switch (p.r) {
    case 8: return NT == 1 ? launch_t<128, 8, 1>(p, st) : NT == 2 ? launch_t<128, 8, 2>(p, st) : launch_t<128, 8, 3>(p, st);
    case 16: return NT == 1 ? launch_t<128, 16, 1>(p, st) : NT == 2 ? launch_t<128, 16, 2>(p, st) : launch_t<128, 16, 3>(p, st);
    case 32: return NT == 1 ? launch_t<128, 32, 1>(p, st) : NT == 2 ? launch_t<128, 32, 2>(p, st) : launch_t<128, 32, 3>(p, st);
    default: return NT == 1 ? launch_t<128, 64, 1>(p, st) : launch_t<128, 64, 2>(p, st);
  }
}

}  // namespace la
