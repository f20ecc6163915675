// Flash-LoRA-Attention decode with the key-side LoRA scored on the tensor
// cores through a cos/sin table (bf16 storage, fp32 accumulate).
//
// The key of agent a at position t is K^a_t = K_base,t + RoPE_t(s LRk_t B_k^a)
// (LRAgent summary App. D.1: the delta is rebuilt in head dimension because
// RoPE blocks the reordering on the key side).  RoPE pairs element i with
// i + d/2 and turns the pair by t theta_i, so for a query row q the delta's
// share of the score is
//   q . RoPE_t(s LRk_t B) = sum_rho LRk_t[rho] W[t, rho],
//   W[t, rho] = sum_{i < d/2} cos(t theta_i) U[rho, i] + sin(t theta_i) V[rho, i],
//   U[rho, i] = s (q_i B[rho, i] + q_{i+d/2} B[rho, i+d/2]),
//   V[rho, i] = s (q_{i+d/2} B[rho, i] - q_i B[rho, i+d/2]).
// U and V depend on the row's query and its agent's B_k^a only, so a CTA
// builds them once ([U | V] is the d-deep B operand, one row per (query row,
// rho)), and per 128-key tile the tensor cores compute W = CS UV^T from the
// tile's table CS[j] = [cos | sin]((k0 + j) theta) (A operand, in TMEM).  What
// is left on the CUDA cores per key is an r-wide dot with LRk_t; no key delta
// is rotated element by element.
//
// One CTA = one (sequence, KV head, agent group, key split).  Its rows are the
// group's agents x the GQA group's query heads, so every base and LR tile
// crosses HBM once for all of them (LRAgent summary §3 BaseLRShared).
//  * warp 9 (one thread) issues per tile S = K_base Q^T and W = CS UV^T, and
//    for the previous tile O^T += V_base^T P^T (tcgen05, fp32 in TMEM);
//  * warps 0-7 (key j = 32 (w % 4) + lane, half w / 4 of the rows) add the
//    r-wide dots to S, run the online softmax and write P (bf16); two tiles
//    ahead they also write the table CS into TMEM (two buffers):
//    (cos, sin)((k0 + j) theta) from the exact (cos, sin)(k0 theta) (angle
//    reduced in fp64) and (cos, sin)(j theta), a per-lane table kept in TMEM;
//  * warp 8 keeps the value side reordered (LRAgent explainer, Metodologia 3;
//    summary App. B): O_lr^T += LRv^T P^T stays r wide (mma.sync); it also
//    streams K_base, V_base and the LR rows of each tile by TMA into a
//    two-stage ring, with a window of later tiles requested into L2.
// The softmax rescales lazily: a row's reference maximum moves only when a
// tile's maximum passes it by more than 2^8, so O and O_lr are rescaled only
// then; out = O / l holds for any reference.
// Splits of the keys merge in the same launch without waiting: each CTA takes
// a ticket when its partial (O_base, O_lr, m, l) is ready; all but the last
// publish it and leave, and the last one merges them all,
//   w_k = 2^(m_k - M) / sum_k 2^(m_k - M) l_k,
//   out = sum_k w_k O_base,k + s (sum_k w_k O_lr,k) B_v^a,
// B_v^a applied once per row.  No CTA waits for one that has not arrived, so
// the launch needs no co-residency and may run in several waves.
#include <cudaTypedefs.h>

#include <cmath>

#include "bf16_common.cuh"
#include "la_internal.cuh"
#include "ptx.cuh"

namespace la {
namespace {

using namespace ptx;

constexpr int KT = 128;            // keys per tile
constexpr int ST = 2;              // pipeline stages
constexpr int D = 128;             // head_dim
constexpr int QP = 16;             // padded query rows: N of S and of P V
constexpr int NSW = 8;             // score warps
constexpr int WV = 8, WM = 9;
constexpr int NTHR = 32 * 10;
constexpr int kL2Ahead = 4;        // tiles requested into L2 ahead of the stage loads
constexpr int kMaxSplits = 16;    // splits of a unit: one cluster (16: non-portable size)
constexpr int kSMs = 148;

// TMEM columns: W (at most 192), the two CS buffers (64 each, bf16 pairs),
// the (cos, sin)(j theta) table (fp32: per half of the frequencies 32 cos,
// then 32 sin), S, O^T
constexpr uint32_t T_W = 0, T_CS = 192, T_CSJ = 320, T_S = 448, T_O = 464, T_COLS = 512;

// barriers (mbarrier slots)
enum { B_FULL = 0, B_EMPTY = ST, B_TFULL = 2 * ST, B_WFREE, B_CSFULL, B_CSFULL1, B_PFULL, B_PFREE,
       B_ODONE, B_PATCH, B_OPS, B_NUM };

template <int R, int RP>
struct Cfg {
  static constexpr int NW = RP * R;                     // W columns: (row, rho)
  static constexpr int RH = RP / 2;                     // rows per score-warp half
  static constexpr int KV_TILE = KT * D * 2;            // a K or V tile: 2 boxes of 64 d
  static constexpr int LB = 2 * R < 64 ? 2 * R : 64;     // LR box columns
  static constexpr int LR_TILE = align1k(KT * 2 * R * 2);
  static constexpr int STAGE = 2 * KV_TILE + LR_TILE;
  static constexpr int UV_BYTES = align1k(NW * D * 2);
  static constexpr int Q_BYTES = align1k(QP * D * 2);
  static constexpr int P_BYTES = align1k(QP * KT * 2);
  static constexpr int WP = D + R + 4;                  // partial row: O | O_lr | m | l | pad
  static constexpr int MR = R / 16;                     // m16 tiles of O_lr^T
  // small area: Mx [2][8][4] f32, Corr [2][QP] f32, cs0 [4][64] f32x2,
  // Lsum [QP][4] f32, Mfin [QP] f32, theta [64] f64, barriers, slots
  static constexpr int SMALL = 2 * 8 * 4 * 4 + 2 * QP * 4 + 4 * 64 * 8 + QP * 4 * 4 + QP * 4 + 64 * 8 +
                               B_NUM * 8 + 64 + 64 + 16 + 10 * 2 * R * 4 + 2 * R * 2;
  static constexpr size_t smem() {
    return 1024 + (size_t)ST * STAGE + UV_BYTES + Q_BYTES + P_BYTES + align1k(SMALL);
  }
  static_assert(NW <= 192, "W is one MMA of N <= 192 (TMEM columns 0..191)");
  static_assert(RP % 4 == 0 && RP <= QP, "rows");
  // after the loop the UV area holds the CTA's partial (read by the cluster)
  static_assert((size_t)RP * WP * 4 <= (size_t)UV_BYTES, "partial area");
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ int ld_acquire(const int* p) { return ld_acquire_gpu(p); }

template <int R, int RP>
__global__ void __launch_bounds__(NTHR, 1)
    decode_cs_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmL, const __grid_constant__ CUtensorMap tmB,
                     const AttnParams p, const __grid_constant__ RopeTheta rt) {
  using C = Cfg<R, RP>;
  constexpr int NW = C::NW, RH = C::RH, WP = C::WP;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* stages = smem;
  unsigned char* uv = stages + ST * C::STAGE;
  unsigned char* qop = uv + C::UV_BYTES;
  unsigned char* pbuf = qop + C::Q_BYTES;
  float* Mx = reinterpret_cast<float*>(pbuf + C::P_BYTES);   // [2 halves][8 rows][4 sub-partitions]
  float* Corr = Mx + 2 * 8 * 4;                                // [2][QP]
  float2* cs0 = reinterpret_cast<float2*>(Corr + 2 * QP);      // [4][64]: (cos, sin)(k0 theta_i)
  float* Lsum = reinterpret_cast<float*>(cs0 + 4 * 64);        // [QP][4]
  float* Mfin = Lsum + QP * 4;                                 // [QP]
  double* theta = reinterpret_cast<double*>(Mfin + QP);        // [64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(theta + 64);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + B_NUM);
  int* s_misc = reinterpret_cast<int*>(tslot + 2);             // [0] fail, [1] ticket
  float* red = reinterpret_cast<float*>(                        // [10 warps][2R]: the new LR row's sums
      (reinterpret_cast<uintptr_t>(s_misc + 16) + 15) & ~uintptr_t(15));
  __nv_bfloat16* newrow = reinterpret_cast<__nv_bfloat16*>(red + 10 * 2 * R);   // [2R]
  float* Part = reinterpret_cast<float*>(uv);                  // [RP][WP], after the last MMA

  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int unit = blockIdx.z;
  const int seq = unit / p.n_kv, kvh = unit % p.n_kv;
  const int split = blockIdx.x, ns = p.n_splits;
  const int agent0 = blockIdx.y * p.agent_group;
  const int g = p.g, na = min(p.agent_group, p.n_agents - agent0), n_rows = na * g;
  const int na_tot = p.n_agents;
  const int lra = p.lr_agent ? agent0 : 0;   // one LR cache per agent: one agent per CTA
  const int unitg = blockIdx.y * (p.n_seqs * p.n_kv) + unit;
  const int n_units_g = gridDim.y * p.n_seqs * p.n_kv;

  const int64_t total_tiles = (p.max_kv_len + KT - 1) / KT;
  const int64_t tb = split * total_tiles / ns;
  const int64_t te = (split + 1) * total_tiles / ns;
  const int64_t k_lo = tb * KT;
  const int n_spec = (int)min((int64_t)ST, te - tb);

  const uint32_t st_u = smem_u32(stages);
  const uint32_t uv_u = smem_u32(uv);
  const uint32_t q_u = smem_u32(qop);
  const uint32_t p_u = smem_u32(pbuf);
  const uint32_t bar_u = smem_u32(bars);
  auto bar = [&](int i) { return bar_u + 8u * (uint32_t)i; };
  const int64_t ldB = (int64_t)p.n_kv * D;

  auto issue = [&](int n) {  // TMA of tile n into stage n % ST (one thread)
    const int s = n % ST;
    const uint32_t sb = st_u + s * C::STAGE;
    const int key0 = (int)(k_lo + (int64_t)n * KT);
    mbar_expect_tx(bar(B_FULL + s), 2 * C::KV_TILE + KT * 2 * R * 2);
#pragma unroll
    for (int b = 0; b < D / 64; ++b) {
      tma_load_4d(sb + b * KT * 128, &tmK, bar(B_FULL + s), 64 * b, key0, kvh, seq);
      tma_load_4d(sb + C::KV_TILE + b * KT * 128, &tmV, bar(B_FULL + s), 64 * b, key0, kvh, seq);
    }
#pragma unroll
    for (int b = 0; b < (2 * R) / C::LB; ++b)
      tma_load_4d(sb + 2 * C::KV_TILE + b * KT * C::LB * 2, &tmL, bar(B_FULL + s), C::LB * b, key0, seq, lra);
  };
  auto prefetch = [&](int n) {  // tile n into L2 only
    const int key0 = (int)(k_lo + (int64_t)n * KT);
#pragma unroll
    for (int b = 0; b < D / 64; ++b) {
      tma_prefetch_l2_4d(&tmK, 64 * b, key0, kvh, seq);
      tma_prefetch_l2_4d(&tmV, 64 * b, key0, kvh, seq);
    }
#pragma unroll
    for (int b = 0; b < (2 * R) / C::LB; ++b) tma_prefetch_l2_4d(&tmL, C::LB * b, key0, seq, lra);
  };

  // ---- barriers, then the first tiles (by max_kv_len: independent of kv_len)
  if (w == WV && lane == 0) {
    s_misc[0] = 0;
    for (int s = 0; s < ST; ++s) {
      mbar_init(bar(B_FULL + s), 1);
      mbar_init(bar(B_EMPTY + s), 2);      // the P V MMA's commit + the value warp
    }
    mbar_init(bar(B_TFULL), 1);
    mbar_init(bar(B_WFREE), NSW);
    mbar_init(bar(B_CSFULL), NSW);
    mbar_init(bar(B_CSFULL1), NSW);
    mbar_init(bar(B_PFULL), NSW + 1);
    mbar_init(bar(B_PFREE), 2);
    mbar_init(bar(B_ODONE), 1);
    mbar_init(bar(B_PATCH), 1);
    mbar_init(bar(B_OPS), 1);
    fence_mbar_init();
    tma_prefetch(&tmK);
    tma_prefetch(&tmV);
    tma_prefetch(&tmL);
    tma_prefetch(&tmB);
  }
  if (tid < D / 2) theta[tid] = rt.theta[tid];
  if (tid < 2 * QP) Corr[tid] = 1.f;
  // the barriers are initialised before any thread polls one: the shared
  // memory still holds what the SM's previous CTA left there, and a stale
  // barrier word may read as a completed phase
  __syncthreads();
  if (w == WV && lane == 0) {
    // a programmatic dependent of the preceding kernel (the step's LR append):
    // everything above overlaps its tail, every input is read after the wait
    pdl_wait();
    // the queries (rows a g + gi, unswizzled, into the P buffer) and the B_k^a
    // head slices (per agent R rows x two 64-column boxes, 128-byte swizzle,
    // into the [U | V] area) before the tiles, so that these few kilobytes do
    // not queue behind the tiles' megabytes
    const __nv_bfloat16* Q = reinterpret_cast<const __nv_bfloat16*>(p.q);
    mbar_expect_tx(bar(B_OPS), (uint32_t)(na * g * D * 2 + na * R * D * 2));
    for (int a = 0; a < na; ++a)
      bulk_load(p_u + a * g * D * 2, Q + (((int64_t)seq * na_tot + agent0 + a) * p.n_q + kvh * g) * D,
                (uint32_t)(g * D * 2), bar(B_OPS));
    for (int a = 0; a < na; ++a)
#pragma unroll
      for (int b = 0; b < D / 64; ++b)
        tma_load_3d(uv_u + a * R * D * 2 + b * R * 128, &tmB, bar(B_OPS), kvh * D + 64 * b, 0, agent0 + a);
    for (int n = 0; n < n_spec; ++n) issue(n);
  }
  pdl_wait();
  const int64_t kvl = p.kv_len[seq];
  const bool bad_len = kvl < 1 || kvl > p.max_kv_len;
  const int64_t k_hi = bad_len ? k_lo : min(te * KT, kvl);
  const int n_tiles = k_hi > k_lo ? (int)((k_hi - k_lo + KT - 1) / KT) : 0;

  // ---- the staged queries into the B operand of S (swizzled); this thread's
  // B_k^a chunks of the [U | V] build into registers.  An item of the build is
  // (agent, rho, 8 frequencies).
  const bool ops_ok = mbar_wait_clk(bar(B_OPS), 0);
  const int n_ag = (RP + g - 1) / g;            // agents whose rows fall within RP
  const int items = n_ag * R * 8;
  constexpr int MAXK = 4;                       // items per thread (at most 4 agents x 32 x 8)
  uint4 b1[MAXK], b2[MAXK];
  {
    for (int it = tid; it < QP * (D / 8); it += NTHR) {
      const int row = it / (D / 8), c = (it % (D / 8)) * 8;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (row < n_rows && !bad_len) v = *reinterpret_cast<const uint4*>(pbuf + row * D * 2 + c * 2);
      *reinterpret_cast<uint4*>(qop + tile_off<D, QP>(row, c)) = v;
    }
#pragma unroll
    for (int k = 0; k < MAXK; ++k) {
      const int it = tid + k * NTHR;
      b1[k] = b2[k] = make_uint4(0, 0, 0, 0);
      const int a = it / (R * 8), rho = (it / 8) % R, i0 = (it & 7) * 8;
      if (it < items && a < na && !bad_len) {
        const unsigned char* br = uv + a * R * D * 2;
        b1[k] = *reinterpret_cast<const uint4*>(br + tile_off<D, R>(rho, i0));
        b2[k] = *reinterpret_cast<const uint4*>(br + tile_off<D, R>(rho, D / 2 + i0));
      }
    }
  }
  // ---- decode step in one launch: the CTA whose keys hold position kv_len - 1
  // forms that token's LR row x_new [A_k | A_v] (fp32 sums, rounded to bf16
  // as the append rounds them); one CTA per LR cache writes it to the cache
  const int64_t p_new = kvl - 1;
  const bool has_new = p.x_new != nullptr && !bad_len && p_new >= k_lo && p_new < k_hi;
  if (has_new) {
    constexpr int CH = 2 * R / 8;            // 16-byte column chunks of an A row
    constexpr int RPI = 32 / CH;             // A rows per warp and iteration
    const __nv_bfloat16* x = reinterpret_cast<const __nv_bfloat16*>(p.x_new) + (int64_t)seq * p.hidden;
    const __nv_bfloat16* A = reinterpret_cast<const __nv_bfloat16*>(p.A_kv) +
                             (p.lr_agent ? (int64_t)agent0 * p.hidden * 2 * R : 0);
    const int ch = lane % CH, rs = lane / CH;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    for (int64_t h = (int64_t)w * RPI + rs; h < p.hidden; h += (int64_t)(NTHR / 32) * RPI) {
      const float xv = __bfloat162float(x[h]);
      const uint4 a = __ldg(reinterpret_cast<const uint4*>(A + h * 2 * R + 8 * ch));
      const uint32_t* aw = reinterpret_cast<const uint32_t*>(&a);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = unpack_bf16(aw[e]);
        acc[2 * e] = fmaf(xv, f.x, acc[2 * e]);
        acc[2 * e + 1] = fmaf(xv, f.y, acc[2 * e + 1]);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e)
#pragma unroll
      for (int o = CH; o < 32; o <<= 1) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
    if (rs == 0)
#pragma unroll
      for (int e = 0; e < 8; ++e) red[w * 2 * R + 8 * ch + e] = acc[e];
  }
  if (w == WM) tmem_alloc(smem_u32(tslot), T_COLS);
  tc_fence_before();
  __syncthreads();   // queries staged, the new row's partial sums, the TMEM address
  tc_fence_after();
  const uint32_t tmem = *tslot;
  if (has_new && tid < 2 * R) {
    float v = 0.f;
#pragma unroll
    for (int ww = 0; ww < NTHR / 32; ++ww) v += red[ww * 2 * R + tid];
    const __nv_bfloat16 b = __float2bfloat16_rn(v);
    newrow[tid] = b;
    if (kvh == 0 && (p.lr_agent || blockIdx.y == 0)) {   // the cache's one writer
      __nv_bfloat16* lr = reinterpret_cast<__nv_bfloat16*>(const_cast<void*>(p.lr)) +
                          (p.lr_agent ? (int64_t)agent0 * p.lr_agent : 0) + (int64_t)seq * p.lr_seq;
      lr[p_new * 2 * R + tid] = b;
    }
  }

  // ---- [U | V]: the B operand of W = CS UV^T, a row per (query row, rho):
  // U = s (q_i B_i + q_{i+d/2} B_{i+d/2}) in K columns i, V = s (q_{i+d/2} B_i -
  // q_i B_{i+d/2}) in K columns d/2 + i, over each of the agent's g query rows
  for (int it = tid; it < C::P_BYTES / 16; it += NTHR)
    *reinterpret_cast<uint4*>(pbuf + it * 16) = make_uint4(0, 0, 0, 0);
  {
    const float s = p.s;
#pragma unroll
    for (int k = 0; k < MAXK; ++k) {
      const int it = tid + k * NTHR;
      if (it >= items) continue;
      const int a = it / (R * 8), rho = (it / 8) % R, i0 = (it & 7) * 8;
      const uint32_t* b1w = reinterpret_cast<const uint32_t*>(&b1[k]);
      const uint32_t* b2w = reinterpret_cast<const uint32_t*>(&b2[k]);
      for (int gi = 0; gi < g; ++gi) {
        const int row = a * g + gi;
        if (row >= RP) break;
        const uint4 q1 = *reinterpret_cast<const uint4*>(qop + tile_off<D, QP>(row, i0));
        const uint4 q2 = *reinterpret_cast<const uint4*>(qop + tile_off<D, QP>(row, D / 2 + i0));
        const uint32_t* q1w = reinterpret_cast<const uint32_t*>(&q1);
        const uint32_t* q2w = reinterpret_cast<const uint32_t*>(&q2);
        uint4 u4, v4;
        uint32_t* uw = reinterpret_cast<uint32_t*>(&u4);
        uint32_t* vw = reinterpret_cast<uint32_t*>(&v4);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 x1 = unpack_bf16(q1w[e]), x2 = unpack_bf16(q2w[e]);
          const float2 c1 = unpack_bf16(b1w[e]), c2 = unpack_bf16(b2w[e]);
          uw[e] = pack_bf16(s * fmaf(x1.x, c1.x, x2.x * c2.x), s * fmaf(x1.y, c1.y, x2.y * c2.y));
          vw[e] = pack_bf16(s * fmaf(x2.x, c1.x, -x1.x * c2.x), s * fmaf(x2.y, c1.y, -x1.y * c2.y));
        }
        const int n = row * R + rho;
        *reinterpret_cast<uint4*>(uv + tile_off<D, NW>(n, i0)) = u4;
        *reinterpret_cast<uint4*>(uv + tile_off<D, NW>(n, D / 2 + i0)) = v4;
      }
    }
  }

  // ---- score warps: the per-lane table (cos, sin)(j theta_i) of their 32
  // frequencies into TMEM, and the exact (cos, sin)(k0 theta_i) of the first
  // three tiles
  const int sp = w & 3, hh = (w >> 2) & 1;
  const int jk = 32 * sp + lane;                  // this thread's key in a tile (its TMEM lane)
  const uint32_t lane_off = (uint32_t)(32 * sp) << 16;
  if (w < NSW) {
    uint32_t cj[32], sj[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const float2 a = sincos_small((float)jk * rt.thetaf[32 * hh + e]);
      cj[e] = __float_as_uint(a.x);
      sj[e] = __float_as_uint(a.y);
    }
    tmem_st32x32b_x32(tmem + T_CSJ + 64 * hh + lane_off, cj);
    tmem_st32x32b_x32(tmem + T_CSJ + 64 * hh + 32 + lane_off, sj);
    tmem_wait_st();
    if (sp == 0) {
      const int i = 32 * hh + lane;
#pragma unroll
      for (int t = 0; t < 3; ++t) cs0[t * 64 + i] = rope_cs_sfu(k_lo + (int64_t)t * KT, rt.theta[i]);
    }
  }

  fence_proxy_async_smem();   // UV, Q and P are read by the tensor cores (async proxy)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // Every wait is bounded in time.  After one has run out, a thread skips its
  // later waits but keeps every arrive, commit and named barrier of its role,
  // so the other roles finish too (their own waits may run out once) and the
  // CTA reaches its end quickly, reporting the failure.
  int fail = 0;
  auto wt = [&](int b, uint32_t parity) {
    if (!fail && !mbar_wait_clk(bar(b), parity)) fail = 1;
  };
  const float sl2 = p.scale * kLog2e;

  // CS of tile n into TMEM buffer n & 1: lane j, columns 16 hh.. (cos) and
  // 32 + 16 hh.. (sin), bf16 pairs; (cos, sin)((k0 + j) theta) by the angle
  // sum from cs0 slot n & 3 and this lane's table
  auto write_cs = [&](int n) {
    uint32_t cj[32], sj[32];
    tmem_ld32x32b_x32(cj, tmem + T_CSJ + 64 * hh + lane_off);
    tmem_ld32x32b_x32(sj, tmem + T_CSJ + 64 * hh + 32 + lane_off);
    tmem_wait_ld_r32(cj);
    tmem_wait_ld_r32(sj);
    const float4* c0 = reinterpret_cast<const float4*>(cs0 + (n & 3) * 64 + 32 * hh);
    uint32_t cw[16], sw[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const float4 v = c0[e];   // (cos, sin) of frequencies 2e, 2e + 1 of this half
      const uint64_t cc = f2(v.x, v.z), ss = f2(v.y, v.w), nss = f2(-v.y, -v.w);
      const uint64_t CJ = f2(__uint_as_float(cj[2 * e]), __uint_as_float(cj[2 * e + 1]));
      const uint64_t SJ = f2(__uint_as_float(sj[2 * e]), __uint_as_float(sj[2 * e + 1]));
      const float2 co = f2_unpack(fma_f2(cc, CJ, mul_f2(nss, SJ)));
      const float2 si = f2_unpack(fma_f2(ss, CJ, mul_f2(cc, SJ)));
      cw[e] = pack_bf16(co.x, co.y);
      sw[e] = pack_bf16(si.x, si.y);
    }
    const uint32_t tb = tmem + T_CS + 64 * (n & 1) + lane_off;
    tmem_st32x32b_x16(tb + 16 * hh, cw);
    tmem_st32x32b_x16(tb + 32 + 16 * hh, sw);
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(bar(B_CSFULL + (n & 1)));
  };

  if (w < NSW) {
    // ======================================================== score warps
    if (n_tiles > 0) write_cs(0);
    if (n_tiles > 1) write_cs(1);
    // the incremental (cos, sin)(k0 theta) of this lane's frequency (sp == 0)
    float2 cs_cur = make_float2(1.f, 0.f), cs_step = cs_cur;
    if (sp == 0) {
      cs_cur = cs0[2 * 64 + 32 * hh + lane];
      cs_step = rope_cs_sfu(KT, theta[32 * hh + lane]);
    }
    float m_ref[RH], l_st[RH];
#pragma unroll
    for (int r = 0; r < RH; ++r) {
      m_ref[r] = -INFINITY;
      l_st[r] = 0.f;
    }
    for (int n = 0; n < n_tiles; ++n) {
      const int s = n % ST;
      const int64_t k0 = k_lo + (int64_t)n * KT;
      const bool valid = k0 + jk < k_hi;
      wt(B_FULL + s, (n / ST) & 1);
      wt(B_TFULL, n & 1);
      if (has_new && p_new >= k0 && p_new < k0 + KT) wt(B_PATCH, 0);   // the new LR row is in place
      tc_fence_after();
      // S (every row), this half's W columns (every load in flight before one
      // wait), this key's LRk
      constexpr int NCH = RH * R / 32;   // 32-column chunks of this half's W
      uint32_t sv[16];
      uint32_t wv[NCH][32];
      tmem_ld32x32b_x16(sv, tmem + T_S + lane_off);
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch)
        tmem_ld32x32b_x32(wv[ch], tmem + T_W + (uint32_t)(hh * RH * R + 32 * ch) + lane_off);
      uint32_t lkw[R / 2];   // LRk of this key as bf16 pairs
      {
        const unsigned char* lrow = stages + s * C::STAGE + 2 * C::KV_TILE;
#pragma unroll
        for (int c = 0; c < R; c += 8) {
          const uint4 v = *reinterpret_cast<const uint4*>(lrow + tile_off<2 * R, KT>(jk, c));
          lkw[c / 2] = v.x; lkw[c / 2 + 1] = v.y; lkw[c / 2 + 2] = v.z; lkw[c / 2 + 3] = v.w;
        }
      }
      tmem_wait_ld_r16(sv);
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch) reg_after_wait32(wv[ch]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_WFREE));   // S and W of this tile are in registers
      float dsc[RH];
      constexpr int RPC = 32 / R;   // rows per 32-column chunk
#pragma unroll
      for (int ch = 0; ch < NCH; ++ch)
#pragma unroll
        for (int rr = 0; rr < RPC; ++rr) {
          uint64_t acc = f2(0.f, 0.f);
#pragma unroll
          for (int rho = 0; rho < R; rho += 2) {
            const float2 l2 = unpack_bf16(lkw[rho / 2]);
            acc = fma_f2(f2(l2.x, l2.y),
                         f2(__uint_as_float(wv[ch][rr * R + rho]), __uint_as_float(wv[ch][rr * R + rho + 1])), acc);
          }
          const float2 a2 = f2_unpack(acc);
          dsc[ch * RPC + rr] = a2.x + a2.y;
        }
      // scores (log2 units) and this tile's row maxima
      float x[RH];
#pragma unroll
      for (int r = 0; r < RH; ++r) {
        const float sb = __uint_as_float(hh ? sv[RH + r] : sv[r]);
        x[r] = valid ? (sb + dsc[r]) * sl2 : -INFINITY;
        const float mt = warp_max(x[r]);
        if (lane == 0) Mx[(hh * 8 + r) * 4 + sp] = mt;
      }
      bar_sync(1 + hh, 128);
      bool moved = false;
      float corr[RH];
#pragma unroll
      for (int r = 0; r < RH; ++r) {
        const float4 m4 = *reinterpret_cast<const float4*>(Mx + (hh * 8 + r) * 4);
        const float tmax = fmaxf(fmaxf(m4.x, m4.y), fmaxf(m4.z, m4.w));
        corr[r] = 1.f;
        if (tmax > m_ref[r] + 8.f) {   // lazy: move the reference only when it is 2^8 behind
          corr[r] = m_ref[r] == -INFINITY ? 0.f : fast_exp2(m_ref[r] - tmax);
          m_ref[r] = tmax;
          l_st[r] *= corr[r];
          moved = true;
        }
        if (sp == 0 && lane == 0) Corr[(n & 1) * QP + hh * RH + r] = corr[r];
      }
      // P V and O_lr of the previous tile are done: P is free, O^T is final
      if (n > 0) wt(B_PFREE, (n - 1) & 1);
      if (moved && n > 0) {   // O^T (TMEM lanes = d, columns = rows) times corr
        tc_fence_after();
#pragma unroll
        for (int r = 0; r < RH; ++r)
          if (corr[r] != 1.f) {
            const uint32_t ta = tmem + T_O + (uint32_t)(hh * RH + r) + lane_off;
            uint32_t o = tmem_ld32x32b_x1(ta);
            tmem_wait_ld_r1(o);
            tmem_st32x32b_x1(ta, __float_as_uint(__uint_as_float(o) * corr[r]));
          }
        tmem_wait_st();
      }
#pragma unroll
      for (int r = 0; r < RH; ++r) {
        const float pr = m_ref[r] == -INFINITY ? 0.f : fast_exp2(x[r] - m_ref[r]);
        l_st[r] += pr;
        const __nv_bfloat16 pb = __float2bfloat16_rn(pr);
        sts16(p_u + tile_off<KT, QP>(hh * RH + r, jk), *reinterpret_cast<const uint16_t*>(&pb));
      }
      fence_proxy_async_smem();   // the P V MMA reads P through the async proxy
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_PFULL));
      // off the tile's critical path: CS two tiles ahead (W of this tile has read
      // its buffer), and (cos, sin)(k0 theta) three tiles ahead: the previous
      // one turned by KT theta in fp32, taken exactly again every 16 tiles
      if (n + 2 < n_tiles) write_cs(n + 2);
      if (sp == 0 && n + 3 < n_tiles) {
        const int m = n + 3;
        cs_cur = (m & 15) == 0 ? rope_cs_sfu(k_lo + (int64_t)m * KT, theta[32 * hh + lane])
                               : make_float2(fmaf(cs_cur.x, cs_step.x, -cs_cur.y * cs_step.y),
                                             fmaf(cs_cur.y, cs_step.x, cs_cur.x * cs_step.y));
        cs0[(m & 3) * 64 + 32 * hh + lane] = cs_cur;
      }
    }
    // ---- partial of this CTA: l (over the keys), m, O^T
#pragma unroll
    for (int r = 0; r < RH; ++r) {
      const float lt = warp_sum(l_st[r]);
      if (lane == 0) Lsum[(hh * RH + r) * 4 + sp] = lt;
      if (sp == 0 && lane == 0) Mfin[hh * RH + r] = m_ref[r];
    }
    uint32_t ov[16];
    if (n_tiles > 0) {
      wt(B_ODONE, 0);
      tc_fence_after();
      tmem_ld32x32b_x16(ov, tmem + T_O + lane_off);
      tmem_wait_ld_r16(ov);
    } else {
#pragma unroll
      for (int c = 0; c < 16; ++c) ov[c] = 0u;
    }
#pragma unroll
    for (int r = 0; r < RH; ++r) Part[(hh * RH + r) * WP + jk] = __uint_as_float(hh ? ov[RH + r] : ov[r]);
  } else if (w == WV) {
    // ======================================================== value warp
    // O_lr^T (r x rows) += LRv^T P^T over the tile's keys (mma.sync), and the
    // rows of a tile past the sequence's end zeroed in V and LRv
    float Olr[C::MR][2][4];
#pragma unroll
    for (int mr = 0; mr < C::MR; ++mr)
#pragma unroll
      for (int pt = 0; pt < 2; ++pt)
#pragma unroll
        for (int e = 0; e < 4; ++e) Olr[mr][pt][e] = 0.f;
    const int mi = lane >> 3, rr = lane & 7, t4 = lane & 3;
    int n_issued = n_spec, n_seen = 0;   // tiles requested / observed landed (lane 0)
    if (lane == 0)
      for (int m = ST; m < n_tiles && m < ST + kL2Ahead; ++m) prefetch(m);
    {   // B_v^a head slices for the epilogue, into L2 while the keys stream
      const __nv_bfloat16* bvp = reinterpret_cast<const __nv_bfloat16*>(p.B_v) + (int64_t)agent0 * R * ldB + kvh * D;
      for (int i = lane; i < na * R * 2; i += 32) prefetch_l2(bvp + (int64_t)(i >> 1) * ldB + 64 * (i & 1));
    }
    for (int n = 0; n < n_tiles; ++n) {
      const int s = n % ST;
      const int64_t k0 = k_lo + (int64_t)n * KT;
      unsigned char* sb = stages + s * C::STAGE;
      wt(B_FULL + s, (n / ST) & 1);
      if (lane == 0 && !fail) n_seen = n + 1;
      if (has_new && p_new >= k0 && p_new < k0 + KT) {   // the new token's LR row over the loaded one
        for (int c = lane; c < 2 * R / 8; c += 32)
          *reinterpret_cast<uint4*>(sb + 2 * C::KV_TILE + tile_off<2 * R, KT>((int)(p_new - k0), 8 * c)) =
              reinterpret_cast<const uint4*>(newrow)[c];
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(B_PATCH));
      }
      if (k0 + KT > k_hi) {   // P is 0 there; zeroed rows keep stale NaN out of P V
        const int first = (int)(k_hi - k0);
        for (int i = lane; i < (KT - first) * (D / 8); i += 32) {
          const int row = first + i / (D / 8), c = 8 * (i % (D / 8));
          *reinterpret_cast<uint4*>(sb + C::KV_TILE + tile_off<D, KT>(row, c)) = make_uint4(0, 0, 0, 0);
        }
        for (int i = lane; i < (KT - first) * (R / 8); i += 32) {
          const int row = first + i / (R / 8), c = R + 8 * (i % (R / 8));
          *reinterpret_cast<uint4*>(sb + 2 * C::KV_TILE + tile_off<2 * R, KT>(row, c)) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(B_PFULL));
      wt(B_PFULL, n & 1);
#pragma unroll
      for (int pt = 0; pt < 2; ++pt) {
        const float c0 = Corr[(n & 1) * QP + 8 * pt + 2 * t4];
        const float c1 = Corr[(n & 1) * QP + 8 * pt + 2 * t4 + 1];
#pragma unroll
        for (int mr = 0; mr < C::MR; ++mr) {
          Olr[mr][pt][0] *= c0; Olr[mr][pt][2] *= c0;
          Olr[mr][pt][1] *= c1; Olr[mr][pt][3] *= c1;
        }
      }
      const uint32_t sl = smem_u32(sb + 2 * C::KV_TILE);
#pragma unroll 2
      for (int ks = 0; ks < KT / 16; ++ks) {
        uint32_t bP[2][2];
#pragma unroll
        for (int pt = 0; pt < 2; ++pt)
          ldsm_x2(bP[pt][0], bP[pt][1], p_u + tile_off<KT, QP>(8 * pt + rr, 16 * ks + ((lane >> 3) & 1) * 8));
#pragma unroll
        for (int mr = 0; mr < C::MR; ++mr) {
          uint32_t aV[4];
          ldsm_x4_t(aV, sl + tile_off<2 * R, KT>(16 * ks + rr + (mi >> 1) * 8, R + 16 * mr + (mi & 1) * 8));
#pragma unroll
          for (int pt = 0; pt < 2; ++pt) mma16816(Olr[mr][pt], aV, bP[pt][0], bP[pt][1]);
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(bar(B_PFREE));
        mbar_arrive(bar(B_EMPTY + s));
        if (n + ST < n_tiles) {   // the stage's refill once the P V MMA has read it
          wt(B_EMPTY + s, (n / ST) & 1);
          if (!fail) {
            issue(n + ST);
            n_issued = n + ST + 1;
            if (n + ST + kL2Ahead < n_tiles) prefetch(n + ST + kL2Ahead);
          }
        }
      }
      __syncwarp();
    }
    // every requested tile lands before the CTA leaves: those loaded ahead of
    // kv_len and not used, and those still in flight after a wait ran out
    if (lane == 0)
      for (int m = max(n_seen, n_issued - ST); m < n_issued; ++m)
        if (!mbar_wait_clk(bar(B_FULL + m % ST), (m / ST) & 1)) fail = 1;
    // the partial's O_lr (the UV area is free once every MMA has completed)
    if (n_tiles > 0) wt(B_ODONE, 0);
#pragma unroll
    for (int mr = 0; mr < C::MR; ++mr)
#pragma unroll
      for (int pt = 0; pt < 2; ++pt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int row = 8 * pt + 2 * t4 + (e & 1);
          const int rho = 16 * mr + (lane >> 2) + (e >> 1) * 8;
          if (row < RP) Part[row * WP + D + rho] = Olr[mr][pt][e];
        }
  } else if (w == WM) {
    // ======================================================== MMA warp
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t ID_S = umma_idesc_bf16(128, QP, 0, 0);
      constexpr uint32_t ID_W = umma_idesc_bf16(128, NW, 0, 0);
      constexpr uint32_t ID_PV = umma_idesc_bf16(128, QP, 1, 0);   // O^T += V^T P^T, A = V MN-major
      const uint64_t dQ = umma_desc(q_u, 16, 1024, 2);
      const uint64_t dUV = umma_desc(uv_u, 16, 1024, 2);
      const uint64_t dP = umma_desc(p_u, 16, 1024, 2);
      auto mma_pv = [&](int m) {
        wt(B_PFULL, m & 1);
        tc_fence_after();
        const uint64_t dV = umma_desc(st_u + (m % ST) * C::STAGE + C::KV_TILE, KT * 128, 1024, 2);
#pragma unroll
        for (int kk = 0; kk < KT / 16; ++kk)
          umma_bf16(tmem + T_O, umma_desc_add(dV, kk * 16 * 128),
                    umma_desc_add(dP, (kk >> 2) * (QP * 128) + (kk & 3) * 32), ID_PV, (m > 0 || kk > 0) ? 1u : 0u);
        umma_commit(bar(B_PFREE));
        umma_commit(bar(B_EMPTY + m % ST));
      };
      for (int n = 0; n < n_tiles; ++n) {
        const int s = n % ST;
        wt(B_FULL + s, (n / ST) & 1);
        if (n > 0) wt(B_WFREE, (n - 1) & 1);
        wt(B_CSFULL + (n & 1), (n >> 1) & 1);
        tc_fence_after();
        const uint64_t dK = umma_desc(st_u + s * C::STAGE, 16, 1024, 2);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_bf16(tmem + T_S, umma_desc_add(dK, (kk >> 2) * (KT * 128) + (kk & 3) * 32),
                    umma_desc_add(dQ, (kk >> 2) * (QP * 128) + (kk & 3) * 32), ID_S, kk > 0);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_bf16_ts(tmem + T_W, tmem + T_CS + 64 * (n & 1) + kk * 8,
                       umma_desc_add(dUV, (kk >> 2) * (NW * 128) + (kk & 3) * 32), ID_W, kk > 0);
        umma_commit(bar(B_TFULL));
        if (n > 0) mma_pv(n - 1);
      }
      mma_pv(n_tiles - 1);
      umma_commit(bar(B_ODONE));
      // TMEM is freed below: every MMA has completed first (an MMA always
      // completes, so this wait does not run out)
      if (!mbar_wait_clk(bar(B_ODONE), 0)) fail = 1;
    }
    __syncwarp();
  }
  if (fail || !ops_ok) s_misc[0] = 1;
  tc_fence_before();
  __syncthreads();
  if (w == WM) {
    tc_fence_after();
    tmem_dealloc(tmem, T_COLS);
  }
  if (bad_len && tid == 0 && split == 0) atomicOr(p.err, 1);
  for (int row = tid; row < RP; row += NTHR) {
    Part[row * WP + D + R] = Mfin[row];
    Part[row * WP + D + R + 1] = Lsum[row * 4] + Lsum[row * 4 + 1] + Lsum[row * 4 + 2] + Lsum[row * 4 + 3];
  }
  if (s_misc[0] && tid == 0) atomicOr(p.err, 2);
  __syncthreads();

  const __nv_bfloat16* bv = reinterpret_cast<const __nv_bfloat16*>(p.B_v) + (int64_t)agent0 * R * ldB + kvh * D;
  // out[row][c..c+3] = (O + s O_lr B_v^a) / l from a merged row record
  auto emit = [&](const float* rec, int row, int c) {
    const int a = row / g, gi = row % g;
    const float* ol = rec + D;
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
    const float l = rec[D + R + 1];
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float4 acc = *reinterpret_cast<const float4*>(rec + c);
    acc.x = fmaf(p.s, z0, acc.x) * inv; acc.y = fmaf(p.s, z1, acc.y) * inv;
    acc.z = fmaf(p.s, z2, acc.z) * inv; acc.w = fmaf(p.s, z3, acc.w) * inv;
    const int64_t oi = (((int64_t)seq * na_tot + agent0 + a) * p.n_q + kvh * g + gi) * D + c;
    if (p.out_bf16) {
      uint2 o;
      o.x = pack_bf16(acc.x, acc.y);
      o.y = pack_bf16(acc.z, acc.w);
      *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(p.out) + oi) = o;
    } else {
      *reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + oi) = acc;
    }
  };

  if (ns == 1) {
    if (s_misc[0] || bad_len) return;
    for (int i = tid; i < n_rows * (D / 4); i += NTHR) {
      const int row = i / (D / 4), c = 4 * (i % (D / 4));
      emit(Part + row * WP, row, c);
    }
    return;
  }

  // ---- split merge over the cluster.  The unit's splits are one thread-block
  // cluster (rank = split); each CTA's partial (O_base, O_lr, m, l) stays in
  // its own shared memory, and after a cluster barrier every CTA merges a share
  // of the unit's (row, 32-column quarter) pieces, reading the partials of all
  // splits over distributed shared memory, one warp per piece:
  //   w_k = 2^(m_k - M) / sum_k 2^(m_k - M) l_k,  M = max_k m_k,
  //   out = sum_k w_k O_base,k + s (sum_k w_k O_lr,k) B_v^a  (B_v^a once per row)
  cluster_sync_all();   // every split's partial is in place
  if (!s_misc[0] && !bad_len) {
    const uint32_t part_u = smem_u32(Part);
    for (int piece = split + ns * w; piece < n_rows * 4; piece += ns * (NTHR / 32)) {
      const int row = piece >> 2, c0 = 32 * (piece & 3);
      const uint32_t rowb = part_u + (uint32_t)(row * WP) * 4;
      // lane k: split k's (m, l)
      float2 ml = make_float2(-INFINITY, 0.f);
      if (lane < ns) ml = dsmem_ld2(dsmem_addr(rowb + (D + R) * 4, lane));
      const float M = warp_max(ml.x);
      const float e = (lane < ns && ml.x != -INFINITY) ? fast_exp2(ml.x - M) : 0.f;
      const float L = warp_sum(e * ml.y);
      const float inv = L > 0.f ? 1.f / L : 0.f;
      // lane c: the merged O_base of column c0 + c; lane rho: O_lr[rho] (R <= 32)
      float o = 0.f, olr = 0.f;
      for (int k = 0; k < ns; ++k) {
        const float wk = __shfl_sync(0xffffffffu, e, k);
        if (wk == 0.f) continue;
        const uint32_t rk = dsmem_addr(rowb, k);
        o = fmaf(wk, dsmem_ld(rk + (c0 + lane) * 4), o);
        if (lane < R) olr = fmaf(wk, dsmem_ld(rk + (D + lane) * 4), olr);
      }
      // out = (O + s O_lr B_v^a) / L for this lane's column
      const int a = row / g, gi = row % g;
      const __nv_bfloat16* bb = bv + (size_t)a * R * ldB + c0 + lane;
      float z = 0.f;
#pragma unroll
      for (int rho = 0; rho < R; ++rho)
        z = fmaf(__shfl_sync(0xffffffffu, olr, rho), __bfloat162float(bb[(size_t)rho * ldB]), z);
      const float val = fmaf(p.s, z, o) * inv;
      const int64_t oi = (((int64_t)seq * na_tot + agent0 + a) * p.n_q + kvh * g + gi) * D + c0 + lane;
      if (p.out_bf16) reinterpret_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(val);
      else reinterpret_cast<float*>(p.out)[oi] = val;
    }
  }
  cluster_sync_all();   // no CTA leaves while the others read its partial
}

// -------------------------------------------------------------------- host
bool make_maps(const AttnParams& p, CUtensorMap* mk, CUtensorMap* mv, CUtensorMap* ml) {
  auto enc = encode_fn();
  if (!enc) return false;
  const int R = p.r;
  cuuint64_t kdims[4] = {(cuuint64_t)D, (cuuint64_t)p.L_max, (cuuint64_t)p.n_kv, (cuuint64_t)p.n_seqs};
  cuuint64_t kstr[3] = {(cuuint64_t)p.kv_tok * 2, (cuuint64_t)p.kv_head * 2, (cuuint64_t)p.kv_seq * 2};
  cuuint32_t kbox[4] = {64, (cuuint32_t)KT, 1, 1};
  cuuint32_t one[4] = {1, 1, 1, 1};
  if (enc(mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(p.k_base), kdims, kstr, kbox, one,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  if (enc(mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(p.v_base), kdims, kstr, kbox, one,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
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

int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
    cudaGetLastError();
    return kSMs;
  }
  return n;
}

// padded rows of a group of G agents (a multiple of 4), 0 if no instance holds it
int rows_padded(const AttnParams& p, int G) {
  const int rows = G * p.g;
  const int rp = (rows + 3) / 4 * 4;
  if (p.r == 16) return rp <= 12 ? rp : 0;
  if (p.r == 32) return rp <= 4 ? rp : 0;
  return 0;
}

size_t smem_of(int r, int rp) {
  if (r == 32) return Cfg<32, 4>::smem();
  switch (rp) {
    case 4: return Cfg<16, 4>::smem();
    case 8: return Cfg<16, 8>::smem();
    default: return Cfg<16, 12>::smem();
  }
}

template <int R, int RP>
cudaError_t launch_t(const AttnParams& pin, cudaStream_t st) {
  AttnParams p = pin;
  using Cf = Cfg<R, RP>;
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
    if (encode_fn()(&mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(p.B_k), dims, str, box, one,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  const size_t sm = Cf::smem();
  auto kern = decode_cs_kernel<R, RP>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  if (p.n_splits > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(NTHR);
  cfg.dynamicSmemBytes = sm;
  cfg.stream = st;
  // the splits of a unit form one cluster (they merge over distributed shared
  // memory); the set-up may overlap the preceding kernel (programmatic
  // dependent launch: the kernel waits for it before reading any input)
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  // as many splits as a resident cluster can hold: halve until one fits
  for (;;) {
    attr[0].val.clusterDim.x = (unsigned)p.n_splits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(p.n_splits, (p.n_agents + p.agent_group - 1) / p.agent_group, p.n_seqs * p.n_kv);
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int nc = 0;
    if (p.n_splits == 1 || (cudaOccupancyMaxActiveClusters(&nc, kern, &cfg) == cudaSuccess && nc >= 1)) break;
    cudaGetLastError();
    p.n_splits = p.n_splits / 2;
  }
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, kern, mk, mv, ml, mb, p, rt);
  if (e != cudaSuccess) {   // without the overlap where the runtime refuses it
    cudaGetLastError();
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, mk, mv, ml, mb, p, rt);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace

// Agents per CTA of the cos/sin-table decode (0: the shape does not run on
// it): the largest group whose padded rows fit an instance and whose shared
// memory fits; one LR cache per agent takes one agent per CTA.
int cs_group_size(const AttnParams& p) {
  if (p.d != 128 || !(p.r == 16 || p.r == 32)) return 0;
  if (!(p.g == 1 || p.g == 2 || p.g == 4 || p.g == 8)) return 0;
  if (p.L_max >= (1ll << 31)) return 0;
  const int gmax = p.lr_agent ? 1 : 4;
  for (int G = p.n_agents < gmax ? p.n_agents : gmax; G >= 1; --G) {
    const int rp = rows_padded(p, G);
    if (rp && smem_of(p.r, rp) <= 227 * 1024) return G;
  }
  return 0;
}

// Splits of each (sequence, KV head, agent group) over the keys.  Fewer units
// than SMs: one wave, as many splits as keep every SM busy (but as few as give
// the same longest split).  More: the split count (up to 4) whose waves are
// fullest, so that the last wave does not leave most SMs idle.
int cs_splits(const AttnParams& p, int G) {
  const int groups = (p.n_agents + G - 1) / G;
  const int units = p.n_seqs * p.n_kv * groups;
  if (units < 1) return 1;
  const int64_t total_tiles = (p.max_kv_len + KT - 1) / KT;
  const int sms = device_sms();
  int64_t ns;
  if (units < sms) {
    ns = sms / units;
    if (ns > kMaxSplits) ns = kMaxSplits;
    if (ns > total_tiles) ns = total_tiles;
    if (ns < 1) ns = 1;
    const int64_t per = (total_tiles + ns - 1) / ns;
    ns = (total_tiles + per - 1) / per;
  } else {
    double best = -1.0;
    ns = 1;
    for (int s = 1; s <= 4 && s * 8 <= total_tiles; ++s) {
      const int64_t ctas = (int64_t)units * s;
      const int64_t waves = (ctas + sms - 1) / sms;
      const double eff = (double)ctas / (double)(waves * sms) - 0.01 * s;
      if (eff > best) {
        best = eff;
        ns = s;
      }
    }
  }
  return (int)ns;
}

cudaError_t launch_decode_cs(const AttnParams& pin, la_dtype out, cudaStream_t st) {
  AttnParams p = pin;
  p.out_bf16 = out == LA_BF16;
  p.agent_group = cs_group_size(p);
  if (p.agent_group < 1) return cudaErrorInvalidValue;
  if (p.n_splits > kMaxSplits) return cudaErrorInvalidValue;
  if (p.r == 32) return launch_t<32, 4>(p, st);
  switch (rows_padded(p, p.agent_group)) {
    case 4: return launch_t<16, 4>(p, st);
    case 8: return launch_t<16, 8>(p, st);
    default: return launch_t<16, 12>(p, st);
  }
}

// The cos/sin-table decode merges its splits inside each cluster: it needs no
// workspace.
size_t cs_partial_bytes(const AttnParams&) { return 0; }
size_t cs_counter_ints(const AttnParams&) { return 0; }

}  // namespace la
