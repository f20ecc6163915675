// Flash-LoRA-Attention prefill on the tcgen05 tensor cores (bf16 storage,
// fp32 accumulation in TMEM).
//
// One CTA = one (sequence, agent, KV head) and a block of 128 query rows: the
// 128 / g query tokens of the block times the g query heads of the GQA group
// (row = token * g + head).  Keys stream in tiles of 128.  Per tile (LRAgent
// summary App. D.1: RoPE blocks reordering on the key side, so the delta is
// rebuilt in head dimension per tile):
//   dK   = LRk B_k^a                       tcgen05, M = 128 keys, N = d, K = r
//   K^a  = K_base + s R(t) dK              CUDA cores, written over K_base in
//                                          shared memory; R(t) = R(k0) R(j)
//   S    = Q K^a^T                         tcgen05, M = 128 rows, N = 128 keys
//   P    = exp2(S log2e / sqrt(d) - m)     CUDA cores, to TMEM as bf16
//   O   += P V_base,  O_lr += P LR         tcgen05, A = P from TMEM; value side
//                                          reordered (LRAgent explainer,
//                                          Metodologia 3): only r wide
// and once per row at the end out = (O + s O_lr B_v^a) / l.
// The running max is rescaled lazily: O and l are corrected only when a row's
// maximum grows by more than 2^8, so P <= 256 and the correction is rare.
//
// Warps: 8 compute warps build K^a in f16x2 arithmetic (16 keys each, the mma fragment layout of
// the delta) and run the softmax (two warps per TMEM sub-partition, 64 keys
// each); warp 8 issues the MMAs (and the first loads), warp 9 the TMA
// refills.  The compute warps build tile n+1
// before the softmax of tile n, so the S MMA of tile n+1 runs during that
// softmax and the P V MMA of tile n during the next build.
// The per-tile value arm (VT, the ablation of the reordering) instead builds
// V^a = V_base + s LRv B_v^a per tile (dV on the tensor cores, the sum over
// V_base in shared memory, like K^a), keeps P in shared memory (TMEM holds dV
// where the reordered arm keeps P and O_lr) and accumulates O += P V^a: the
// head-dimension rebuild per tile that the reordering removes.
// Where whole CTAs would leave SMs idle, the launch runs each block as a
// cluster of two CTAs over the two halves of its key tiles (template KS = 2),
// merged over distributed shared memory.  With one LR cache per agent the LR
// tiles are the CTA's agent's own (an agent coordinate of the LR tensor map).
#include <cmath>

#include <cuda_fp16.h>

#include "bf16_common.cuh"
#include "la_internal.cuh"
#include "ptx.cuh"

namespace la {
namespace {

using namespace ptx;

// bf16 pair + fp32 pair, rounded once to an fp16 pair (the K^a operand)
__device__ __forceinline__ uint32_t add_to_f16x2(uint32_t base_bf16x2, float2 d) {
  const float2 b = unpack_bf16(base_bf16x2);
  __half2 h = __floats2half2_rn(b.x + d.x, b.y + d.y);
  return *reinterpret_cast<uint32_t*>(&h);
}
// f16 pairs as 32-bit words and back, and a bf16 pair as an f16 pair (exact
// within f16's range)
__device__ __forceinline__ uint32_t h2_bits(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
__device__ __forceinline__ __half2 bits_h2(uint32_t v) { return *reinterpret_cast<__half2*>(&v); }
__device__ __forceinline__ __half2 bf16x2_h2(uint32_t v) {
  return __floats2half2_rn(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}
// a bf16 pair as a packed fp32 pair (exact), and a packed fp32 pair rounded
// once to an fp16 pair
__device__ __forceinline__ uint64_t bf16x2_f2(uint32_t v) {
  return f2(__uint_as_float(v << 16), __uint_as_float(v & 0xffff0000u));
}
__device__ __forceinline__ uint32_t f2_f16x2(uint64_t v) {
  const float2 f = f2_unpack(v);
  __half2 h = __floats2half2_rn(f.x, f.y);
  return *reinterpret_cast<uint32_t*>(&h);
}

// 2^x for a pair on the FMA pipe, beside the SFU's ex2 (the softmax's
// exponentials would otherwise queue on the SFU alone): x = n + f with n the
// nearest integer (the 1.5 * 2^23 rounding constant), f in [-1/2, 1/2]; 2^f by
// a degree-3 polynomial fitted here for least maximum relative error on that
// interval (Remez exchange: 7.5e-5, below the bf16 rounding P gets), and 2^n
// added to the exponent field.  x is clamped at -126, so a masked score gives
// about 1e-38 instead of 0 and the sum never leaves the normal range.
__device__ __forceinline__ uint64_t exp2_poly_f2(uint64_t x2) {
  constexpr float kRound = 12582912.f;   // 1.5 * 2^23
  const float2 xv = f2_unpack(x2);
  const uint64_t x = f2(fmaxf(xv.x, -126.f), fmaxf(xv.y, -126.f));
  const uint64_t t = add_f2(x, f2(kRound, kRound));
  const uint64_t fr = sub_f2(x, sub_f2(t, f2(kRound, kRound)));
  uint64_t p = fma_f2(f2(0.05517166853f, 0.05517166853f), fr, f2(0.24261112511f, 0.24261112511f));
  p = fma_f2(p, fr, f2(0.69326096773f, 0.69326096773f));
  p = fma_f2(p, fr, f2(0.99992805719f, 0.99992805719f));
  const float2 pv = f2_unpack(p), tv = f2_unpack(t);
  return f2(__uint_as_float(__float_as_uint(pv.x) + (__float_as_uint(tv.x) << 23)),
            __uint_as_float(__float_as_uint(pv.y) + (__float_as_uint(tv.y) << 23)));
}
// every kPolyExpEvery-th pair of a softmax row goes through exp2_poly_f2 (0: none)
constexpr int kPolyExpEvery = 4;

constexpr int PD = 128;                  // head_dim
constexpr int PKT = 128;                 // keys per tile
constexpr int PM = 128;                  // query rows per CTA
constexpr int PNC = 8;                   // compute warps
constexpr int PNTHR = 32 * (PNC + 2);  // + the MMA warp + the TMA refill warp
// TMEM columns (the per-tile value arm: dV at 256, O at 384, P in shared memory)
constexpr int T_DK = 0, T_S = 128, T_P = 256, T_O = 320, T_OL = 448, T_COLS = 512;
constexpr int T_DV = 256, T_OV = 384;
// named barriers (0 is __syncthreads)
constexpr int PBAR_CW = 1, PBAR_PAIR = 2;  // PBAR_PAIR + sub-partition: the two warps of a row block

template <int R, bool VT = false>
struct PCfg {
  // a K stage holds the K_base tile and the tile's LRk columns, a V stage the
  // V_base tile and its LRv columns: r columns of the LR rows, one TMA box
  static constexpr int LR_ROWB = R * 2;                         // bytes per LRk / LRv row
  static constexpr uint32_t LR_LAYOUT = LR_ROWB == 128 ? 2u : (LR_ROWB == 64 ? 4u : 6u);
  static constexpr int KV = PKT * PD * 2;                       // a K or V tile
  static constexpr int LR_TILE = align1k(PKT * R * 2);
  static constexpr int STAGE = KV + LR_TILE;
  static constexpr int NV = R >= 64 ? 1 : 2;                    // V stages (one at r = 64: room)
  static constexpr int Q_BYTES = PM * PD * 2;
  static constexpr int B_BYTES = R * PD * 2;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_BYTES;                 // [2] K stages
  static constexpr int OFF_V = OFF_K + 2 * STAGE;               // [NV] V stages
  static constexpr int OFF_BK = OFF_V + NV * STAGE;
  static constexpr int OFF_BV = OFF_BK + align1k(B_BYTES);
  static constexpr int OFF_P = OFF_BV + align1k(B_BYTES);       // per-tile value arm: P [128][128] bf16
  static constexpr int OFF_MISC = OFF_P + (VT ? PM * PKT * 2 : 0);
  // misc: anchors [2][64] float2, exchange [2][8][32] float, theta [64] double,
  // 18 mbarriers, the TMEM slot
  static constexpr int MISC = 1024 + 2048 + 512 + 144 + 16;
  static constexpr size_t SMEM = 1024 + OFF_MISC + MISC;
};

template <int R, int KS, bool VT>
__global__ void __launch_bounds__(PNTHR, 1)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmL,
                      const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmBv, const AttnParams p,
                      const __grid_constant__ RopeTheta rt) {
  constexpr int ksplit = KS;   // 1, or 2: the keys of a block split over a cluster of two CTAs
  using C = PCfg<R, VT>;
  constexpr int TO = VT ? T_OV : T_O;   // O^T's TMEM columns
  constexpr int D = PD;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(smem);
  const uint32_t q_u = sb + C::OFF_Q, k_u = sb + C::OFF_K, v_u = sb + C::OFF_V;
  const uint32_t bk_u = sb + C::OFF_BK, bv_u = sb + C::OFF_BV;
  unsigned char* misc = smem + C::OFF_MISC;
  float2* anc = reinterpret_cast<float2*>(misc);               // [2][64] s (cos, sin)(k0 theta_i)
  float* xch = reinterpret_cast<float*>(misc + 1024);          // [2][8][32]
  double* theta = reinterpret_cast<double*>(misc + 3072);      // [64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(misc + 3584);   // [18]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(misc + 3584 + 144);
  const uint32_t p_u = sb + C::OFF_P;   // the per-tile value arm's P
  const __nv_bfloat16* bvs = reinterpret_cast<const __nv_bfloat16*>(smem + C::OFF_BV);
  __shared__ int s_fail;

  const uint32_t b0 = smem_u32(bars);
  auto kfull = [&](int s) { return b0 + 8 * s; };
  auto vfull = [&](int s) { return b0 + 16 + 8 * s; };
  auto kempty = [&](int s) { return b0 + 32 + 8 * s; };
  auto vempty = [&](int s) { return b0 + 48 + 8 * s; };
  const uint32_t qbar = b0 + 64, bvbar = b0 + 72, dkfull = b0 + 80, kaready = b0 + 88;
  const uint32_t sfull = b0 + 96, staken = b0 + 104, pfull = b0 + 112, pvdone = b0 + 120;
  const uint32_t dvfull = b0 + 128, varready = b0 + 136;   // the per-tile value arm

  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int gq = lane >> 2, t4 = lane & 3;
  const int seq = blockIdx.z;
  const int agent = blockIdx.y / p.n_kv, kvh = blockIdx.y % p.n_kv;
  const int lra = p.lr_agent ? agent : 0;   // the agent's own LR cache, or the shared one
  const int g = p.g, na = p.n_agents;
  const int QB = PM / g;
  // the split launch covers the blocks from p.blk0 on (the whole-CTA launch from 0)
  const int tok0 = ((KS > 1 ? p.blk0 : 0) + (int)(blockIdx.x / ksplit)) * QB;
  const int ntok = min(QB, p.n_q_tokens - tok0);
  const int64_t qmin = p.q_pos0 + tok0;               // position of the block's first token
  const int64_t kend = qmin + ntok;                    // keys [0, kend)
  const int N = (int)((kend + PKT - 1) / PKT);
  // key split over a CTA pair (a cluster of two): half 0 takes tiles [0, T0),
  // half 1 tiles [T0, N) and hands its partial (O, O_lr, m, l) to half 0
  const int half = ksplit > 1 ? (int)cluster_ctarank() : 0;
  const int T0 = ksplit > 1 ? max(1, N / 2) : N;
  const int nb = half ? T0 : 0;          // first tile of this CTA
  const int NT = half ? N - T0 : T0;     // tiles of this CTA (local index 0 .. NT-1)
  const bool work = KS == 1 || NT > 0;   // half 1 of a one-tile block has no keys

  // lr_col: 0 for the LRk columns (with K), r for LRv (with V)
  auto load_stage = [&](const CUtensorMap* m, uint32_t base, uint32_t bar, int n, int lr_col) {
    const int key0 = (nb + n) * PKT;
    mbar_expect_tx(bar, (uint32_t)(C::KV + PKT * R * 2));
#pragma unroll
    for (int b = 0; b < D / 64; ++b) tma_load_4d(base + b * PKT * 128, m, bar, 64 * b, key0, kvh, seq);
    tma_load_4d(base + C::KV, &tmL, bar, lr_col, key0, seq, lra);
  };
  auto load_k = [&](int n) { load_stage(&tmK, k_u + (n & 1) * C::STAGE, kfull(n & 1), n, 0); };
  auto load_v = [&](int n) { load_stage(&tmV, v_u + (n % C::NV) * C::STAGE, vfull(n % C::NV), n, R); };

  if (w == PNC && lane == 0) {
    s_fail = 0;
    for (int s = 0; s < 2; ++s) {
      mbar_init(kfull(s), 1);
      mbar_init(vfull(s), 1);
      mbar_init(kempty(s), 1);
      mbar_init(vempty(s), 1);
    }
    mbar_init(qbar, 1);
    mbar_init(bvbar, 1);
    mbar_init(dkfull, 1);
    mbar_init(kaready, PNC);
    mbar_init(sfull, 1);
    mbar_init(staken, PNC);
    mbar_init(pfull, PNC);
    mbar_init(pvdone, 1);
    mbar_init(dvfull, 1);
    mbar_init(varready, PNC);
    fence_mbar_init();
    tma_prefetch(&tmQ);
    tma_prefetch(&tmB);
    tma_prefetch(&tmK);
    tma_prefetch(&tmV);
    tma_prefetch(&tmL);
    if (work) {
      // the block's rows: g heads of each of its tokens, two 64-column boxes
      mbar_expect_tx(qbar, (uint32_t)(C::Q_BYTES + C::B_BYTES));
#pragma unroll
      for (int b = 0; b < D / 64; ++b)
        tma_load_4d(q_u + b * PM * 128, &tmQ, qbar, 64 * b, kvh * g, tok0, seq * na + agent);
#pragma unroll
      for (int b = 0; b < D / 64; ++b)
        tma_load_3d(bk_u + b * R * 128, &tmB, qbar, kvh * D + 64 * b, 0, agent);
      load_k(0);
      load_v(0);
      if (NT > 1) {
        load_k(1);
        if (C::NV > 1) load_v(1);
      }
    }
    if constexpr (VT) {  // B_v^a, the B operand of dV (every CTA)
      tma_prefetch(&tmBv);
      mbar_expect_tx(bvbar, (uint32_t)C::B_BYTES);
#pragma unroll
      for (int b = 0; b < D / 64; ++b)
        tma_load_3d(bv_u + b * R * 128, &tmBv, bvbar, kvh * D + 64 * b, 0, agent);
    } else if (half == 0) {  // B_v^a: only the CTA that writes the output
      const __nv_bfloat16* Bv = reinterpret_cast<const __nv_bfloat16*>(p.B_v);
      mbar_expect_tx(bvbar, (uint32_t)C::B_BYTES);
      for (int j = 0; j < R; ++j)
        bulk_load(bv_u + j * D * 2, Bv + ((int64_t)agent * R + j) * p.n_kv * D + kvh * D, D * 2, bvbar);
    }
  }
  if (w == PNC) tmem_alloc(smem_u32(tslot), T_COLS);

  // ---- compute-warp constants: R(j) for the two keys of the build fragment,
  // frequencies, and the first two tiles' anchors s R(k0)
  const int sp = w & 3, ch = w >> 2;
  const int kb = 32 * sp + 16 * ch;   // build: this warp's 16 keys (its TMEM lanes)
  // (cos, cos) and (sin, sin) f16 pairs over two adjacent frequencies: the
  // operands of the packed f16x2 rotation
  uint32_t RC[4][2][2], RS[4][2][2];
  if (w < PNC) {
#pragma unroll
    for (int grp = 0; grp < 4; ++grp)
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int i = 16 * grp + 8 * q + 2 * t4;
        const float th0 = rt.thetaf[i], th1 = rt.thetaf[i + 1];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const float j = (float)(kb + gq + 8 * hh);
          const float2 a = sincos_small(j * th0), b = sincos_small(j * th1);
          RC[grp][hh][q] = h2_bits(__floats2half2_rn(a.x, b.x));
          RS[grp][hh][q] = h2_bits(__floats2half2_rn(a.y, b.y));
        }
      }
  }
  if (tid < D / 2) theta[tid] = rt.theta[tid];
  if (tid < 2 * (D / 2)) {
    const int n = tid / (D / 2), i = tid % (D / 2);
    const float2 cs = rope_cs_exact((int64_t)(nb + n) * PKT, rt.theta[i]);
    anc[n * 64 + i] = make_float2(cs.x * p.s, cs.y * p.s);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  int fail = 0;

  if (w == PNC) {
    // ============================================================ TMA / MMA warp
    if (lane == 0 && work) {
      constexpr uint32_t ID_DK = umma_idesc_bf16(128, PD, 0, 1);
      constexpr uint32_t ID_S = umma_idesc_f16(128, PKT, 0, 0);   // Q and K^a in fp16
      constexpr uint32_t ID_PV = umma_idesc_bf16(128, PD, 0, 1);
      constexpr uint32_t ID_PL = umma_idesc_bf16(128, R, 0, 1);
      // operand descriptors of stage 0; the others are fixed byte offsets on
      const uint64_t dQ = umma_desc(q_u, 16, 1024, 2);
      const uint64_t dK = umma_desc(k_u, 16, 1024, 2);
      const uint64_t dLRk = umma_desc(k_u + C::KV, 16, 8 * C::LR_ROWB, C::LR_LAYOUT);
      const uint64_t dBk = umma_desc(bk_u, R * 128, 1024, 2);
      const uint64_t dV = umma_desc(v_u, PKT * 128, 1024, 2);
      const uint64_t dLRv = umma_desc(v_u + C::KV, PKT * C::LR_ROWB, 8 * C::LR_ROWB, C::LR_LAYOUT);
      // the per-tile value arm: LRv as the K-major A operand of dV, B_v^a, P
      const uint64_t dLRvA = umma_desc(v_u + C::KV, 16, 8 * C::LR_ROWB, C::LR_LAYOUT);
      const uint64_t dBv = umma_desc(bv_u, R * 128, 1024, 2);
      const uint64_t dPs = umma_desc(p_u, 16, 1024, 2);
      auto mma_dk = [&](int n) {  // dK = LRk B_k^a
        if (!mbar_wait(kfull(n & 1), (n >> 1) & 1)) fail = 1;
        tc_fence_after();
        const uint64_t lr = umma_desc_add(dLRk, (n & 1) * C::STAGE);
#pragma unroll
        for (int ks = 0; ks < R / 16; ++ks)
          umma_bf16(tmem + T_DK, umma_desc_add(lr, ks * 32), umma_desc_add(dBk, ks * 16 * 128), ID_DK, ks > 0);
        umma_commit(dkfull);
      };
      auto mma_dv = [&](int n) {  // dV = LRv B_v^a (the per-tile value arm)
        if (!mbar_wait(vfull(n % C::NV), (n / C::NV) & 1)) fail = 1;
        tc_fence_after();
        const uint64_t lr = umma_desc_add(dLRvA, (n % C::NV) * C::STAGE);
#pragma unroll
        for (int ks = 0; ks < R / 16; ++ks)
          umma_bf16(tmem + T_DV, umma_desc_add(lr, ks * 32), umma_desc_add(dBv, ks * 16 * 128), ID_DK, ks > 0);
        umma_commit(dvfull);
      };
      auto mma_pv = [&](int n) {  // O += P V_base, O_lr += P LR (the per-tile arm: O += P V^a)
        if (!mbar_wait(pfull, n & 1)) fail = 1;
        if (!mbar_wait(vfull(n % C::NV), (n / C::NV) & 1)) fail = 1;
        if (VT && !mbar_wait(varready, n & 1)) fail = 1;
        tc_fence_after();
        const uint64_t vd = umma_desc_add(dV, (n % C::NV) * C::STAGE);
        const uint64_t ld = umma_desc_add(dLRv, (n % C::NV) * C::STAGE);
        const uint32_t acc = n > 0 ? 1u : 0u;
        if constexpr (VT) {
#pragma unroll
          for (int ks = 0; ks < PKT / 16; ++ks)
            umma_bf16(tmem + TO, umma_desc_add(dPs, (ks >> 2) * (PM * 128) + (ks & 3) * 32),
                      umma_desc_add(vd, ks * 16 * 128), ID_PV, ks > 0 ? 1u : acc);
          umma_commit(pvdone);
          umma_commit(vempty(n % C::NV));
          return;
        }
#pragma unroll
        for (int ks = 0; ks < PKT / 16; ++ks)
          umma_bf16_ts(tmem + T_O, tmem + T_P + ks * 8, umma_desc_add(vd, ks * 16 * 128), ID_PV,
                       ks > 0 ? 1u : acc);
#pragma unroll
        for (int ks = 0; ks < PKT / 16; ++ks)
          umma_bf16_ts(tmem + T_OL, tmem + T_P + ks * 8, umma_desc_add(ld, ks * 16 * C::LR_ROWB), ID_PL,
                       ks > 0 ? 1u : acc);
        umma_commit(pvdone);
        umma_commit(vempty(n % C::NV));
      };
      if (!mbar_wait(qbar, 0)) fail = 1;
      if (VT && !mbar_wait(bvbar, 0)) fail = 1;
      mma_dk(0);
      for (int n = 0; n < NT; ++n) {
        if (!mbar_wait(kaready, n & 1)) fail = 1;
        if (n > 0 && !mbar_wait(staken, (n - 1) & 1)) fail = 1;
        tc_fence_after();
        const uint64_t kd = umma_desc_add(dK, (n & 1) * C::STAGE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          umma_bf16(tmem + T_S, umma_desc_add(dQ, (kk >> 2) * (PM * 128) + (kk & 3) * 32),
                    umma_desc_add(kd, (kk >> 2) * (PKT * 128) + (kk & 3) * 32), ID_S, kk > 0);
        umma_commit(sfull);
        umma_commit(kempty(n & 1));
        if (n + 1 < NT) mma_dk(n + 1);
        if (n > 0) mma_pv(n - 1);
        if constexpr (VT) mma_dv(n);   // dV(n-1) has been read: P V(n-1) waited for V^a(n-1)
      }
      mma_pv(NT - 1);
      // loads in flight when the loop ends are all consumed: every issued tile is used
    }
    __syncwarp();
    if (ksplit > 1) {
      cluster_sync_all();
      cluster_sync_all();
    }
  } else if (w == PNC + 1) {
    // ============================================================ TMA refill warp
    // refills in the order the MMAs free the stages (S of tile n, then P V of
    // tile n-1), so that the MMA warp never waits for an MMA to finish
    if (lane == 0) {
      for (int n = 0; n < NT; ++n) {
        if (n + 2 < NT) {
          if (!mbar_wait(kempty(n & 1), (n >> 1) & 1)) fail = 1;   // S_n has read K^a_n
          load_k(n + 2);
        }
        if (n > 0 && n - 1 + C::NV < NT) {  // V stage of tile n-1 is free once its P V is done
          if (!mbar_wait(vempty((n - 1) % C::NV), ((n - 1) / C::NV) & 1)) fail = 1;
          load_v(n - 1 + C::NV);
        }
      }
    }
    __syncwarp();
    if (ksplit > 1) {
      cluster_sync_all();
      cluster_sync_all();
    }
  } else {
    // ============================================================ compute warps
    const float sl2 = p.scale * kLog2e;
    const int row = 32 * sp + lane;          // softmax: this thread's query row (TMEM lane)
    const int rtok = row / g;
    const bool rvalid = rtok < ntok;
    const int64_t qpos = qmin + rtok;
    float m_ref = -INFINITY, lsum = 0.f;

    auto build = [&](int n) {  // K^a = K_base + s R(k0) R(j) dK, over K_base in place
      if (!mbar_wait(dkfull, n & 1)) fail = 1;
      if (!mbar_wait(kfull(n & 1), (n >> 1) & 1)) fail = 1;
      tc_fence_after();
      const uint32_t kst = k_u + (n & 1) * C::STAGE;
      const float2* an = anc + (n & 1) * 64;
      const uint32_t tl = tmem + T_DK + ((uint32_t)kb << 16);
      // this lane's pair of K elements in a 128-byte-swizzled row: key kb + gq
      // (+8), 16-byte chunk (2 grp + q) ^ gq, word t4; columns + d/2 are one box on
      const uint32_t rowb = kst + (uint32_t)(kb + gq) * 128 + 4 * t4;
#pragma unroll
      for (int grp = 0; grp < 4; ++grp) {
        uint32_t xl[8], xh[8];
        tmem_ld16x256_x2(xl, tl + 16 * grp);
        tmem_ld16x256_x2(xh, tl + 16 * grp + D / 2);
        tmem_wait_ld_regs(xl, xh);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int i0 = 16 * grp + 8 * q + 2 * t4;
          const float2 a0 = an[i0], a1 = an[i0 + 1];
          const __half2 ac = __floats2half2_rn(a0.x, a1.x), as = __floats2half2_rn(a0.y, a1.y);
          const __half2 nas = __hneg2(as);
          const uint32_t cx = (uint32_t)(((2 * grp + q) ^ gq) << 4);
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            // in f16x2 arithmetic: the delta pairs, R(j) dK, then K_base + s R(k0) y
            // with the base added inside the rotation's FMAs
            const __half2 x1 = __floats2half2_rn(__uint_as_float(xl[4 * q + 2 * hh]), __uint_as_float(xl[4 * q + 2 * hh + 1]));
            const __half2 x2 = __floats2half2_rn(__uint_as_float(xh[4 * q + 2 * hh]), __uint_as_float(xh[4 * q + 2 * hh + 1]));
            const __half2 c = bits_h2(RC[grp][hh][q]), sn = bits_h2(RS[grp][hh][q]);
            const __half2 y1 = __hfma2(x1, c, __hneg2(__hmul2(x2, sn)));   // R(j) dK
            const __half2 y2 = __hfma2(x2, c, __hmul2(x1, sn));
            const uint32_t o1 = rowb + hh * 1024 + cx, o2 = o1 + PKT * 128;
            const __half2 z1 = __hfma2(ac, y1, __hfma2(nas, y2, bf16x2_h2(lds32(o1))));
            const __half2 z2 = __hfma2(ac, y2, __hfma2(as, y1, bf16x2_h2(lds32(o2))));
            sts32(o1, h2_bits(z1));
            sts32(o2, h2_bits(z2));
          }
        }
      }
      fence_proxy_async_smem();  // the S MMA reads K^a through the async proxy
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(kaready);
    };

    auto softmax = [&](int n) {
      if (!mbar_wait(sfull, n & 1)) fail = 1;
      tc_fence_after();
      const uint32_t ts = tmem + T_S + 64 * ch + ((uint32_t)(32 * sp) << 16);
      uint32_t sv[2][32];
      tmem_ld32x32b_x32(sv[0], ts);
      tmem_ld32x32b_x32(sv[1], ts + 32);
      tmem_wait_ld_r32(sv[0]);
      tmem_wait_ld_r32(sv[1]);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(staken);  // S may be overwritten by the next tile's MMA

      // row maximum of the raw scores (the scale is positive); keys past a row's
      // position are set to -inf (only the tiles that reach the block's first
      // position need it; rows past the chunk are never written out)
      const int64_t key0 = (int64_t)(nb + n) * PKT + 64 * ch;
      if (key0 + 63 > qmin) {
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (key0 + 32 * h + c > qpos) sv[h][c] = __float_as_uint(-INFINITY);
      }
      float mr[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float m = __uint_as_float(sv[h][0]);
#pragma unroll
        for (int c = 1; c < 31; c += 2) m = max3f(m, __uint_as_float(sv[h][c]), __uint_as_float(sv[h][c + 1]));
        mr[h] = fmaxf(m, __uint_as_float(sv[h][31]));
      }
      const float mloc = fmaxf(mr[0], mr[1]) * sl2;
      float* xb = xch + (n & 1) * 256;
      xb[w * 32 + lane] = mloc;
      bar_sync(PBAR_PAIR + sp, 64);
      const float mt = fmaxf(mloc, xb[(w ^ 4) * 32 + lane]);
      // lazy rescale: move the reference max only when a row's max grew by > 8
      const bool need = mt > m_ref + 8.f || (m_ref == -INFINITY && mt != -INFINITY);
      if (__any_sync(0xffffffffu, need)) {
        const float m_new = fmaxf(m_ref, mt);
        const float corr = m_ref == -INFINITY ? 0.f : fast_exp2(m_ref - m_new);
        if (n > 0 && __any_sync(0xffffffffu, m_ref != -INFINITY)) {
          if (!mbar_wait(pvdone, (n - 1) & 1)) fail = 1;  // O holds every tile before this one
          tc_fence_after();
          const uint32_t to = tmem + TO + 64 * ch + ((uint32_t)(32 * sp) << 16);
#pragma unroll 1
          for (int h = 0; h < 4; ++h) {
            uint32_t ov[16];
            tmem_ld32x32b_x16(ov, to + 16 * h);
            tmem_wait_ld_r16(ov);
#pragma unroll
            for (int c = 0; c < 16; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * corr);
            tmem_st32x32b_x16(to + 16 * h, ov);
          }
          if (!VT && ch == 0) {
            const uint32_t tol = tmem + T_OL + ((uint32_t)(32 * sp) << 16);
#pragma unroll 1
            for (int h = 0; h < R / 16; ++h) {
              uint32_t ov[16];
              tmem_ld32x32b_x16(ov, tol + 16 * h);
              tmem_wait_ld_r16(ov);
#pragma unroll
              for (int c = 0; c < 16; ++c) ov[c] = __float_as_uint(__uint_as_float(ov[c]) * corr);
              tmem_st32x32b_x16(tol + 16 * h, ov);
            }
          }
          tmem_wait_st();
        }
        lsum *= corr;
        m_ref = m_new;
      }
      // p = 2^(S scale log2e - m): one packed fma per pair, then the SFU
      const float mu = m_ref == -INFINITY ? 0.f : m_ref;   // rows with no visible key yet: p = 0
      const uint64_t scl = f2(sl2, sl2), nmu = f2(-mu, -mu);
      uint32_t pk[32];
      uint64_t acc = f2(0.f, 0.f);
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const uint64_t xa2 = fma_f2(f2(__uint_as_float(sv[h][c]), __uint_as_float(sv[h][c + 1])), scl, nmu);
          float p0, p1;
          if (kPolyExpEvery > 0 && (c / 2) % (kPolyExpEvery > 0 ? kPolyExpEvery : 1) == 0) {
            const float2 pp = f2_unpack(exp2_poly_f2(xa2));
            p0 = pp.x;
            p1 = pp.y;
          } else {
            const float2 xa = f2_unpack(xa2);
            p0 = fast_exp2(xa.x);
            p1 = fast_exp2(xa.y);
          }
          acc = add_f2(acc, f2(p0, p1));
          pk[16 * h + c / 2] = pack_bf16(p0, p1);
        }
      const float2 accf = f2_unpack(acc);
      const float ls = accf.x + accf.y;
      lsum += ls;
      if (n > 0 && !mbar_wait(pvdone, (n - 1) & 1)) fail = 1;  // the P V MMA of tile n-1 is done
      tc_fence_after();
      if constexpr (VT) {   // P into shared memory: row `row`, keys 64 ch .. +63 (one 128-byte-swizzled box row)
        const uint32_t prow = p_u + (uint32_t)ch * (PM * 128) + (uint32_t)row * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c)
          sts128(prow + (uint32_t)((c ^ (row & 7)) << 4), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        fence_proxy_async_smem();
      } else {
        tmem_st32x32b_x32(tmem + T_P + 32 * ch + ((uint32_t)(32 * sp) << 16), pk);
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pfull);
    };

    // the per-tile value arm: V^a = V_base + s dV over V_base in shared memory;
    // this thread: key 32 sp + lane, the 64 columns of box ch
    auto vbuild = [&](int n) {
      if (!mbar_wait(dvfull, n & 1)) fail = 1;
      tc_fence_after();
      const int key = 32 * sp + lane;
      uint32_t dv[2][32];
      const uint32_t td = tmem + T_DV + 64 * ch + ((uint32_t)(32 * sp) << 16);
      tmem_ld32x32b_x32(dv[0], td);
      tmem_ld32x32b_x32(dv[1], td + 32);
      tmem_wait_ld_r32(dv[0]);
      tmem_wait_ld_r32(dv[1]);
      const uint32_t vrow = v_u + (uint32_t)(n % C::NV) * C::STAGE + (uint32_t)ch * (PKT * 128) + (uint32_t)key * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c) {   // 8 columns a 16-byte chunk
        const uint32_t a = vrow + (uint32_t)((c ^ (key & 7)) << 4);
        const uint4 v = lds128(a);
        const uint32_t* d8 = dv[c >> 2] + 8 * (c & 3);
        const float2 b0 = unpack_bf16(v.x), b1 = unpack_bf16(v.y), b2 = unpack_bf16(v.z), b3 = unpack_bf16(v.w);
        sts128(a, pack_bf16(fmaf(p.s, __uint_as_float(d8[0]), b0.x), fmaf(p.s, __uint_as_float(d8[1]), b0.y)),
               pack_bf16(fmaf(p.s, __uint_as_float(d8[2]), b1.x), fmaf(p.s, __uint_as_float(d8[3]), b1.y)),
               pack_bf16(fmaf(p.s, __uint_as_float(d8[4]), b2.x), fmaf(p.s, __uint_as_float(d8[5]), b2.y)),
               pack_bf16(fmaf(p.s, __uint_as_float(d8[6]), b3.x), fmaf(p.s, __uint_as_float(d8[7]), b3.y)));
      }
      fence_proxy_async_smem();   // the P V MMA reads V^a through the async proxy
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(varready);
    };

    if (work) {
      // the queries to fp16 in place: the S MMA takes Q and K^a in fp16, whose
      // 11-bit significand keeps the rounding of K^a = K_base + delta small
      // against |K| (bf16 values convert exactly within fp16's range)
      if (!mbar_wait(qbar, 0)) fail = 1;
      for (int i = tid; i < C::Q_BYTES / 16; i += 32 * PNC) {
        uint4* qp = reinterpret_cast<uint4*>(smem + C::OFF_Q) + i;
        uint4 v = *qp;
        v.x = add_to_f16x2(v.x, make_float2(0.f, 0.f));
        v.y = add_to_f16x2(v.y, make_float2(0.f, 0.f));
        v.z = add_to_f16x2(v.z, make_float2(0.f, 0.f));
        v.w = add_to_f16x2(v.w, make_float2(0.f, 0.f));
        *qp = v;
      }
      build(0);   // its proxy fence also covers the queries
    }
    for (int i = 0; i < NT; ++i) {
      bar_sync(PBAR_CW, 32 * PNC);  // anchors of tile i+1 are in place
      if (i + 1 < NT) build(i + 1);
      softmax(i);
      if constexpr (VT) vbuild(i);
      if (tid < D / 2 && i + 2 < NT) {
        const float2 cs = rope_cs_exact((int64_t)(nb + i + 2) * PKT, theta[tid]);
        anc[(i & 1) * 64 + tid] = make_float2(cs.x * p.s, cs.y * p.s);
      }
    }

    // half 1's partial goes to its drained K / V stages: O as float4 [d/4][128
    // rows], O_lr as float4 [r/4][128 rows], then m_ref and l per row
    const uint32_t xo = k_u, xl = xo + PM * PD * 4, xm = xl + PM * R * 4, xs = xm + PM * 4;
    if constexpr (KS > 1) {
      if (half == 1) {
        if (work) {
          if (!mbar_wait(pvdone, (NT - 1) & 1)) fail = 1;
          tc_fence_after();
          float* lx = xch + (NT & 1) * 256;  // the exchange buffer the last softmax did not use
          lx[w * 32 + lane] = lsum;
          bar_sync(PBAR_PAIR + sp, 64);
          const float l = lsum + lx[(w ^ 4) * 32 + lane];
#pragma unroll 1
          for (int h = 0; h < 4; ++h) {
            uint32_t ov[16];
            tmem_ld32x32b_x16(ov, tmem + TO + 64 * ch + 16 * h + ((uint32_t)(32 * sp) << 16));
            tmem_wait_ld_r16(ov);
#pragma unroll
            for (int c = 0; c < 16; c += 4)
              sts128(xo + (uint32_t)(((64 * ch + 16 * h + c) / 4) * PM + row) * 16, ov[c], ov[c + 1], ov[c + 2],
                     ov[c + 3]);
          }
          if (ch == 0) {
#pragma unroll 1
            for (int h = 0; h < (VT ? 0 : R / 16); ++h) {
              uint32_t t16[16];
              tmem_ld32x32b_x16(t16, tmem + T_OL + 16 * h + ((uint32_t)(32 * sp) << 16));
              tmem_wait_ld_r16(t16);
#pragma unroll
              for (int c = 0; c < 16; c += 4)
                sts128(xl + (uint32_t)(((16 * h + c) / 4) * PM + row) * 16, t16[c], t16[c + 1], t16[c + 2],
                       t16[c + 3]);
            }
            sts32(xm + row * 4, __float_as_uint(m_ref));
            sts32(xs + row * 4, __float_as_uint(l));
          }
        }
        cluster_sync_all();  // the partial is in place
        cluster_sync_all();  // half 0 has read it
      }
    }
    if (half == 0) {
    // ---- epilogue: out = (O + s O_lr B_v^a) / l for this warp's 64 columns
    // (the per-tile value arm: out = O / l)
    if (!mbar_wait(pvdone, (NT - 1) & 1)) fail = 1;
    if (!mbar_wait(bvbar, 0)) fail = 1;
    tc_fence_after();
    float* lx = xch + (NT & 1) * 256;  // the exchange buffer the last softmax did not use
    lx[w * 32 + lane] = lsum;
    bar_sync(PBAR_PAIR + sp, 64);
    float l = lsum + lx[(w ^ 4) * 32 + lane];
    uint32_t olr[R];   // P LRv, this thread's row (the reordered arm)
#pragma unroll
    for (int h = 0; h < (VT ? 0 : R / 16); ++h) {
      uint32_t t16[16];
      tmem_ld32x32b_x16(t16, tmem + T_OL + 16 * h + ((uint32_t)(32 * sp) << 16));
      tmem_wait_ld_r16(t16);
#pragma unroll
      for (int c = 0; c < 16; ++c) olr[16 * h + c] = t16[c];
    }
    // with split keys: merge with half 1's partial, both rescaled to the larger
    // of the two reference maxima
    float a0 = 1.f, a1 = 0.f;
    bool merge = false;
    if constexpr (KS > 1) {
      cluster_sync_all();
      merge = N - T0 > 0;
      if (merge) {
        const float m1 = dsmem_ld(dsmem_addr(xm + row * 4, 1));
        const float l1 = dsmem_ld(dsmem_addr(xs + row * 4, 1));
        const float M = fmaxf(m_ref, m1);
        a0 = m_ref == -INFINITY ? 0.f : fast_exp2(m_ref - M);
        a1 = m1 == -INFINITY ? 0.f : fast_exp2(m1 - M);
        l = a0 * l + a1 * l1;
#pragma unroll
        for (int j = 0; j < (VT ? 0 : R); j += 4) {
          const float4 r4 = dsmem_ld4(dsmem_addr(xl + (uint32_t)((j / 4) * PM + row) * 16, 1));
          olr[j] = __float_as_uint(fmaf(a0, __uint_as_float(olr[j]), a1 * r4.x));
          olr[j + 1] = __float_as_uint(fmaf(a0, __uint_as_float(olr[j + 1]), a1 * r4.y));
          olr[j + 2] = __float_as_uint(fmaf(a0, __uint_as_float(olr[j + 2]), a1 * r4.z));
          olr[j + 3] = __float_as_uint(fmaf(a0, __uint_as_float(olr[j + 3]), a1 * r4.w));
        }
      }
    }
    const float inv_l = l > 0.f ? 1.f / l : 0.f;
    const int head = kvh * g + row % g;
    const int64_t obase = (((int64_t)seq * na + agent) * p.n_q_tokens + tok0 + rtok) * p.n_q + head;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      uint32_t ov[32];
      tmem_ld32x32b_x32(ov, tmem + TO + 64 * ch + 32 * h + ((uint32_t)(32 * sp) << 16));
      tmem_wait_ld_r32(ov);
      if constexpr (KS > 1) {
        if (merge) {
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            const float4 r4 =
                dsmem_ld4(dsmem_addr(xo + (uint32_t)(((64 * ch + 32 * h + c) / 4) * PM + row) * 16, 1));
            ov[c] = __float_as_uint(fmaf(a0, __uint_as_float(ov[c]), a1 * r4.x));
            ov[c + 1] = __float_as_uint(fmaf(a0, __uint_as_float(ov[c + 1]), a1 * r4.y));
            ov[c + 2] = __float_as_uint(fmaf(a0, __uint_as_float(ov[c + 2]), a1 * r4.z));
            ov[c + 3] = __float_as_uint(fmaf(a0, __uint_as_float(ov[c + 3]), a1 * r4.w));
          }
        }
      }
      float z[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) z[c] = 0.f;
#pragma unroll
      for (int j = 0; j < (VT ? 0 : R); ++j) {   // the per-tile arm has V^a in O already
        const float o = __uint_as_float(olr[j]);
        const __nv_bfloat16* brow = bvs + j * D + 64 * ch + 32 * h;
#pragma unroll
        for (int c = 0; c < 32; c += 2) {
          const float2 bb = unpack_bf16(*reinterpret_cast<const uint32_t*>(brow + c));
          z[c] = fmaf(o, bb.x, z[c]);
          z[c + 1] = fmaf(o, bb.y, z[c + 1]);
        }
      }
      if (rvalid) {
        const int64_t oi = obase * D + 64 * ch + 32 * h;
        if (p.out_bf16) {
          uint32_t* o = reinterpret_cast<uint32_t*>(reinterpret_cast<__nv_bfloat16*>(p.out) + oi);
#pragma unroll
          for (int c = 0; c < 32; c += 2)
            o[c / 2] = pack_bf16(fmaf(p.s, z[c], __uint_as_float(ov[c])) * inv_l,
                                 fmaf(p.s, z[c + 1], __uint_as_float(ov[c + 1])) * inv_l);
        } else {
          float4* o = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.out) + oi);
#pragma unroll
          for (int c = 0; c < 32; c += 4)
            o[c / 4] = make_float4(fmaf(p.s, z[c], __uint_as_float(ov[c])) * inv_l,
                                   fmaf(p.s, z[c + 1], __uint_as_float(ov[c + 1])) * inv_l,
                                   fmaf(p.s, z[c + 2], __uint_as_float(ov[c + 2])) * inv_l,
                                   fmaf(p.s, z[c + 3], __uint_as_float(ov[c + 3])) * inv_l);
        }
      }
    }
    if constexpr (KS > 1) cluster_sync_all();
    }
  }
  if (fail) s_fail = 1;
  tc_fence_before();
  __syncthreads();
  if (w == PNC) {
    tc_fence_after();
    tmem_dealloc(tmem, T_COLS);
  }
  if (s_fail && tid == 0) atomicOr(p.err, 2);
}

// ------------------------------------------------------------------ host
bool prefill_maps(const AttnParams& p, CUtensorMap* mq, CUtensorMap* mk, CUtensorMap* mv,
                  CUtensorMap* ml, CUtensorMap* mb, CUtensorMap* mbv) {
  auto enc = encode_fn();
  if (!enc) return false;
  const int D = PD, R = p.r, g = p.g;
  cuuint32_t one[4] = {1, 1, 1, 1};
  // queries [n_seqs * n_agents][n_tok][n_q][d]: boxes of 64 columns x g heads x 128/g tokens
  cuuint64_t qd[4] = {(cuuint64_t)D, (cuuint64_t)p.n_q, (cuuint64_t)p.n_q_tokens,
                      (cuuint64_t)p.n_seqs * p.n_agents};
  cuuint64_t qs[3] = {(cuuint64_t)D * 2, (cuuint64_t)p.n_q * D * 2,
                      (cuuint64_t)p.n_q_tokens * p.n_q * D * 2};
  cuuint32_t qb[4] = {64, (cuuint32_t)g, (cuuint32_t)(PM / g), 1};
  if (enc(mq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(p.q), qd, qs, qb, one,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  cuuint64_t kd[4] = {(cuuint64_t)D, (cuuint64_t)p.L_max, (cuuint64_t)p.n_kv, (cuuint64_t)p.n_seqs};
  cuuint64_t ks[3] = {(cuuint64_t)p.kv_tok * 2, (cuuint64_t)p.kv_head * 2, (cuuint64_t)p.kv_seq * 2};
  cuuint32_t kb[4] = {64, (cuuint32_t)PKT, 1, 1};
  if (enc(mk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(p.k_base), kd, ks, kb, one,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  if (enc(mv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(p.v_base), kd, ks, kb, one,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  // LR rows [2r]: boxes of r columns (LRk at column 0, LRv at column r), in
  // [n_lr][n_seqs][L_max][2r]: one shared cache, or one per agent
  const int64_t n_lr = p.lr_agent ? p.n_agents : 1;
  const int64_t lr_agent_b = p.lr_agent ? p.lr_agent * 2 : p.lr_seq * 2 * p.n_seqs;
  cuuint64_t ld[4] = {(cuuint64_t)(2 * R), (cuuint64_t)p.L_max, (cuuint64_t)p.n_seqs, (cuuint64_t)n_lr};
  cuuint64_t ls[3] = {(cuuint64_t)(2 * R * 2), (cuuint64_t)p.lr_seq * 2, (cuuint64_t)lr_agent_b};
  cuuint32_t lbx[4] = {(cuuint32_t)R, (cuuint32_t)PKT, 1, 1};
  if (enc(ml, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(p.lr), ld, ls, lbx, one,
          CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle_for(R * 2), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  // B_k as (n_kv * d, r, n_agents): r x 64 slices of one head
  cuuint64_t bd[3] = {(cuuint64_t)p.n_kv * D, (cuuint64_t)R, (cuuint64_t)p.n_agents};
  cuuint64_t bs[2] = {(cuuint64_t)p.n_kv * D * 2, (cuuint64_t)R * p.n_kv * D * 2};
  cuuint32_t bb[3] = {64, (cuuint32_t)R, 1};
  if (enc(mb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(p.B_k), bd, bs, bb, one,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  // B_v the same way (the per-tile value arm's dV operand)
  if (enc(mbv, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(p.B_v), bd, bs, bb, one,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  return true;
}

// Which blocks of rows run as whole CTAs and which as key halves on CTA pairs
// (KS = 2): the first nA blocks whole, the rest split, in two launches.  The
// CTAs of one wave run about equally long, so a launch takes ceil(CTAs /
// resident CTAs) waves; a half costs more than half a CTA (its own start-up,
// pipeline fill and the merge: about 15 % measured at 65 tiles a half).  The
// split pays where whole CTAs would leave SMs idle -- fewer CTAs than SMs, or
// a last wave that is mostly empty (768 CTAs on 148 SMs: 720 whole in 5 waves,
// the last two blocks' 48 as 96 halves in one half-length wave, instead of
// 6 waves).  Returns nA in [0, nblk].
template <int R, bool VT>
int prefill_whole_blocks(const AttnParams& p, int nblk) {
  using C = PCfg<R, VT>;
  const int64_t tiles = (p.q_pos0 + p.n_q_tokens + PKT - 1) / PKT;
  if (tiles < 4) return nblk;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1) {
    cudaGetLastError();
    return nblk;
  }
  static int pairs[2][64] = {};   // resident CTA pairs per device (0: not queried yet)
  int& np = pairs[VT ? 1 : 0][dev & 63];
  if (np == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (unsigned)sms, 1, 1);
    cfg.blockDim = dim3(PNTHR);
    cfg.dynamicSmemBytes = C::SMEM;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaFuncSetAttribute(prefill_tc_kernel<R, 2, VT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)C::SMEM) != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&n, prefill_tc_kernel<R, 2, VT>, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = -1;
    }
    np = n;
  }
  if (np < 1) return nblk;
  const double per_blk = (double)p.n_agents * p.n_kv * p.n_seqs;   // CTAs (or pairs) per block
  int best = nblk;
  double best_t = std::ceil(nblk * per_blk / sms);
  for (int na = nblk - 1; na >= 0; --na) {
    const double t = std::ceil(na * per_blk / sms) + 0.5 * 1.15 * std::ceil((nblk - na) * per_blk / np);
    if (t < best_t - 1e-9) {
      best_t = t;
      best = na;
    }
  }
  return best;
}

template <int R, bool VT>
cudaError_t launch_prefill_tc(const AttnParams& p, cudaStream_t st) {
  using C = PCfg<R, VT>;
  RopeTheta rt;
  for (int i = 0; i < 64; ++i) {
    rt.theta[i] = std::pow(p.rope_base, -2.0 * i / PD);
    rt.thetaf[i] = (float)rt.theta[i];
  }
  CUtensorMap mq, mk, mv, ml, mb, mbv;
  if (!prefill_maps(p, &mq, &mk, &mv, &ml, &mb, &mbv)) return cudaErrorInvalidValue;
  const int QB = PM / p.g;
  const int nblk = (p.n_q_tokens + QB - 1) / QB;
  const int nA = prefill_whole_blocks<R, VT>(p, nblk);
  // blocks [0, nA) as whole CTAs, blocks [nA, nblk) as key halves on CTA pairs
  for (int ks = 1; ks <= 2; ++ks) {
    const int nb = ks == 1 ? nA : nblk - nA;
    if (nb == 0) continue;
    auto kern = ks > 1 ? prefill_tc_kernel<R, 2, VT> : prefill_tc_kernel<R, 1, VT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM);
    if (e != cudaSuccess) return e;
    AttnParams pk = p;
    pk.blk0 = ks > 1 ? nA : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(nb * ks), p.n_agents * p.n_kv, p.n_seqs);
    cfg.blockDim = dim3(PNTHR);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)ks;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = ks > 1 ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, kern, mq, mk, mv, ml, mb, mbv, pk, rt);
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

}  // namespace

bool bf16_prefill_supported(const AttnParams& p) {
  // r = 8 would make the P LRv MMA N = 8, below the M = 128 minimum of 16
  if (p.d != PD || !(p.r == 16 || p.r == 32 || p.r == 64)) return false;
  if (!(p.g == 1 || p.g == 2 || p.g == 4 || p.g == 8)) return false;
  if (p.L_max >= (1ll << 31) || p.n_q_tokens < 1 || p.n_q_tokens > (1 << 29)) return false;
  if ((int64_t)p.n_agents * p.n_kv > 65535 || p.n_seqs > 65535) return false;
  return PCfg<16>::SMEM <= 227 * 1024 && PCfg<32>::SMEM <= 227 * 1024 && PCfg<64>::SMEM <= 227 * 1024;
}

// The per-tile value arm (V^a rebuilt per tile): r = 16, where its P buffer
// fits beside the stages
bool bf16_prefill_per_tile_supported(const AttnParams& p) {
  return bf16_prefill_supported(p) && p.r == 16 && PCfg<16, true>::SMEM <= 227 * 1024;
}

cudaError_t launch_prefill_bf16(const AttnParams& pin, la_dtype out, cudaStream_t st) {
  AttnParams p = pin;
  p.out_bf16 = out == LA_BF16;
  if (p.value_path == LA_VALUE_PER_TILE) {
    if (!bf16_prefill_per_tile_supported(p)) return cudaErrorInvalidValue;
    return launch_prefill_tc<16, true>(p, st);
  }
  switch (p.r) {
    case 16: return launch_prefill_tc<16, false>(p, st);
    case 32: return launch_prefill_tc<32, false>(p, st);
    default: return launch_prefill_tc<64, false>(p, st);
  }
}

}  // namespace la
