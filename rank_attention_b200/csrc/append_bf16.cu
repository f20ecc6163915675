// lr_cache_append on the tensor cores (bf16 in, fp32 accumulate, bf16 out).
//
// PreLRShared precompute (PReCache abstract and blog; LRAgent summary §3
// BaseLRShared): LR[pos0 + i] = X_i [A_k | A_v], computed once per new chunk
// through the A every agent shares.  The rows are stored unscaled and
// unrotated, K part first.
//
// A CTA owns 64 chunk rows and all 2r output columns; its 8 warps split
// them as 4 row groups of 16 x 2 column halves (one half at r = 8); TMA
// stages 64 x 64 slices of X and of A_kv (128/64/32-byte swizzle, no
// multicast) through a 3-stage mbarrier pipeline, and warp-level bf16 MMAs
// accumulate in fp32.  The hidden dimension is split over the CTAs of a
// thread-block cluster so that short chunks (a single decode token) still
// spread over many SMs; the partial sums meet in distributed shared memory,
// where each CTA reduces and writes its share of the rows.
#include <cooperative_groups.h>
#include <cudaTypedefs.h>

#include "bf16_common.cuh"
#include "la_internal.cuh"
#include "ptx.cuh"

namespace la {
namespace {

namespace cg = cooperative_groups;
using namespace ptx;

constexpr int TM = 64;     // chunk rows per CTA
constexpr int KC = 64;     // hidden columns per stage
constexpr int NTHR = 256;     // 4 row groups x 2 column groups
constexpr int NSTAGE = 3;
constexpr int kMaxHS = 16;
// SMs of the current device, for splitting the hidden dimension over about
// one wave of CTAs (148 on B200, also the answer when the query fails)
int current_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) {
    cudaGetLastError();
    return 148;
  }
  return n;
}


template <int R>
struct ACfg {
  static constexpr int C = 2 * R;                       // output columns
  static constexpr int X_TILE = TM * KC * 2;            // 8 KB
  static constexpr int A_TILE = align1k(KC * C * 2);
  static constexpr int STAGE = X_TILE + A_TILE;
  static constexpr int RED = TM * C * 4;                // fp32 partial
  static constexpr int AREA = NSTAGE * STAGE > RED ? NSTAGE * STAGE : align1k(RED);
  static constexpr size_t smem = 1024 + AREA + 64;
};

template <int R>
__global__ void __launch_bounds__(NTHR, 1)
    append_bf16_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmA,
                       __nv_bfloat16* __restrict__ lr, int64_t pos0, int64_t n, int64_t slr,
                       int hs, int kchunks, int* err) {
  using Cf = ACfg<R>;
  constexpr int C = Cf::C;
  constexpr int NTN = C / 8;       // n-tiles of the output
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t area_u = smem_u32(smem);
  const uint32_t bar_u = smem_u32(smem + Cf::AREA);
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int gq = lane >> 2, t4 = lane & 3, mi = lane >> 3, rr = lane & 7;
  const int cr = blockIdx.x % hs;              // rank in the cluster = hidden split
  const int mtile = blockIdx.x / hs;
  const int seq = blockIdx.y;
  const int64_t t0 = (int64_t)mtile * TM;
  const int kb = cr * kchunks / hs, ke = (cr + 1) * kchunks / hs;
  const int nk = ke - kb;
  cg::cluster_group cluster = cg::this_cluster();

  // the next kernel of the stream (the decode of the step) may start its
  // set-up now; it waits for this grid's completion before reading the LR cache
  pdl_launch_dependents();
  if (tid == 0) {
    for (int s = 0; s < NSTAGE; ++s) mbar_init(bar_u + 8 * s, 1);
    fence_mbar_init();
    tma_prefetch(&tmX);
    tma_prefetch(&tmA);
  }
  __syncthreads();
  auto issue = [&](int j) {
    const int s = j % NSTAGE;
    const uint32_t sb = area_u + s * Cf::STAGE;
    const uint32_t bar = bar_u + 8 * s;
    const int h0 = (kb + j) * KC;
    mbar_expect_tx(bar, Cf::X_TILE + KC * C * 2);
    tma_load_3d(sb, &tmX, bar, h0, (int)t0, seq);
    constexpr int AB = C < 64 ? C : 64;
#pragma unroll
    for (int b = 0; b < C / AB; ++b) tma_load_2d_(sb + Cf::X_TILE + b * KC * AB * 2, &tmA, bar, AB * b, h0);
  };
  if (tid == 0)
    for (int j = 0; j < NSTAGE && j < nk; ++j) issue(j);

  // warp w: rows 16 (w & 3) .. +15, n-tiles [wc NTW, (wc + 1) NTW) of the output
  constexpr int CG = NTN >= 4 ? 2 : 1;   // column groups (n-tiles are taken in pairs)
  constexpr int NTW = NTN / CG;
  const int wr = w & 3, wc = w >> 2;
  const bool mma_warp = wc < CG;
  float acc[NTW][4];
#pragma unroll
  for (int q = 0; q < NTW; ++q)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[q][e] = 0.f;

  int fail = 0;
  for (int j = 0; j < nk; ++j) {
    const int s = j % NSTAGE;
    if (!mbar_wait(bar_u + 8 * s, (j / NSTAGE) & 1)) fail = 1;
    if (__syncthreads_or(fail)) {
      fail = 1;
      break;
    }
    const uint32_t sX = area_u + s * Cf::STAGE;
    const uint32_t sA = sX + Cf::X_TILE;
    if (mma_warp) {
#pragma unroll
      for (int ks = 0; ks < KC / 16; ++ks) {
        uint32_t a[4];
        ldsm_x4(a, sX + tile_off<KC, TM>(16 * wr + rr + (mi & 1) * 8, 16 * ks + (mi >> 1) * 8));
#pragma unroll
        for (int q = 0; q < NTW; q += 2) {
          uint32_t b[4];
          ldsm_x4_t(b, sA + tile_off<C, KC>(16 * ks + rr + (mi & 1) * 8, 8 * (wc * NTW + q + (mi >> 1))));
          mma16816(acc[q], a, b[0], b[1]);
          mma16816(acc[q + 1], a, b[2], b[3]);
        }
      }
    }
    __syncthreads();
    if (tid == 0 && j + NSTAGE < nk) issue(j + NSTAGE);
  }
  if (fail && tid == 0) atomicOr(err, 2);

  // partial sums -> shared memory (stage area reused), then reduce over the cluster
  __syncthreads();
  float* red = reinterpret_cast<float*>(smem);
  if (mma_warp) {
#pragma unroll
    for (int q = 0; q < NTW; ++q)
#pragma unroll
      for (int e = 0; e < 4; ++e)
        red[(16 * wr + gq + (e >> 1) * 8) * C + 8 * (wc * NTW + q) + 2 * t4 + (e & 1)] = acc[q][e];
  }
  if (hs > 1) cluster.sync();
  else __syncthreads();
  if (!fail) {
    const int rows_per = (TM + hs - 1) / hs;
    const int r0 = cr * rows_per;
    for (int i = tid; i < rows_per * C; i += NTHR) {
      const int row = r0 + i / C, c = i % C;
      if (row >= TM || t0 + row >= n) continue;
      float v = 0.f;
      for (int k = 0; k < hs; ++k) v += cluster.map_shared_rank(red, k)[row * C + c];
      lr[seq * slr + (pos0 + t0 + row) * C + c] = __float2bfloat16_rn(v);
    }
  }
  if (hs > 1) cluster.sync();
}

// ---------------------------------------------------------------------------
// r = 32 and 64: the product is a GEMM of 4 r flops per hidden element and
// token, past what warp-level MMAs sustain (about a sixteenth of the tcgen05
// rate), so it runs on the 5th-generation tensor cores.  A CTA owns 128 chunk
// rows: D (128 rows x 2r, fp32 in TMEM) += X tile (128 x 64, K-major, 128-byte
// swizzle) x A_kv tile (64 x 2r, read MN-major in 64-column boxes), issued by
// one thread as tcgen05 MMAs (M = 128, N = 2r, K = 16) over a 4-stage TMA
// pipeline.  The four warps then read their 32 TMEM lanes (rows) and the
// cluster reduces the hidden-split partial sums as above.
constexpr int TM2 = 128;
constexpr int NTHR2 = 128;
constexpr int NSTAGE2 = 4;

template <int R>
struct TCfgA {
  static constexpr int C = 2 * R;                 // 64 or 128 output columns
  static constexpr int X_TILE = TM2 * KC * 2;     // 16 KB
  static constexpr int A_TILE = KC * C * 2;       // 8 or 16 KB
  static constexpr int STAGE = X_TILE + A_TILE;
  static constexpr int CP = C + 4;                // fp32 partial row stride (16-byte rows, few bank conflicts)
  static constexpr int RED = TM2 * CP * 4;
  static constexpr int AREA = NSTAGE2 * STAGE > RED ? NSTAGE2 * STAGE : align1k(RED);
  static constexpr size_t smem = 1024 + AREA + 128;
};

template <int R>
__global__ void __launch_bounds__(NTHR2, 1)
    append_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmA,
                     __nv_bfloat16* __restrict__ lr, int64_t pos0, int64_t n, int64_t slr, int hs,
                     int kchunks, int* err) {
  using Cf = TCfgA<R>;
  constexpr int C = Cf::C;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t area_u = smem_u32(smem);
  const uint32_t bar_u = smem_u32(smem + Cf::AREA);
  auto full = [&](int st) { return bar_u + 8 * st; };
  auto empty = [&](int st) { return bar_u + 8 * (NSTAGE2 + st); };
  const uint32_t done = bar_u + 8 * (2 * NSTAGE2);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + Cf::AREA + 8 * (2 * NSTAGE2 + 1));
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  const int cr = blockIdx.x % hs;              // rank in the cluster = hidden split
  const int mtile = blockIdx.x / hs;
  const int seq = blockIdx.y;
  const int64_t t0 = (int64_t)mtile * TM2;
  const int kb = cr * kchunks / hs, ke = (cr + 1) * kchunks / hs;
  const int nk = ke - kb;
  cg::cluster_group cluster = cg::this_cluster();

  // the next kernel of the stream (the decode of the step) may start its
  // set-up now; it waits for this grid's completion before reading the LR cache
  pdl_launch_dependents();
  if (tid == 0) {
    for (int st = 0; st < NSTAGE2; ++st) {
      mbar_init(full(st), 1);
      mbar_init(empty(st), 1);
    }
    mbar_init(done, 1);
    fence_mbar_init();
    tma_prefetch(&tmX);
    tma_prefetch(&tmA);
  }
  if (w == 0) tmem_alloc(smem_u32(tslot), C);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  int fail = 0;

  if (tid == 0) {
    auto issue = [&](int j) {
      const int st = j % NSTAGE2;
      const uint32_t sb = area_u + st * Cf::STAGE;
      const int h0 = (kb + j) * KC;
      mbar_expect_tx(full(st), (uint32_t)Cf::STAGE);
      tma_load_3d(sb, &tmX, full(st), h0, (int)t0, seq);
#pragma unroll
      for (int b = 0; b < C / 64; ++b) tma_load_2d_(sb + Cf::X_TILE + b * KC * 128, &tmA, full(st), 64 * b, h0);
    };
    for (int j = 0; j < NSTAGE2 && j < nk; ++j) issue(j);
    constexpr uint32_t ID = umma_idesc_bf16(128, C, 0, 1);
    const uint64_t dX = umma_desc(area_u, 16, 1024, 2);
    const uint64_t dA = umma_desc(area_u + Cf::X_TILE, KC * 128, 1024, 2);
    for (int j = 0; j < nk; ++j) {
      const int st = j % NSTAGE2;
      if (!mbar_wait(full(st), (j / NSTAGE2) & 1)) fail = 1;
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < KC / 16; ++ks)
        umma_bf16(tmem, umma_desc_add(dX, st * Cf::STAGE + ks * 32),
                  umma_desc_add(dA, st * Cf::STAGE + ks * 16 * 128), ID, (j > 0 || ks > 0) ? 1u : 0u);
      umma_commit(empty(st));
      // refill the stage the previous tile's MMAs have finished reading
      if (j >= 1 && j - 1 + NSTAGE2 < nk) {
        const int sp = (j - 1) % NSTAGE2;
        if (!mbar_wait(empty(sp), ((j - 1) / NSTAGE2) & 1)) fail = 1;
        issue(j - 1 + NSTAGE2);
      }
    }
    umma_commit(done);
  }
  __syncwarp();
  if (!mbar_wait(done, 0)) fail = 1;   // every MMA (and so every load) is complete
  tc_fence_after();
  // partial sums: TMEM lane = row -> shared memory [TM2][C + 1] (stage area reused)
  float* red = reinterpret_cast<float*>(smem);
#pragma unroll
  for (int c0 = 0; c0 < C; c0 += 16) {
    uint32_t v[16];
    tmem_ld32x32b_x16(v, tmem + c0 + ((uint32_t)(32 * w) << 16));
    tmem_wait_ld_r16(v);
    float4* dst = reinterpret_cast<float4*>(red + (32 * w + lane) * Cf::CP + c0);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                           __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
  }
  tc_fence_before();
  if (__syncthreads_or(fail) && tid == 0) atomicOr(err, 2);
  if (hs > 1) cluster.sync();
  // this CTA's share of the rows, 4 columns a thread, summed over the cluster
  const int rows_per = (TM2 + hs - 1) / hs;
  const int r0 = cr * rows_per;
  for (int i = tid; i < rows_per * (C / 4); i += NTHR2) {
    const int row = r0 + i / (C / 4), c = 4 * (i % (C / 4));
    if (row >= TM2 || t0 + row >= n) continue;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int k = 0; k < hs; ++k) {
      const float4 x = *reinterpret_cast<const float4*>(cluster.map_shared_rank(red, k) + row * Cf::CP + c);
      v.x += x.x; v.y += x.y; v.z += x.z; v.w += x.w;
    }
    uint2 o;
    o.x = pack_bf16(v.x, v.y);
    o.y = pack_bf16(v.z, v.w);
    *reinterpret_cast<uint2*>(lr + seq * slr + (pos0 + t0 + row) * C + c) = o;
  }
  if (hs > 1) cluster.sync();
  __syncthreads();
  if (w == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, C);
  }
}

template <int R>
cudaError_t launch_r(const void* X, int64_t ldx, int64_t n, int64_t H, const void* A, void* lr,
                     int64_t pos0, int n_seqs, int64_t sx, int64_t slr, int* err, cudaStream_t st) {
  using Cf = ACfg<R>;
  constexpr int C = 2 * R;
  auto enc = encode_fn();
  if (!enc) return cudaErrorInvalidValue;
  CUtensorMap mx, ma;
  cuuint64_t xd[3] = {(cuuint64_t)H, (cuuint64_t)n, (cuuint64_t)n_seqs};
  cuuint64_t xs[2] = {(cuuint64_t)ldx * 2, (cuuint64_t)(n_seqs > 1 ? sx : n * ldx) * 2};
  cuuint32_t xb[3] = {KC, TM, 1};
  cuuint32_t one[3] = {1, 1, 1};
  if (enc(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(X), xd, xs, xb, one,
          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  constexpr int AB = C < 64 ? C : 64;
  cuuint64_t ad[2] = {(cuuint64_t)C, (cuuint64_t)H};
  cuuint64_t as[1] = {(cuuint64_t)C * 2};
  cuuint32_t ab[2] = {AB, KC};
  const CUtensorMapSwizzle sw = AB * 2 == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                : AB * 2 == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
  if (enc(&ma, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(A), ad, as, ab, one,
          CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  const int kchunks = (int)((H + KC - 1) / KC);
  if constexpr (R >= 32) {
    // tensor-core path: 128-row X boxes, otherwise the same maps
    CUtensorMap mx2;
    cuuint32_t xb2[3] = {KC, TM2, 1};
    if (enc(&mx2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(X), xd, xs, xb2, one,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    using Tf = TCfgA<R>;
    const int64_t mt2 = (n + TM2 - 1) / TM2;
    int hs2 = (int)(current_sms() / (mt2 * n_seqs));
    if (hs2 > kMaxHS) hs2 = kMaxHS;
    if (hs2 > kchunks) hs2 = kchunks;
    if (hs2 < 1) hs2 = 1;
    auto kern2 = append_tc_kernel<R>;
    cudaError_t e2 = cudaFuncSetAttribute(kern2, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Tf::smem);
    if (e2 != cudaSuccess) return e2;
    if (hs2 > 8) {
      e2 = cudaFuncSetAttribute(kern2, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
      if (e2 != cudaSuccess) return e2;
    }
    cudaLaunchConfig_t cfg2 = {};
    cfg2.gridDim = dim3((unsigned)(mt2 * hs2), n_seqs);
    cfg2.blockDim = dim3(NTHR2);
    cfg2.dynamicSmemBytes = Tf::smem;
    cfg2.stream = st;
    cudaLaunchAttribute attr2[1];
    attr2[0].id = cudaLaunchAttributeClusterDimension;
    attr2[0].val.clusterDim.x = hs2;
    attr2[0].val.clusterDim.y = 1;
    attr2[0].val.clusterDim.z = 1;
    cfg2.attrs = attr2;
    cfg2.numAttrs = 1;
    e2 = cudaLaunchKernelEx(&cfg2, kern2, mx2, ma, static_cast<__nv_bfloat16*>(lr), pos0, n, slr, hs2,
                            kchunks, err);
    if (e2 != cudaSuccess) return e2;
    return cudaGetLastError();
  }
  const int64_t mtiles = (n + TM - 1) / TM;
  int hs = (int)(current_sms() / (mtiles * n_seqs));
  if (hs > kMaxHS) hs = kMaxHS;
  if (hs > kchunks) hs = kchunks;
  if (hs < 1) hs = 1;
  auto kern = append_bf16_kernel<R>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Cf::smem);
  if (e != cudaSuccess) return e;
  if (hs > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(mtiles * hs), n_seqs);
  cfg.blockDim = dim3(NTHR);
  cfg.dynamicSmemBytes = Cf::smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = hs;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, mx, ma, static_cast<__nv_bfloat16*>(lr), pos0, n, slr, hs,
                         kchunks, err);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

bool bf16_append_supported(int64_t H, int r) {
  return H >= 16 && H < (1ll << 31) && (r == 8 || r == 16 || r == 32 || r == 64);
}

cudaError_t launch_append_bf16_mma(const void* X, int64_t ldx, int64_t n, int64_t H,
                                   const void* A, int r, void* lr, int64_t pos0, int n_seqs,
                                   int64_t sx, int64_t slr, cudaStream_t st) {
  int* err = error_word_ptr();
  if (!err) return cudaErrorInvalidValue;
  switch (r) {
    case 8: return launch_r<8>(X, ldx, n, H, A, lr, pos0, n_seqs, sx, slr, err, st);
    case 16: return launch_r<16>(X, ldx, n, H, A, lr, pos0, n_seqs, sx, slr, err, st);
    case 32: return launch_r<32>(X, ldx, n, H, A, lr, pos0, n_seqs, sx, slr, err, st);
    default: return launch_r<64>(X, ldx, n, H, A, lr, pos0, n_seqs, sx, slr, err, st);
  }
}

}  // namespace la
