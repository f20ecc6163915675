// Generic Flash-LoRA-Attention kernel on the CUDA cores (fp32 arithmetic).
//
// This is the exact-arithmetic path: it serves fp32 inputs (whose 1e-4
// parity bar tensor-core bf16 operands cannot meet), any shape the ABI
// accepts, and is the fallback shape-wise for bf16 inputs the tensor-core
// kernels do not cover.
//
// One CTA owns one (sequence, KV head) and a block of query tokens (prefill)
// or one split of the keys (decode).  Its rows are every agent x every query
// head of the GQA group (x the query tokens of the block), so the shared base
// and LR tiles are read once for all agents (LRAgent summary §3 BaseLRShared:
// one base cache and one LR cache for the whole system).
//
// Per key tile (LRAgent summary App. B, Flash-LoRA-Attention):
//   1. stage K_base, V_base and the LR rows of the tile in shared memory;
//   2. per agent, rebuild the key tile in head dimension,
//      K^a = K_base + RoPE_t(s LRk B_k^a) (App. D.1: the key side cannot be
//      reordered because RoPE depends on the position), and score it;
//   3. online softmax over the tile;
//   4. O_base += P V_base and O_lr += P LRv: the value side stays rank r
//      (explainer, Metodologia 3: O = P V_base + (P V_lr) B).
// Epilogue: out = (O_base + s O_lr B_v^a) / l, the single up-projection per
// query block.  Decode splits the keys over CTAs; the last CTA of a unit to
// arrive merges the (m, l, O_base, O_lr) partials and runs the epilogue.
// With one LR cache per agent (BaseShared) every agent's LR tile is staged.
// A second instance rebuilds V^a = V_base + s LRv B_v^a per tile instead of
// step 4's rank-r partial (the naive reconstruction, measured against the
// reordering).
#include "la_internal.cuh"

#include <math.h>

namespace la {
namespace {

constexpr int TK = 32;    // keys per tile (one per lane in the softmax step)
constexpr int NT = 256;   // threads per CTA
constexpr int NW = NT / 32;

struct SmemLayout {
  int rows, D, R;
  size_t theta, cs, q, kb, vb, ka, lr, s, o, m, l, alpha, pos, total;
  // n_lr: LR tiles staged per key tile (1 shared cache, or one per agent)
  __host__ __device__ SmemLayout(int rows_, int D_, int R_, int n_lr) : rows(rows_), D(D_), R(R_) {
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off += (bytes + 15) / 16 * 16; return o; };
    theta = take(sizeof(double) * 64);
    cs = take(sizeof(float2) * TK * (D / 2));
    q = take(sizeof(float) * rows * D);
    kb = take(sizeof(float) * TK * D);
    vb = take(sizeof(float) * TK * D);
    ka = take(sizeof(float) * TK * D);
    lr = take(sizeof(float) * TK * 2 * R * n_lr);
    s = take(sizeof(float) * rows * TK);
    o = take(sizeof(float) * rows * (D + R));
    m = take(sizeof(float) * rows);
    l = take(sizeof(float) * rows);
    alpha = take(sizeof(float) * rows);
    pos = take(sizeof(int64_t) * rows);
    total = off;
  }
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

// cos / sin of t * theta: the angle is formed and reduced modulo 2 pi in fp64,
// so large positions (up to 2^17 and beyond) keep full fp32 accuracy.
__device__ __forceinline__ float2 rope_cs(int64_t t, double theta) {
  const double two_pi = 6.283185307179586476925286766559;
  double ang = (double)t * theta;
  double k = rint(ang * (1.0 / two_pi));
  float red = (float)fma(-k, two_pi, ang);
  float sn, cs;
  sincosf(red, &sn, &cs);
  return make_float2(cs, sn);
}

// NAIVE: the value side rebuilt in head dimension per tile and agent,
// V^a = V_base + s LRv B_v^a, then O += P V^a (no rank-r partial; the
// naive-reconstruction baseline the reordering is measured against).
template <typename IO, typename OUT, bool NAIVE>
__global__ void __launch_bounds__(NT) attn_simt_kernel(const AttnParams p, const int qb) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int D = p.d, R = p.r, H2 = D / 2, g = p.g, na = p.n_agents;
  const int unit = blockIdx.z;
  const int seq = unit / p.n_kv, kvh = unit % p.n_kv;
  const int tok0 = blockIdx.y * qb;
  const int ntok = min(qb, p.n_q_tokens - tok0);
  const int rows = ntok * p.rows_per_tok;
  const int rows_cap = qb * p.rows_per_tok;
  const int split = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  const int n_lr = p.lr_agent ? na : 1;
  SmemLayout L(rows_cap, D, R, n_lr);
  double* theta = reinterpret_cast<double*>(smem + L.theta);
  float2* CS = reinterpret_cast<float2*>(smem + L.cs);
  float* Qs = reinterpret_cast<float*>(smem + L.q);
  float* Kb = reinterpret_cast<float*>(smem + L.kb);
  float* Vb = reinterpret_cast<float*>(smem + L.vb);
  float* Ka = reinterpret_cast<float*>(smem + L.ka);
  float* LRs = reinterpret_cast<float*>(smem + L.lr);
  float* S = reinterpret_cast<float*>(smem + L.s);
  float* O = reinterpret_cast<float*>(smem + L.o);
  float* M = reinterpret_cast<float*>(smem + L.m);
  float* Ls = reinterpret_cast<float*>(smem + L.l);
  float* Al = reinterpret_cast<float*>(smem + L.alpha);
  int64_t* Pos = reinterpret_cast<int64_t*>(smem + L.pos);

  // ---- key range of this CTA
  int64_t k_begin, k_end;
  if (p.decode) {
    const int64_t kvl = p.kv_len[seq];
    if (kvl < 1 || kvl > p.max_kv_len) {
      if (tid == 0 && split == 0) atomicOr(p.err, 1);
      return;  // every CTA of this unit returns: no partial, no arrival
    }
    k_begin = (int64_t)split * p.split_len;
    k_end = min(k_begin + p.split_len, kvl);
    if (k_end < k_begin) k_end = k_begin;
  } else {
    k_begin = 0;
    k_end = p.q_pos0 + tok0 + ntok;  // last query's position + 1
  }

  const IO* kbase = reinterpret_cast<const IO*>(p.k_base) + seq * p.kv_seq + kvh * p.kv_head;
  const IO* vbase = reinterpret_cast<const IO*>(p.v_base) + seq * p.kv_seq + kvh * p.kv_head;
  const IO* lrp = reinterpret_cast<const IO*>(p.lr) + seq * p.lr_seq;
  const int64_t ldB = (int64_t)p.n_kv * D;

  // ---- setup: theta, queries, accumulators
  for (int i = tid; i < H2; i += NT) theta[i] = exp2(-2.0 * i / D * log2(p.rope_base));
  for (int i = tid; i < rows * D; i += NT) {
    const int row = i / D, c = i % D;
    const int tl = row / p.rows_per_tok, a = (row / g) % na, gi = row % g;
    const int64_t qi =
        ((((int64_t)seq * na + a) * p.n_q_tokens + tok0 + tl) * p.n_q + kvh * g + gi) * D + c;
    Qs[i] = to_f32(reinterpret_cast<const IO*>(p.q)[qi]);
  }
  for (int i = tid; i < rows * (D + R); i += NT) O[i] = 0.f;
  for (int row = tid; row < rows; row += NT) {
    M[row] = -INFINITY;
    Ls[row] = 0.f;
    const int tl = row / p.rows_per_tok;
    Pos[row] = p.decode ? (k_end > 0 ? (int64_t)p.kv_len[seq] - 1 : 0) : p.q_pos0 + tok0 + tl;
  }
  __syncthreads();

  for (int64_t k0 = k_begin; k0 < k_end; k0 += TK) {
    // 1. stage the tile
    for (int i = tid; i < TK * D; i += NT) {
      const int t = i / D, c = i % D;
      const int64_t key = k0 + t;
      float kv = 0.f, vv = 0.f;
      if (key < k_end) {
        kv = to_f32(kbase[key * p.kv_tok + c]);
        vv = to_f32(vbase[key * p.kv_tok + c]);
      }
      Kb[i] = kv;
      Vb[i] = vv;
    }
    // LR tile [n_lr][TK][2r]: the shared cache, or agent a's own (BaseShared)
    for (int i = tid; i < n_lr * TK * 2 * R; i += NT) {
      const int al = i / (TK * 2 * R), t = (i / (2 * R)) % TK, c = i % (2 * R);
      const int64_t key = k0 + t;
      LRs[i] = key < k_end ? to_f32(lrp[al * p.lr_agent + key * 2 * R + c]) : 0.f;
    }
    for (int i = tid; i < TK * H2; i += NT) {
      const int t = i / H2, c = i % H2;
      CS[i] = rope_cs(k0 + t, theta[c]);
    }
    __syncthreads();

    for (int a = 0; a < na; ++a) {
      // 2a. key expansion for agent a: K^a = K_base + RoPE(s * LRk * B_k^a)
      const IO* Bk = reinterpret_cast<const IO*>(p.B_k) + (int64_t)a * R * ldB + kvh * D;
      const float* LRa = LRs + (n_lr > 1 ? a : 0) * TK * 2 * R;
      for (int i = tid; i < TK * H2; i += NT) {
        const int t = i / H2, c = i % H2;
        float x1 = 0.f, x2 = 0.f;
        for (int j = 0; j < R; ++j) {
          const float lv = LRa[t * 2 * R + j];
          x1 = fmaf(lv, to_f32(Bk[j * ldB + c]), x1);
          x2 = fmaf(lv, to_f32(Bk[j * ldB + c + H2]), x2);
        }
        x1 *= p.s;
        x2 *= p.s;
        const float2 cs = CS[i];
        Ka[t * D + c] = Kb[t * D + c] + (x1 * cs.x - x2 * cs.y);
        Ka[t * D + c + H2] = Kb[t * D + c + H2] + (x2 * cs.x + x1 * cs.y);
      }
      __syncthreads();
      // 2b. scores of agent a's rows
      const int rows_a = ntok * g;
      for (int i = tid; i < rows_a * TK; i += NT) {
        const int ra = i / TK, t = i % TK;
        const int row = ((ra / g) * na + a) * g + (ra % g);
        const int64_t key = k0 + t;
        float acc = 0.f;
        for (int c = 0; c < D; ++c) acc = fmaf(Qs[row * D + c], Ka[t * D + c], acc);
        const bool vis = key < k_end && key <= Pos[row];
        S[row * TK + t] = vis ? acc * p.scale : -INFINITY;
      }
      __syncthreads();
    }

    // 3. online softmax, one warp per row
    for (int row = warp; row < rows; row += NW) {
      const float v = S[row * TK + lane];
      const float mt = warp_max(v);
      const float mold = M[row];
      const float mnew = fmaxf(mold, mt);
      float pv = 0.f, corr = 0.f;
      if (mnew != -INFINITY) {
        pv = expf(v - mnew);
        corr = (mold == -INFINITY) ? 0.f : expf(mold - mnew);
      }
      const float ps = warp_sum(pv);
      S[row * TK + lane] = pv;
      if (lane == 0) {
        M[row] = mnew;
        Ls[row] = Ls[row] * corr + ps;
        Al[row] = corr;
      }
    }
    __syncthreads();

    const int W = D + R;
    if constexpr (NAIVE) {
      // 4'. per agent: V^a tile in head dimension (over the key buffer), then
      // O_base += P V^a for the agent's rows; O_lr stays zero
      for (int a = 0; a < na; ++a) {
        const IO* Bv = reinterpret_cast<const IO*>(p.B_v) + (int64_t)a * R * ldB + kvh * D;
        const float* LRa = LRs + (n_lr > 1 ? a : 0) * TK * 2 * R;
        for (int i = tid; i < TK * D; i += NT) {
          const int t = i / D, c = i % D;
          float x = 0.f;
          for (int j = 0; j < R; ++j) x = fmaf(LRa[t * 2 * R + R + j], to_f32(Bv[j * ldB + c]), x);
          Ka[i] = fmaf(p.s, x, Vb[i]);
        }
        __syncthreads();
        const int rows_a = ntok * g;
        for (int i = tid; i < rows_a * D; i += NT) {
          const int ra = i / D, c = i % D;
          const int row = ((ra / g) * na + a) * g + (ra % g);
          float acc = O[row * W + c] * Al[row];
          const float* Pr = S + row * TK;
          for (int t = 0; t < TK; ++t) acc = fmaf(Pr[t], Ka[t * D + c], acc);
          O[row * W + c] = acc;
        }
        __syncthreads();
      }
      continue;
    }
    // 4. O_base += P V_base ; O_lr += P LRv
    for (int i = tid; i < rows * W; i += NT) {
      const int row = i / W, c = i % W;
      float acc = O[i] * Al[row];
      const float* Pr = S + row * TK;
      if (c < D) {
        for (int t = 0; t < TK; ++t) acc = fmaf(Pr[t], Vb[t * D + c], acc);
      } else {
        const int j = R + (c - D);
        const float* LRa = LRs + (n_lr > 1 ? (row / g) % na : 0) * TK * 2 * R;   // the row's agent
        for (int t = 0; t < TK; ++t) acc = fmaf(Pr[t], LRa[t * 2 * R + j], acc);
      }
      O[i] = acc;
    }
    __syncthreads();
  }

  const int W = D + R;
  if (p.decode && p.n_splits > 1) {
    // write this split's partial (m, l, O_base, O_lr) and arrive
    const int WP = W + 2;
    float* part = p.partials + ((size_t)unit * p.n_splits + split) * (size_t)rows_cap * WP;
    for (int i = tid; i < rows * W; i += NT) part[(i / W) * WP + (i % W)] = O[i];
    for (int row = tid; row < rows; row += NT) {
      part[row * WP + W] = M[row];
      part[row * WP + W + 1] = Ls[row];
    }
    __threadfence();
    __syncthreads();
    __shared__ int s_last;
    if (tid == 0) s_last = (atomicAdd(&p.counters[unit], 1) == p.n_splits - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    // merge every split's partial into shared memory
    const float* base = p.partials + (size_t)unit * p.n_splits * (size_t)rows_cap * WP;
    const size_t sstride = (size_t)rows_cap * WP;
    for (int row = warp; row < rows; row += NW) {
      float mx = -INFINITY;
      for (int k = lane; k < p.n_splits; k += 32) mx = fmaxf(mx, __ldcg(base + k * sstride + row * WP + W));
      mx = warp_max(mx);
      float lt = 0.f;
      for (int k = lane; k < p.n_splits; k += 32) {
        const float mk = __ldcg(base + k * sstride + row * WP + W);
        if (mk != -INFINITY) lt += expf(mk - mx) * __ldcg(base + k * sstride + row * WP + W + 1);
      }
      lt = warp_sum(lt);
      if (lane == 0) {
        M[row] = mx;
        Ls[row] = lt;
      }
    }
    __syncthreads();
    for (int i = tid; i < rows * W; i += NT) {
      const int row = i / W, c = i % W;
      float acc = 0.f;
      for (int k = 0; k < p.n_splits; ++k) {
        const float mk = __ldcg(base + k * sstride + row * WP + W);
        if (mk != -INFINITY) acc += expf(mk - M[row]) * __ldcg(base + k * sstride + row * WP + c);
      }
      O[i] = acc;
    }
    if (tid == 0) p.counters[unit] = 0;  // leave the workspace reusable
    __syncthreads();
  }

  // epilogue: out = (O_base + s * O_lr B_v^a) / l
  for (int i = tid; i < rows * D; i += NT) {
    const int row = i / D, c = i % D;
    const int tl = row / p.rows_per_tok, a = (row / g) % na, gi = row % g;
    const IO* Bv = reinterpret_cast<const IO*>(p.B_v) + (int64_t)a * R * ldB + kvh * D + c;
    float lora = 0.f;
    for (int j = 0; j < R; ++j) lora = fmaf(O[row * W + D + j], to_f32(Bv[j * ldB]), lora);
    const float l = Ls[row];
    const float val = l > 0.f ? (O[row * W + c] + p.s * lora) / l : 0.f;
    const int64_t oi =
        ((((int64_t)seq * na + a) * p.n_q_tokens + tok0 + tl) * p.n_q + kvh * g + gi) * D + c;
    reinterpret_cast<OUT*>(p.out)[oi] = from_f32<OUT>(val);
  }
}

template <typename IO, typename OUT, bool NAIVE>
cudaError_t launch_typed(const AttnParams& p, cudaStream_t st) {
  const int qb = p.decode ? 1 : max(1, kMaxRowsSimt / p.rows_per_tok);
  const int rows_cap = qb * p.rows_per_tok;
  SmemLayout L(rows_cap, p.d, p.r, p.lr_agent ? p.n_agents : 1);
  if (L.total > 227 * 1024) return cudaErrorInvalidConfiguration;
  cudaError_t e = cudaFuncSetAttribute(attn_simt_kernel<IO, OUT, NAIVE>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  const int units = p.n_seqs * p.n_kv;
  dim3 grid(p.decode ? p.n_splits : 1, p.decode ? 1 : (p.n_q_tokens + qb - 1) / qb, units);
  attn_simt_kernel<IO, OUT, NAIVE><<<grid, NT, L.total, st>>>(p, qb);
  return cudaGetLastError();
}

}  // namespace

size_t simt_rows_cap(const AttnParams& p) {
  const int qb = p.decode ? 1 : max(1, kMaxRowsSimt / p.rows_per_tok);
  return (size_t)qb * p.rows_per_tok;
}

int simt_key_tile() { return TK; }

size_t simt_smem_bytes(const AttnParams& p) {
  return SmemLayout((int)simt_rows_cap(p), p.d, p.r, p.lr_agent ? p.n_agents : 1).total;
}

template <bool NAIVE>
cudaError_t launch_io(const AttnParams& p, la_dtype io, la_dtype out, cudaStream_t st) {
  if (io == LA_F32 && out == LA_F32) return launch_typed<float, float, NAIVE>(p, st);
  if (io == LA_F32 && out == LA_BF16) return launch_typed<float, __nv_bfloat16, NAIVE>(p, st);
  if (io == LA_BF16 && out == LA_F32) return launch_typed<__nv_bfloat16, float, NAIVE>(p, st);
  return launch_typed<__nv_bfloat16, __nv_bfloat16, NAIVE>(p, st);
}

cudaError_t launch_attn_simt(const AttnParams& p, la_dtype io, la_dtype out, cudaStream_t st) {
  const bool per_tile = p.value_path == LA_VALUE_PER_TILE || p.value_path == LA_VALUE_PER_TILE_GENERIC;
  return per_tile ? launch_io<true>(p, io, out, st)
                                           : launch_io<false>(p, io, out, st);
}

}  // namespace la
