// Internal declarations shared by the library's translation units.
// Nothing here is part of the public ABI (include/lora_attn.h).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "lora_attn.h"

namespace la {

constexpr int kMaxRowsSimt = 64;   // agents x GQA group rows one generic CTA holds

// Parameters of one attention launch, resolved on the host.
struct AttnParams {
  int n_seqs, n_agents, n_q, n_kv, d, r, g;
  int rows_per_tok;        // n_agents * g
  float s;                 // lora_scale
  float scale;             // softmax_scale
  double rope_base;
  int64_t L_max;
  const void* k_base;
  const void* v_base;
  int64_t kv_seq, kv_head, kv_tok;
  const void* lr;
  int64_t lr_seq;
  int64_t lr_agent;        // elements between agents' LR caches; 0 = one shared cache
  const void* B_k;
  const void* B_v;
  const void* q;
  void* out;
  const int32_t* kv_len;   // decode only
  int64_t max_kv_len;
  int64_t q_pos0;          // prefill only
  int n_q_tokens;
  int decode;              // 1 = decode, 0 = prefill
  // decode split-K
  int n_splits;
  int64_t split_len;       // keys per split (multiple of the key tile)
  float* partials;         // [units][n_splits][rows][d + r + 2]
  int* counters;           // [units]
  int* err;                // device error word
  int out_bf16;            // tensor-core kernels: 1 = bf16 outputs, 0 = fp32
  int agent_group;         // tensor-core decode: agents per CTA (grid z runs over the groups)
  int value_path;          // la_value_path: 0 fastest reordered, 1 generic reordered, 2 per tile
  int blk0;                // tensor-core prefill, split launch: the first block of rows it covers
  int early;               // decode step: the kernel before it writes only LR rows
  int64_t key_pos0;        // decode: position of key row 0 (sequence-sharded decode)
  float* row_stats;        // decode: (M, L) per output row, or null
};

// Device error word of the library (address on the current device).
int* error_word_ptr();

// Launchers (return cudaError_t of the launch).
cudaError_t launch_append_simt(const void* X, int64_t ldx, int64_t n, int64_t H, const void* A,
                               int r, void* lr, int64_t pos0, int n_seqs, int64_t sx,
                               int64_t slr, la_dtype dt, cudaStream_t st);
cudaError_t launch_append_bf16_mma(const void* X, int64_t ldx, int64_t n, int64_t H,
                                   const void* A, int r, void* lr, int64_t pos0, int n_seqs,
                                   int64_t sx, int64_t slr, cudaStream_t st);
cudaError_t launch_attn_simt(const AttnParams& p, la_dtype io, la_dtype out, cudaStream_t st);
// the bf16 decode of these parameters runs on the tensor-core kernel
bool bf16_decode_uses_tc(const AttnParams& p);
cudaError_t launch_append_row_at_len(const void* x, const void* A, int64_t a_stride, void* lr,
                                     int64_t lr_seq, int64_t lr_agent, int n_lr,
                                     const int32_t* kv_len, int64_t max_kv_len, int n_seqs,
                                     int64_t H, int r, la_dtype dt, int* err, cudaStream_t st);
cudaError_t launch_query_expand(const void* q_base, const void* lr_q, const void* B_q, void* q_out,
                                int n_seqs, int n_agents, int n_tok, int n_q, int d, int r, float s,
                                double rope_base, const int32_t* pos_end, la_dtype dt,
                                cudaStream_t st);
cudaError_t launch_output_delta(const void* o, const void* A_o, int64_t a_agent_stride,
                                const void* B_o, void* y, int n_seqs, int n_agents, int n_tok,
                                int d_in, int d_out, int r, float s, la_dtype dt, cudaStream_t st);
cudaError_t launch_materialize(const AttnParams& p, la_dtype io, void* kout, void* vout, cudaStream_t st);

// Decode split-K plan shared by the workspace query and the launch.
struct DecodePlan {
  int kind;                // 0 = generic SIMT kernel, 1 = bf16 tensor-core kernel
  int n_splits;
  int64_t split_len;
  int rows;                // rows per unit
  size_t partial_bytes;
  size_t counter_bytes;
  int groups;              // agent groups of the tensor-core decode (1 otherwise)
};

// ---------------------------------------------------------------------------
// small device helpers
// ---------------------------------------------------------------------------
template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

}  // namespace la
