// The C ABI: argument checks, launch planning and dispatch to the kernels.
// Every check runs before anything is enqueued; on error nothing is written.
#include <math.h>
#include <string.h>

#include "la_internal.cuh"

namespace la {

__device__ int g_error_word;

int* error_word_ptr() {
  static int* cached[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return nullptr;
  if (dev < 64 && cached[dev]) return cached[dev];
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_error_word) != cudaSuccess) return nullptr;
  if (dev < 64) cached[dev] = static_cast<int*>(ptr);
  return static_cast<int*>(ptr);
}

size_t simt_rows_cap(const AttnParams& p);
int simt_key_tile();
size_t simt_smem_bytes(const AttnParams& p);
bool bf16_decode_supported(const AttnParams& p);
size_t bf16_decode_partial_bytes(const AttnParams& p);
size_t bf16_decode_counter_ints(const AttnParams& p);
void bf16_decode_plan(const AttnParams& p, int* n_splits, int64_t* split_len, int* rows, int* groups);
cudaError_t launch_decode_bf16(const AttnParams& p, la_dtype out, cudaStream_t st);
bool bf16_prefill_supported(const AttnParams& p);
bool bf16_prefill_per_tile_supported(const AttnParams& p);
cudaError_t launch_prefill_bf16(const AttnParams& p, la_dtype out, cudaStream_t st);
bool bf16_append_supported(int64_t H, int r);

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t esize(la_dtype t) { return t == LA_F32 ? 4 : 2; }
bool dtype_ok(int t) { return t == LA_F32 || t == LA_BF16; }
bool rank_ok(int r) { return r == 8 || r == 16 || r == 32 || r == 64; }
bool stride_ok(int64_t s, la_dtype t) { return s > 0 && ((s * (int64_t)esize(t)) % 16) == 0; }

// Checks common to prefill and decode; fills p on success.
la_status check_attn(const la_attn_args* a, int decode, AttnParams* p) {
  if (!a) return LA_ERR_INVALID_ARG;
  if (!dtype_ok(a->io_dtype) || !dtype_ok(a->out_dtype)) return LA_ERR_INVALID_ARG;
  if (a->n_seqs < 0 || a->n_agents < 1 || a->n_q_heads < 1 || a->n_kv_heads < 1)
    return LA_ERR_INVALID_ARG;
  if (a->n_q_heads % a->n_kv_heads != 0) return LA_ERR_INVALID_ARG;
  if (a->head_dim != 64 && a->head_dim != 128) return LA_ERR_UNSUPPORTED;
  if (!rank_ok(a->r)) return LA_ERR_UNSUPPORTED;
  if (!isfinite(a->lora_scale) || !isfinite(a->softmax_scale) || !(a->softmax_scale > 0.f))
    return LA_ERR_INVALID_ARG;
  if (!isfinite(a->rope_base) || !(a->rope_base > 1.0)) return LA_ERR_INVALID_ARG;
  if (a->L_max < 1) return LA_ERR_INVALID_ARG;
  if (!a->k_base || !a->v_base || !a->lr_cache || !a->B_k || !a->B_v || !a->q || !a->out)
    return LA_ERR_INVALID_ARG;
  if (!aligned16(a->k_base) || !aligned16(a->v_base) || !aligned16(a->lr_cache) ||
      !aligned16(a->B_k) || !aligned16(a->B_v) || !aligned16(a->q) || !aligned16(a->out))
    return LA_ERR_INVALID_ARG;
  const la_dtype io = a->io_dtype;
  if (a->kv_tok_stride < a->head_dim || !stride_ok(a->kv_tok_stride, io) ||
      !stride_ok(a->kv_head_stride, io) || !stride_ok(a->kv_seq_stride, io))
    return LA_ERR_INVALID_ARG;
  if (a->lr_seq_stride < a->L_max * 2 * a->r || !stride_ok(a->lr_seq_stride, io))
    return LA_ERR_INVALID_ARG;
  if (a->lr_agent_stride != 0 &&
      (!stride_ok(a->lr_agent_stride, io) ||
       a->lr_agent_stride < (int64_t)(a->n_seqs > 0 ? a->n_seqs - 1 : 0) * a->lr_seq_stride + a->L_max * 2 * a->r))
    return LA_ERR_INVALID_ARG;
  if (a->value_path < LA_VALUE_REORDERED || a->value_path > LA_VALUE_PER_TILE_GENERIC) return LA_ERR_INVALID_ARG;
  if (a->key_pos0 < 0 || (reinterpret_cast<uintptr_t>(a->row_stats) & 7u) != 0) return LA_ERR_INVALID_ARG;
  if (!decode && (a->key_pos0 != 0 || a->row_stats)) return LA_ERR_UNSUPPORTED;   // decode only
  const int g = a->n_q_heads / a->n_kv_heads;
  if ((int64_t)a->n_agents * g > kMaxRowsSimt) return LA_ERR_UNSUPPORTED;
  if (decode) {
    if (a->n_q_tokens != 1) return LA_ERR_INVALID_ARG;
    if (!a->kv_len) return LA_ERR_INVALID_ARG;
    if (a->max_kv_len < 1) return LA_ERR_INVALID_ARG;
    if (a->max_kv_len > a->L_max) return LA_ERR_CAPACITY;
  } else {
    if (a->n_q_tokens < 0 || a->q_pos0 < 0) return LA_ERR_INVALID_ARG;
    if (a->q_pos0 + a->n_q_tokens > a->L_max) return LA_ERR_CAPACITY;
  }
  memset(p, 0, sizeof(*p));
  p->n_seqs = a->n_seqs;
  p->n_agents = a->n_agents;
  p->n_q = a->n_q_heads;
  p->n_kv = a->n_kv_heads;
  p->d = a->head_dim;
  p->r = a->r;
  p->g = g;
  p->rows_per_tok = a->n_agents * g;
  p->s = a->lora_scale;
  p->scale = a->softmax_scale;
  p->rope_base = a->rope_base;
  p->L_max = a->L_max;
  p->k_base = a->k_base;
  p->v_base = a->v_base;
  p->kv_seq = a->kv_seq_stride;
  p->kv_head = a->kv_head_stride;
  p->kv_tok = a->kv_tok_stride;
  p->lr = a->lr_cache;
  p->lr_seq = a->lr_seq_stride;
  p->lr_agent = a->lr_agent_stride;
  p->value_path = a->value_path;
  p->B_k = a->B_k;
  p->B_v = a->B_v;
  p->q = a->q;
  p->out = a->out;
  p->kv_len = a->kv_len;
  p->max_kv_len = a->max_kv_len;
  p->q_pos0 = a->q_pos0;
  p->n_q_tokens = decode ? 1 : a->n_q_tokens;
  p->decode = decode;
  p->key_pos0 = a->key_pos0;
  p->row_stats = a->row_stats;
  return LA_OK;
}

constexpr int kNumSMs = 148;

DecodePlan plan_decode(const AttnParams& p, la_dtype io) {
  DecodePlan d;
  memset(&d, 0, sizeof(d));
  const int units = p.n_seqs * p.n_kv;
  if (io == LA_BF16 && p.value_path == LA_VALUE_REORDERED && bf16_decode_supported(p)) {
    d.kind = 1;
    bf16_decode_plan(p, &d.n_splits, &d.split_len, &d.rows, &d.groups);
  } else {
    d.kind = 0;
    d.groups = 1;
    const int tk = simt_key_tile();
    const int64_t max_tiles = (p.max_kv_len + tk - 1) / tk;
    int64_t want = (2 * kNumSMs + units - 1) / (units > 0 ? units : 1);
    if (want > max_tiles) want = max_tiles;
    if (want < 1) want = 1;
    int64_t tiles_per = (max_tiles + want - 1) / want;
    d.split_len = tiles_per * tk;
    d.n_splits = (int)((p.max_kv_len + d.split_len - 1) / d.split_len);
    d.rows = (int)simt_rows_cap(p);
  }
  const size_t W = (size_t)p.d + p.r + 2;
  if (d.kind == 1)
    d.partial_bytes = bf16_decode_partial_bytes(p);
  else
    d.partial_bytes = d.n_splits > 1 ? (size_t)units * d.n_splits * d.rows * W * sizeof(float) : 0;
  d.partial_bytes = (d.partial_bytes + 255) / 256 * 256;
  // the split merge's counters: per unit an arrival and a departure counter
  // (generic kernel), or the bf16 decode's own
  const size_t ints = d.kind == 1 ? bf16_decode_counter_ints(p) : (size_t)2 * units * d.groups;
  d.counter_bytes = (ints * sizeof(int) + 255) / 256 * 256;
  return d;
}

}  // namespace
}  // namespace la

using namespace la;

extern "C" const char* la_status_string(la_status s) {
  switch (s) {
    case LA_OK: return "LA_OK";
    case LA_ERR_INVALID_ARG: return "LA_ERR_INVALID_ARG: invalid argument";
    case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED: configuration not supported";
    case LA_ERR_CAPACITY: return "LA_ERR_CAPACITY: rows beyond L_max";
    case LA_ERR_WORKSPACE: return "LA_ERR_WORKSPACE: workspace missing or too small";
    case LA_ERR_CUDA: return "LA_ERR_CUDA: CUDA call or launch failed";
    case LA_ERR_DEVICE_CHECK: return "LA_ERR_DEVICE_CHECK: a kernel bounds check fired";
    case LA_ERR_SCRATCH_LIMIT:
      return "LA_ERR_SCRATCH_LIMIT: decode scratch exceeds the library's static array";
  }
  return "unknown la_status";
}

namespace {
// The checks of lr_cache_append; *empty: valid, but nothing to read or write.
la_status append_check(const void* X, int64_t ldx, int64_t n_tokens, int64_t hidden,
                       const void* A_kv, int32_t r, const void* lr_cache, int64_t L_max,
                       int64_t pos0, int32_t n_seqs, int64_t seq_stride_x, int64_t seq_stride_lr,
                       la_dtype dt, bool* empty) {
  *empty = false;
  if (!dtype_ok(dt)) return LA_ERR_INVALID_ARG;
  if (n_tokens < 0 || n_seqs < 0 || hidden < 1 || L_max < 1) return LA_ERR_INVALID_ARG;
  if (!rank_ok(r)) return LA_ERR_UNSUPPORTED;
  if (pos0 < 0 || pos0 + n_tokens > L_max) return LA_ERR_CAPACITY;
  if (n_tokens == 0 || n_seqs == 0) {  // nothing is read or written
    *empty = true;
    return LA_OK;
  }
  if (!X || !A_kv || !lr_cache) return LA_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(A_kv) || !aligned16(lr_cache)) return LA_ERR_INVALID_ARG;
  if (ldx < hidden || !stride_ok(ldx, dt)) return LA_ERR_INVALID_ARG;
  if (n_seqs > 1 && (!stride_ok(seq_stride_x, dt) || !stride_ok(seq_stride_lr, dt)))
    return LA_ERR_INVALID_ARG;
  if (n_seqs > 1 && seq_stride_lr < L_max * 2 * r) return LA_ERR_INVALID_ARG;
  if ((hidden * (int64_t)esize(dt)) % 16 != 0) return LA_ERR_INVALID_ARG;
  if (n_seqs > 65535) return LA_ERR_UNSUPPORTED;
  return LA_OK;
}

// lr_cache_append's launch, after append_check passed with *empty false.
la_status append_launch(const void* X, int64_t ldx, int64_t n_tokens, int64_t hidden,
                        const void* A_kv, int32_t r, void* lr_cache, int64_t pos0,
                        int32_t n_seqs, int64_t seq_stride_x, int64_t seq_stride_lr, la_dtype dt,
                        cudaStream_t st) {
  cudaError_t e;
  if (dt == LA_BF16 && bf16_append_supported(hidden, r))
    e = launch_append_bf16_mma(X, ldx, n_tokens, hidden, A_kv, r, lr_cache, pos0, n_seqs,
                               seq_stride_x, seq_stride_lr, st);
  else
    e = launch_append_simt(X, ldx, n_tokens, hidden, A_kv, r, lr_cache, pos0, n_seqs,
                           seq_stride_x, seq_stride_lr, dt, st);
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}
}  // namespace

extern "C" la_status lr_cache_append(const void* X, int64_t ldx, int64_t n_tokens, int64_t hidden,
                                     const void* A_kv, int32_t r, void* lr_cache, int64_t L_max,
                                     int64_t pos0, int32_t n_seqs, int64_t seq_stride_x,
                                     int64_t seq_stride_lr, la_dtype dt, la_stream_t stream) {
  bool empty = false;
  const la_status s = append_check(X, ldx, n_tokens, hidden, A_kv, r, lr_cache, L_max, pos0,
                                   n_seqs, seq_stride_x, seq_stride_lr, dt, &empty);
  if (s != LA_OK || empty) return s;
  return append_launch(X, ldx, n_tokens, hidden, A_kv, r, lr_cache, pos0, n_seqs, seq_stride_x,
                       seq_stride_lr, dt, static_cast<cudaStream_t>(stream));
}

extern "C" la_status lr_cache_append_agents(const void* X, int64_t ldx, int64_t n_tokens,
                                            int64_t hidden, const void* A_kv, int32_t n_agents,
                                            int32_t r, void* lr_cache, int64_t lr_agent_stride,
                                            int64_t L_max, int64_t pos0, int32_t n_seqs,
                                            int64_t seq_stride_x, int64_t seq_stride_lr,
                                            la_dtype dt, la_stream_t stream) {
  if (!dtype_ok(dt) || n_agents < 1) return LA_ERR_INVALID_ARG;
  if (n_agents > 1) {
    if (!stride_ok(lr_agent_stride, dt)) return LA_ERR_INVALID_ARG;
    if (rank_ok(r) && n_seqs >= 1 && L_max >= 1 &&
        lr_agent_stride < (int64_t)(n_seqs - 1) * seq_stride_lr + L_max * 2 * r)
      return LA_ERR_INVALID_ARG;
  }
  // agent a: the single-A append of X A_a into its own cache; the checks of
  // the first call cover every agent (same shapes, strides and alignment)
  const size_t a_bytes = (size_t)hidden * 2 * r * esize(dt);
  for (int32_t a = 0; a < n_agents; ++a) {
    const la_status st = lr_cache_append(
        X, ldx, n_tokens, hidden, A_kv ? static_cast<const char*>(A_kv) + a * a_bytes : nullptr, r,
        lr_cache ? static_cast<char*>(lr_cache) + (size_t)a * lr_agent_stride * esize(dt) : nullptr,
        L_max, pos0, n_seqs, seq_stride_x, seq_stride_lr, dt, stream);
    if (st != LA_OK) return st;
  }
  return LA_OK;
}

extern "C" la_status lora_query_expand(const void* q_base, const void* lr_q, const void* B_q,
                                       void* q_out, int32_t n_seqs, int32_t n_agents,
                                       int32_t n_tok, int32_t n_q_heads, int32_t head_dim,
                                       int32_t r, float lora_scale, double rope_base,
                                       const int32_t* pos_end, la_dtype dt, la_stream_t stream) {
  if (!dtype_ok(dt)) return LA_ERR_INVALID_ARG;
  if (n_seqs < 1 || n_agents < 1 || n_tok < 1 || n_q_heads < 1) return LA_ERR_INVALID_ARG;
  if (!isfinite(lora_scale) || !isfinite(rope_base) || !(rope_base > 1.0)) return LA_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128) return LA_ERR_UNSUPPORTED;
  if (!rank_ok(r)) return LA_ERR_UNSUPPORTED;
  if (!q_base || !lr_q || !B_q || !q_out || !pos_end) return LA_ERR_INVALID_ARG;
  if (!aligned16(q_base) || !aligned16(lr_q) || !aligned16(B_q) || !aligned16(q_out) ||
      (reinterpret_cast<uintptr_t>(pos_end) & 3u) != 0)
    return LA_ERR_INVALID_ARG;
  if (n_agents > 65535 || n_seqs > 65535) return LA_ERR_UNSUPPORTED;
  if ((int64_t)n_tok * ((n_q_heads + 7) / 8) > 0x7fffffff) return LA_ERR_UNSUPPORTED;
  const cudaError_t e = la::launch_query_expand(q_base, lr_q, B_q, q_out, n_seqs, n_agents, n_tok,
                                                n_q_heads, head_dim, r, lora_scale, rope_base,
                                                pos_end, dt, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

extern "C" la_status lora_output_delta(const void* o, const void* A_o, int64_t a_agent_stride,
                                       const void* B_o, void* y, int32_t n_seqs, int32_t n_agents,
                                       int32_t n_tok, int32_t d_in, int32_t d_out, int32_t r,
                                       float lora_scale, la_dtype dt, la_stream_t stream) {
  if (!dtype_ok(dt)) return LA_ERR_INVALID_ARG;
  if (n_seqs < 1 || n_agents < 1 || n_tok < 1 || d_in < 1 || d_out < 1) return LA_ERR_INVALID_ARG;
  if (a_agent_stride < 0 || !isfinite(lora_scale)) return LA_ERR_INVALID_ARG;
  if ((a_agent_stride * (int64_t)esize(dt)) % 16 != 0) return LA_ERR_INVALID_ARG;
  if (!rank_ok(r) || d_out % 8 != 0) return LA_ERR_UNSUPPORTED;   // 8-column vectors of B_o and y
  if (!o || !A_o || !B_o || !y) return LA_ERR_INVALID_ARG;
  if (!aligned16(o) || !aligned16(A_o) || !aligned16(B_o) || !aligned16(y)) return LA_ERR_INVALID_ARG;
  if (n_agents > 65535 || n_seqs > 65535) return LA_ERR_UNSUPPORTED;
  const cudaError_t e = la::launch_output_delta(o, A_o, a_agent_stride, B_o, y, n_seqs, n_agents,
                                                n_tok, d_in, d_out, r, lora_scale, dt,
                                                static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

namespace la {
// Byte range of the arrival counters inside a decode workspace for these
// arguments (they must read zero when a decode starts).  False if invalid.
bool decode_counter_range(const la_attn_args* a, size_t* offset, size_t* bytes) {
  AttnParams p;
  if (check_attn(a, 1, &p) != LA_OK) return false;
  DecodePlan d = plan_decode(p, a->io_dtype);
  *offset = d.partial_bytes;
  *bytes = d.counter_bytes;
  return true;
}

// What lora_attn_decode's argument checks say about these arguments alone
// (no workspace considered): LA_OK for valid arguments.
la_status decode_args_status(const la_attn_args* a) {
  AttnParams p;
  return check_attn(a, 1, &p);
}
}  // namespace la

extern "C" size_t lora_attn_decode_workspace_bytes(const la_attn_args* a) {
  AttnParams p;
  if (check_attn(a, 1, &p) != LA_OK) return 0;
  DecodePlan d = plan_decode(p, a->io_dtype);
  return d.partial_bytes + d.counter_bytes;
}

namespace {
// The checks and the plan of lora_attn_decode.  On LA_OK with *empty false,
// *p is ready to launch as *kind (1: tensor-core decode, 0: generic kernel).
la_status decode_prepare(const la_attn_args* a, void* workspace, size_t workspace_bytes,
                         AttnParams* p, int* kind, bool* empty) {
  *empty = false;
  la_status s = check_attn(a, 1, p);
  if (s != LA_OK) return s;
  if (p->n_seqs == 0) {  // an empty batch needs no workspace (its size is 0)
    *empty = true;
    return LA_OK;
  }
  DecodePlan d = plan_decode(*p, a->io_dtype);
  // the sequence-sharded decode's inputs: the tensor-core decode only
  if ((p->key_pos0 != 0 || p->row_stats) && !(d.kind == 1 && bf16_decode_uses_tc(*p)))
    return LA_ERR_UNSUPPORTED;
  const size_t need = d.partial_bytes + d.counter_bytes;   // 0: no workspace, NULL allowed
  if (need > 0 && (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 ||
                   workspace_bytes < need))
    return LA_ERR_WORKSPACE;
  if ((int64_t)p->n_seqs * p->n_kv > 65535) return LA_ERR_UNSUPPORTED;
  if (d.kind == 0 && simt_smem_bytes(*p) > 227 * 1024) return LA_ERR_UNSUPPORTED;
  p->n_splits = d.n_splits;
  p->split_len = d.split_len;
  p->partials = static_cast<float*>(workspace);
  p->counters = reinterpret_cast<int*>(static_cast<char*>(workspace) + d.partial_bytes);
  *kind = d.kind;
  return LA_OK;
}

la_status decode_launch(AttnParams& p, int kind, const la_attn_args* a, cudaStream_t st) {
  p.err = error_word_ptr();
  if (!p.err) return LA_ERR_CUDA;
  cudaError_t e = kind == 1 ? launch_decode_bf16(p, a->out_dtype, st)
                            : launch_attn_simt(p, a->io_dtype, a->out_dtype, st);
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

// The checks of a decode step's new-row inputs.
la_status step_check(const la_attn_args* a, const void* A_kv, const void* x_new, int64_t hidden) {
  if (!A_kv || !x_new || hidden < 1) return LA_ERR_INVALID_ARG;
  if (!aligned16(A_kv) || !aligned16(x_new)) return LA_ERR_INVALID_ARG;
  if ((hidden * (int64_t)esize(a->io_dtype)) % 16 != 0) return LA_ERR_INVALID_ARG;
  return LA_OK;
}

// A decode step after decode_prepare: the new token's LR row at kv_len[q] - 1
// of every LR cache (one small kernel), then the decode, a programmatic
// dependent of it (its set-up overlaps the row's write).
la_status step_launch(AttnParams& p, int kind, const la_attn_args* a, const void* A_kv,
                      const void* x_new, int64_t hidden, cudaStream_t st) {
  p.err = error_word_ptr();
  if (!p.err) return LA_ERR_CUDA;
  const int n_lr = a->lr_agent_stride > 0 ? a->n_agents : 1;
  const cudaError_t e = launch_append_row_at_len(x_new, A_kv, hidden * 2 * a->r,
                                                 const_cast<void*>(a->lr_cache), a->lr_seq_stride,
                                                 a->lr_agent_stride, n_lr, a->kv_len, a->max_kv_len,
                                                 a->n_seqs, hidden, a->r, a->io_dtype, p.err, st);
  if (e != cudaSuccess) return LA_ERR_CUDA;
  p.early = 1;   // the append writes LR rows only: the decode may read its other inputs at once
  return decode_launch(p, kind, a, st);
}
}  // namespace

extern "C" la_status lora_attn_decode_step(const la_attn_args* a, const void* A_kv,
                                           const void* x_new, int64_t hidden, void* workspace,
                                           size_t workspace_bytes, la_stream_t stream) {
  AttnParams p;
  int kind = 0;
  bool empty = false;
  la_status s = decode_prepare(a, workspace, workspace_bytes, &p, &kind, &empty);
  if (s != LA_OK || empty) return s;
  s = step_check(a, A_kv, x_new, hidden);
  if (s != LA_OK) return s;
  return step_launch(p, kind, a, A_kv, x_new, hidden, static_cast<cudaStream_t>(stream));
}

extern "C" la_status lora_attn_decode(const la_attn_args* a, void* workspace,
                                      size_t workspace_bytes, la_stream_t stream) {
  AttnParams p;
  int kind = 0;
  bool empty = false;
  const la_status s = decode_prepare(a, workspace, workspace_bytes, &p, &kind, &empty);
  if (s != LA_OK || empty) return s;
  return decode_launch(p, kind, a, static_cast<cudaStream_t>(stream));
}

extern "C" la_status lora_decode_step_host(const la_attn_args* a, void* workspace,
                                           size_t workspace_bytes, const void* A_kv,
                                           int64_t hidden, void* x_dev, const void* x_host,
                                           const void* q_host, const int32_t* kv_len_host,
                                           void* out_host, la_stream_t stream) {
  AttnParams p;
  int kind = 0;
  bool empty = false;
  la_status s = decode_prepare(a, workspace, workspace_bytes, &p, &kind, &empty);
  if (s != LA_OK || empty) return s;
  if (!x_dev || !x_host || !q_host || !kv_len_host || !out_host || !a->lr_cache)
    return LA_ERR_INVALID_ARG;
  // the new token of sequence q sits at position kv_len_host[q] - 1
  for (int32_t q = 0; q < a->n_seqs; ++q)
    if (kv_len_host[q] < 1 || kv_len_host[q] > a->max_kv_len) return LA_ERR_INVALID_ARG;
  s = step_check(a, A_kv, x_dev, hidden);
  if (s != LA_OK) return s;
  const la_dtype dt = a->io_dtype;
  const int32_t n_seqs = a->n_seqs;
  const size_t es = esize(dt), eo = esize(a->out_dtype);
  const size_t x_bytes = (size_t)n_seqs * hidden * es;
  const size_t q_elems = (size_t)n_seqs * a->n_agents * a->n_q_heads * a->head_dim;
  const size_t q_bytes = q_elems * es, kv_bytes = (size_t)n_seqs * 4;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // x, q and kv_len back to back in one host and one device buffer: one copy
  // (each copy on the stream costs microseconds of latency, whatever its size)
  const char* xh = static_cast<const char*>(x_host);
  const char* xd = static_cast<const char*>(x_dev);
  const bool packed = xh + x_bytes == static_cast<const char*>(q_host) &&
                      xh + x_bytes + q_bytes == reinterpret_cast<const char*>(kv_len_host) &&
                      xd + x_bytes == static_cast<const char*>(a->q) &&
                      xd + x_bytes + q_bytes == reinterpret_cast<const char*>(a->kv_len);
  if (packed) {
    if (cudaMemcpyAsync(x_dev, x_host, x_bytes + q_bytes + kv_bytes, cudaMemcpyHostToDevice,
                        st) != cudaSuccess)
      return LA_ERR_CUDA;
  } else if (cudaMemcpyAsync(x_dev, x_host, x_bytes, cudaMemcpyHostToDevice, st) != cudaSuccess ||
             cudaMemcpyAsync(const_cast<void*>(a->q), q_host, q_bytes, cudaMemcpyHostToDevice,
                             st) != cudaSuccess ||
             cudaMemcpyAsync(const_cast<int32_t*>(a->kv_len), kv_len_host, kv_bytes,
                             cudaMemcpyHostToDevice, st) != cudaSuccess) {
    return LA_ERR_CUDA;
  }
  // out_host mapped into the device's address space (pinned memory under
  // unified addressing): the decode stores there directly, one stream copy
  // (microseconds of latency) fewer; other host memory gets the copy
  void* out_alias = nullptr;
  {
    cudaPointerAttributes pa;
    if (cudaPointerGetAttributes(&pa, out_host) == cudaSuccess) {
      if (pa.type == cudaMemoryTypeHost && pa.devicePointer && aligned16(pa.devicePointer))
        out_alias = pa.devicePointer;
    } else {
      cudaGetLastError();
    }
  }
  if (out_alias) p.out = out_alias;
  // the new rows (shared LR cache, or every agent's own) and the decode
  s = step_launch(p, kind, a, A_kv, x_dev, hidden, st);
  if (s != LA_OK) return s;
  if (!out_alias &&
      cudaMemcpyAsync(out_host, a->out, q_elems * eo, cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return LA_ERR_CUDA;
  return LA_OK;
}

extern "C" la_status lora_attn_prefill(const la_attn_args* a, la_stream_t stream) {
  AttnParams p;
  la_status s = check_attn(a, 0, &p);
  if (s != LA_OK) return s;
  if (p.n_seqs == 0 || p.n_q_tokens == 0) return LA_OK;
  if ((int64_t)p.n_seqs * p.n_kv > 65535) return LA_ERR_UNSUPPORTED;
  const bool tc = a->io_dtype == LA_BF16 &&
                  ((p.value_path == LA_VALUE_REORDERED && bf16_prefill_supported(p)) ||
                   (p.value_path == LA_VALUE_PER_TILE && bf16_prefill_per_tile_supported(p)));
  if (!tc && simt_smem_bytes(p) > 227 * 1024) return LA_ERR_UNSUPPORTED;
  p.err = error_word_ptr();
  if (!p.err) return LA_ERR_CUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e = tc ? launch_prefill_bf16(p, a->out_dtype, st)
                           : launch_attn_simt(p, a->io_dtype, a->out_dtype, st);
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

extern "C" la_status lora_materialize_agent_kv(const la_attn_args* a, void* k_out, void* v_out,
                                               la_stream_t stream) {
  AttnParams p;
  la_status s = check_attn(a, 1, &p);
  if (s != LA_OK) return s;
  if (a->key_pos0 != 0 || a->row_stats) return LA_ERR_UNSUPPORTED;   // the whole cache, unsharded
  if (!k_out || !v_out || !aligned16(k_out) || !aligned16(v_out)) return LA_ERR_INVALID_ARG;
  if (p.n_seqs == 0) return LA_OK;
  if (p.n_seqs > 65535 || (p.max_kv_len + 3) / 4 > 0x7fffffff) return LA_ERR_UNSUPPORTED;
  cudaError_t e = launch_materialize(p, a->io_dtype, k_out, v_out, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}

extern "C" la_status la_device_check_word(int32_t* word) {
  if (word) *word = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return LA_ERR_CUDA;
  int* ptr = error_word_ptr();
  if (!ptr) return LA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, ptr, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return LA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(ptr, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess)
      return LA_ERR_CUDA;
    if (word) *word = v;
    return LA_ERR_DEVICE_CHECK;
  }
  return LA_OK;
}

extern "C" la_status la_device_check(void) { return la_device_check_word(nullptr); }
