/*
 * lora_attn.h -- C ABI of the Flash-LoRA-Attention library (liblora_attn.so).
 *
 * Multi-LoRA agents that share one trajectory keep ONE base KV cache
 * (K_base = RoPE(X W_k), V_base = X W_v, computed with the pretrained
 * weights) and ONE low-rank (LR) cache LR = X [A_k | A_v] of width 2r,
 * because the LoRA down-projection A is shared by every agent (shared-A
 * multi-LoRA).  Agent a owns only its up-projections B_k^a and B_v^a.
 *   - Cache decomposition Y = X W_0 + (X A) B: LRAgent summary
 *     (paperlayer.ai/abs/2602.01053v2), App. A.3; LRAgent explainer
 *     (gist.science/pt/paper/2602.01053), Metodologia 1.
 *   - One shared LR cache (BaseLRShared): LRAgent summary §3; explainer,
 *     Metodologia 2.
 *   - LR rows computed once when a chunk is first processed (PreLRShared):
 *     PReCache abstract (ai.info, PReCache paper page) and PReCache blog
 *     (rit.work).
 *   - Flash-LoRA-Attention, which streams K/V blocks, keeps the value-side
 *     LoRA at rank r inside an online softmax and applies B once per query
 *     block: LRAgent summary App. B; explainer, Metodologia 3.
 *   - Key-side LoRA rebuilt in head dimension and rotated, since RoPE blocks
 *     the reordering on the key side: LRAgent summary App. D.1.
 *
 * What the attention entry points compute, per sequence, agent a, query head
 * h and its KV head j = floor(h / g), g = n_q_heads / n_kv_heads:
 *   K^a_t = K_base[j]_t + RoPE_t( s * LRk_t * B_k^a[:, j*d:(j+1)*d] )
 *   V^a_t = V_base[j]_t +         s * LRv_t * B_v^a[:, j*d:(j+1)*d]
 *   out   = softmax( q K^a^T * softmax_scale, causal ) V^a
 * with s = lora_scale = alpha / r, LRk_t = LR[t, 0:r], LRv_t = LR[t, r:2r].
 * RoPE pairs element i with i + d/2 and turns the pair by angle
 * t * rope_base^(-2i/d) at 0-based position t.  Queries arrive already
 * rotated.  Per-agent K^a / V^a are never written to memory.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, except
 *     the *_host buffers of lora_decode_step_host.  Nothing is retained
 *     after return.  The library never allocates device memory; decode
 *     scratch comes from the caller's workspace.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously; the library does not synchronise.
 *   - Argument errors are reported synchronously, BEFORE anything is
 *     launched, and nothing is written.  Launch failures return LA_ERR_CUDA.
 *   - Strides are in ELEMENTS.  Every base pointer must be 16-byte aligned
 *     and every stride a multiple of 16 bytes.
 *   - No C++ exception crosses this interface.
 */
#ifndef LORA_ATTN_H_
#define LORA_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* la_stream_t; /* a cudaStream_t */

typedef enum {
  LA_OK = 0,
  LA_ERR_INVALID_ARG = 1,  /* null pointer, bad shape, stride or alignment */
  LA_ERR_UNSUPPORTED = 2,  /* valid but not built: head_dim, rank, dtype mix */
  LA_ERR_CAPACITY = 3,     /* rows would land at or beyond L_max */
  LA_ERR_WORKSPACE = 4,    /* decode workspace missing or too small */
  LA_ERR_CUDA = 5,         /* a CUDA call or launch failed */
  LA_ERR_DEVICE_CHECK = 6, /* a kernel's own bounds check fired (see la_device_check) */
  LA_ERR_SCRATCH_LIMIT = 7 /* decode scratch would exceed LA_STATIC_SCRATCH_BYTES */
} la_status;

typedef enum { LA_F32 = 0, LA_BF16 = 1 } la_dtype;

/* How the value side is computed (la_attn_args.value_path).  All give the
 * same outputs up to rounding; 1 to 3 exist to measure the reordering (the
 * naive-reconstruction ablation of LRAgent summary App. B / explainer,
 * Metodologia 3):
 *   LA_VALUE_REORDERED          O = P V_base + (P LRv) s B_v^a, B_v applied once
 *                               per row; the fastest kernel for the shape.
 *   LA_VALUE_REORDERED_GENERIC  the same on the generic CUDA-core kernel.
 *   LA_VALUE_PER_TILE           naive: per key tile and agent, V^a = V_base +
 *                               s LRv B_v^a rebuilt in head dimension (rounded
 *                               to the io dtype), then O += P V^a.  The
 *                               tensor-core prefill has this arm at r = 16
 *                               (bf16, head_dim 128); the decode and other
 *                               shapes run it on the generic kernel.
 *   LA_VALUE_PER_TILE_GENERIC   the per-tile arm on the generic kernel. */
typedef enum {
  LA_VALUE_REORDERED = 0,
  LA_VALUE_REORDERED_GENERIC = 1,
  LA_VALUE_PER_TILE = 2,
  LA_VALUE_PER_TILE_GENERIC = 3
} la_value_path;

/* Human-readable name of a status code (static string, never NULL). */
const char* la_status_string(la_status s);

/*
 * lr_cache_append -- PreLRShared precompute of the shared LR cache.
 *
 * For every sequence q in [0, n_seqs) and chunk row i in [0, n_tokens):
 *   lr_cache[q][pos0 + i][c] = sum_k X[q][i][k] * A_kv[k][c],  c in [0, 2r)
 * i.e. the row [X A_k | X A_v]: unscaled (s is applied when rows are read)
 * and unrotated.  Accumulation is fp32; bf16 outputs are rounded to nearest
 * even.  Rows outside [pos0, pos0 + n_tokens) are not touched.
 *
 *   X        [n_seqs][n_tokens][hidden], row stride ldx, sequence stride
 *            seq_stride_x (elements).
 *   A_kv     [hidden][2r] row-major (A_k in columns 0..r-1, A_v in r..2r-1),
 *            shared by all sequences.
 *   lr_cache [n_seqs][L_max][2r], row stride 2r, sequence stride
 *            seq_stride_lr (elements).
 *   dt       dtype of X, A_kv and lr_cache (all the same).
 * Errors: LA_ERR_INVALID_ARG (null pointer, non-positive size, misaligned
 * pointer or stride), LA_ERR_UNSUPPORTED (r not in {8,16,32,64}),
 * LA_ERR_CAPACITY (pos0 < 0 or pos0 + n_tokens > L_max).
 */
la_status lr_cache_append(const void* X, int64_t ldx, int64_t n_tokens, int64_t hidden,
                          const void* A_kv, int32_t r, void* lr_cache, int64_t L_max,
                          int64_t pos0, int32_t n_seqs, int64_t seq_stride_x,
                          int64_t seq_stride_lr, la_dtype dt, la_stream_t stream);

/*
 * lr_cache_append_agents -- PreLRShared precompute of every agent's own LR
 * cache when each agent a has its own down-projection A_a (BaseShared): the
 * new chunk's hidden states are multiplied by every agent's A_a as they first
 * pass through the model (PReCache blog, how PReCache precomputes each role's
 * cache; LRAgent summary §3 "BaseShared": Y_lr,a = X A_a).
 *
 * For every agent a in [0, n_agents), sequence q and chunk row i:
 *   lr_cache[a][q][pos0 + i][c] = sum_k X[q][i][k] * A_kv[a][k][c]
 * with the layout, rounding and untouched rows of lr_cache_append.
 *
 *   A_kv      [n_agents][hidden][2r], each agent's [A_k,a | A_v,a] contiguous.
 *   lr_cache  agent a's cache starts at lr_cache + a * lr_agent_stride
 *             (elements; a multiple of 16 bytes, at least
 *             (n_seqs - 1) * seq_stride_lr + L_max * 2r).
 * Other arguments and errors as lr_cache_append; n_agents < 1 or a bad
 * lr_agent_stride is LA_ERR_INVALID_ARG.
 */
la_status lr_cache_append_agents(const void* X, int64_t ldx, int64_t n_tokens, int64_t hidden,
                                 const void* A_kv, int32_t n_agents, int32_t r, void* lr_cache,
                                 int64_t lr_agent_stride, int64_t L_max, int64_t pos0,
                                 int32_t n_seqs, int64_t seq_stride_x, int64_t seq_stride_lr,
                                 la_dtype dt, la_stream_t stream);

/* Arguments shared by lora_attn_prefill and lora_attn_decode. */
typedef struct {
  int32_t n_seqs;       /* independent sequences, each with its own caches */
  int32_t n_agents;     /* agents sharing each sequence's caches */
  int32_t n_q_heads;    /* query heads; a multiple of n_kv_heads */
  int32_t n_kv_heads;
  int32_t head_dim;     /* d: 64 or 128 */
  int32_t r;            /* LoRA rank: 8, 16, 32 or 64 */
  float lora_scale;     /* s = alpha / r */
  float softmax_scale;  /* usually 1 / sqrt(d) */
  double rope_base;     /* theta_i = rope_base^(-2i/d) */
  int64_t L_max;        /* rows allocated per (sequence, KV head) and per sequence in lr_cache */
  /* Base cache, already rotated: element (q, j, t, c) at
   * q*kv_seq_stride + j*kv_head_stride + t*kv_tok_stride + c; kv_tok_stride >= d. */
  const void* k_base;
  const void* v_base;
  int64_t kv_seq_stride, kv_head_stride, kv_tok_stride;
  /* LR cache [n_seqs][L_max][2r]: element (q, t, c) at q*lr_seq_stride + t*2r + c. */
  const void* lr_cache;
  int64_t lr_seq_stride;
  /* Per-agent up-projections [n_agents][r][n_kv_heads*d], contiguous. */
  const void* B_k;
  const void* B_v;
  /* Queries (already rotated) and outputs, contiguous
   * [n_seqs][n_agents][n_q_tokens][n_q_heads][d]. */
  const void* q;
  void* out;
  /* Decode: device int32 [n_seqs]; sequence q's query sits at position
   * kv_len[q]-1 and sees keys [0, kv_len[q]).  Ignored by prefill. */
  const int32_t* kv_len;
  int64_t max_kv_len;   /* decode: host upper bound on every kv_len[q], <= L_max */
  /* Prefill: query token j sits at position q_pos0 + j and sees keys
   * [0, q_pos0 + j]; the chunk's own base and LR rows must already be cached. */
  int64_t q_pos0;
  int32_t n_q_tokens;   /* decode: must be 1 */
  la_dtype io_dtype;    /* dtype of k_base, v_base, lr_cache, B_k, B_v and q */
  la_dtype out_dtype;   /* dtype of out */
  /* Elements between two agents' LR caches.  0: one LR cache shared by every
   * agent (shared A: BaseLRShared).  > 0: agent a owns its down-projection A_a
   * and reads its own LR cache X A_a (BaseShared; filled for every agent at
   * once by lr_cache_append_agents, PreLRShared), laid out as above and
   * starting at lr_cache + a * lr_agent_stride; a multiple of 16 bytes, at
   * least (n_seqs - 1) * lr_seq_stride + L_max * 2r (the caches do not
   * overlap).  LRAgent summary §3 "BaseShared"; LRAgent explainer, "Esquemas
   * de Compartilhamento"; PReCache blog, how PReCache precomputes each
   * role's cache.  The base cache stays shared in both cases. */
  int64_t lr_agent_stride;
  int32_t value_path;   /* la_value_path; 0 (zeroed struct) = LA_VALUE_REORDERED */
  /* Sequence-sharded decode: several devices each hold a slice of every
   * sequence's keys (both fields 0 / NULL in a zeroed struct: the unsharded
   * decode).  key_pos0: position of the caches' key row 0, so local key t is
   * RoPE'd as position key_pos0 + t.  row_stats: device float
   * [n_seqs][n_agents][n_q_heads][2] that the decode fills, per output row,
   * with M = max_t (q . K^a_t) * softmax_scale * log2(e) over its keys and
   * L = sum_t 2^(q . K^a_t * softmax_scale * log2(e) - M); with row_stats a
   * kv_len[q] of 0 is allowed (no keys: output 0, M = -inf, L = 0).  Either
   * needs the tensor-core decode (bf16, head_dim 128, r in {16, 32, 64});
   * elsewhere it returns LA_ERR_UNSUPPORTED.  lora_attn_decode_combine merges
   * the slices' outputs. */
  int64_t key_pos0;
  float* row_stats;
} la_attn_args;

/*
 * lora_attn_decode_step -- a decode step on device buffers: for every
 * sequence q the new token's LR row
 *   lr_cache[q][kv_len[q] - 1][c] = sum_k x_new[q][k] A_kv[k][c],  c in [0, 2r)
 * (with args->lr_agent_stride > 0 every agent's own cache, from its own
 * A_kv[a]; rounding as lr_cache_append), then lora_attn_decode over
 * [0, kv_len[q]), that row included: a small row-append kernel (positions
 * read from kv_len on the device), then the decode, whose set-up overlaps the
 * append's tail (programmatic dependent launch).
 * The new token's base K and V rows must already be in k_base / v_base.
 *
 *   A_kv    device, [hidden][2r] (shared A), or [n_agents][hidden][2r] with
 *           args->lr_agent_stride > 0; io dtype, 16-byte aligned.
 *   x_new   device, [n_seqs][hidden], io dtype, 16-byte aligned.
 *   hidden  > 0; hidden * element size a multiple of 16 bytes.
 * Other arguments, workspace and errors as lora_attn_decode, plus
 * LA_ERR_INVALID_ARG for a null or misaligned A_kv / x_new or a bad hidden.
 * (The pages have PreLRShared fill the LR rows when a chunk first passes
 * through the model, PReCache blog; for a decode token that chunk is the
 * token itself.)
 */
la_status lora_attn_decode_step(const la_attn_args* args, const void* A_kv, const void* x_new,
                                int64_t hidden, void* workspace, size_t workspace_bytes,
                                la_stream_t stream);

/*
 * lora_decode_step_host -- one whole decode step with the step's inputs and
 * outputs in HOST memory, as a serving loop runs it.  Queued on `stream`, in
 * this order, with nothing synchronised:
 *   1. copies x_host -> x_dev, q_host -> args->q, kv_len_host -> args->kv_len;
 *   2. lora_attn_decode_step(args, A_kv, x_dev, hidden, workspace, ...): the
 *      new token's LR row of every sequence q at position kv_len_host[q] - 1
 *      (with args->lr_agent_stride > 0, one row per agent into that agent's
 *      own cache, X A_a), then the decode;
 *   3. copies args->out -> out_host; or, when out_host is pinned host memory
 *      mapped into the device's address space (as memory from cudaHostAlloc
 *      is under unified addressing; cudaPointerGetAttributes reports a device
 *      alias), no copy: the decode writes its outputs straight into out_host
 *      and args->out is left as it was.
 * out_host holds the step's outputs once the stream has been synchronised.
 * Pinned (page-locked) host buffers make the copies asynchronous; pageable
 * ones are still correct, with the copies staged by the CUDA runtime.  When
 * x, q and kv_len lie back to back in that order, with no gap, both on the
 * host (x_host, q_host, kv_len_host) and on the device (x_dev, args->q,
 * args->kv_len), step 1 is a single copy instead of three: each copy on a
 * stream costs microseconds of latency, more than these few kilobytes take.
 *
 *   args        as lora_attn_decode; args->q, args->kv_len and args->lr_cache
 *               are device buffers this call writes (the copies and the
 *               append), args->out the device buffer it copies back (not
 *               used when out_host is mapped pinned memory, step 3).
 *   A_kv        device, [hidden][2r] (shared A) or [n_agents][hidden][2r]
 *               (args->lr_agent_stride > 0), io dtype.
 *   x_dev       device staging of n_seqs * hidden elements (io dtype), 16-byte
 *               aligned; hidden * element size a multiple of 16 bytes.
 *   x_host      host [n_seqs][hidden]: the new token's hidden row per sequence.
 *   q_host      host [n_seqs][n_agents][1][n_q_heads][d], io dtype.
 *   kv_len_host host int32 [n_seqs], each in [1, max_kv_len] (read by this
 *               call on the host and copied to args->kv_len).
 *   out_host    host [n_seqs][n_agents][1][n_q_heads][d], out dtype.
 * Errors, all before anything is queued: those of lora_attn_decode and
 * lr_cache_append, and LA_ERR_INVALID_ARG for a null host or staging pointer
 * or a kv_len_host[q] outside [1, max_kv_len].  LA_ERR_CUDA if a copy or a
 * launch fails to queue (the steps before it may have been queued).
 */
la_status lora_decode_step_host(const la_attn_args* args, void* workspace,
                                size_t workspace_bytes, const void* A_kv, int64_t hidden,
                                void* x_dev, const void* x_host, const void* q_host,
                                const int32_t* kv_len_host, void* out_host, la_stream_t stream);

/*
 * lora_attn_prefill -- causal Flash-LoRA-Attention for a chunk of n_q_tokens
 * query tokens per (sequence, agent) over prefix + chunk.
 * On the tensor-core path (bf16, head_dim 128, r in {16, 32, 64}) the score
 * product takes the queries and each agent's keys K^a = K_base + delta in
 * fp16 (the sum rounded once): queries and keys must stay below 65504 in
 * magnitude there.
 * Errors: LA_ERR_INVALID_ARG, LA_ERR_UNSUPPORTED, LA_ERR_CAPACITY
 * (q_pos0 + n_q_tokens > L_max), LA_ERR_CUDA.
 */
la_status lora_attn_prefill(const la_attn_args* args, la_stream_t stream);

/*
 * lora_attn_decode -- one query token per (sequence, agent), split over the
 * sequence (split-K).  On the tensor-core path (bf16, head_dim 128, r in
 * {16, 32, 64}, at most three agents) the rotated key delta and the scaled
 * queries s q are scored in fp16: they must stay below 65504 in magnitude
 * there.  On that path the partial results are merged inside
 * the same launch: that launch is cooperative (every CTA resident at once,
 * at most one per SM), so it fails with LA_ERR_CUDA on a device whose SMs
 * are partly taken by a context limit.  Other shapes merge in the same
 * launch (fp32) or in a second kernel (bf16).
 *
 * workspace: device memory of at least lora_attn_decode_workspace_bytes(args)
 * bytes, 256-byte aligned, ZERO-FILLED BEFORE ITS FIRST USE (may be NULL for
 * an empty batch, n_seqs = 0, which returns LA_OK and launches nothing).  Each call
 * leaves the arrival counters it used back at zero, so a workspace can be
 * reused by later calls on the same stream; calls that run concurrently
 * need separate workspaces.
 * Errors: as prefill, plus LA_ERR_WORKSPACE.  A kv_len[q] outside
 * [1, max_kv_len] is caught on the device: that sequence's outputs are left
 * unwritten and la_device_check() reports LA_ERR_DEVICE_CHECK.
 */
la_status lora_attn_decode(const la_attn_args* args, void* workspace, size_t workspace_bytes,
                           la_stream_t stream);

/* Workspace bytes lora_attn_decode needs for these arguments (0 if invalid). */
size_t lora_attn_decode_workspace_bytes(const la_attn_args* args);

/*
 * lora_attn_decode_combine -- merge the decodes of n_parts key slices of the
 * same queries (the sequence-sharded decode: each slice decoded with
 * row_stats, on its own device, and the slices' outputs and stats gathered,
 * e.g. by an all-gather over NCCL).  The combine step of the split-K decode,
 * across devices: with M* = max_p M_p and w_p = 2^(M_p - M*) L_p,
 *   out[row] = sum_p w_p outs[p][row] / sum_p w_p
 * (0 where every L_p is 0).  Each slice's output already holds its own
 * B_v^a term, which is linear, so the merge needs nothing else.  The pages
 * show no multi-device step: this is the decode's split-K combine (the
 * online-softmax merge of partial results) taken across devices.
 *   outs   device, [n_parts][rows][d] of out_dtype (fp32 or bf16)
 *   stats  device fp32, [n_parts][rows][2]: (M, L) as row_stats writes them
 *   out    device, [rows][d] of out_dtype; may not overlap outs
 * rows = n_seqs * n_agents * n_q_heads.  Asynchronous on `stream`.
 * Errors: LA_ERR_INVALID_ARG (null or unaligned pointers, n_parts < 1,
 * rows < 0, d not a positive multiple of 4, bad dtype), LA_ERR_CUDA.
 */
la_status lora_attn_decode_combine(const void* outs, const float* stats, int32_t n_parts,
                                   int64_t rows, int32_t d, la_dtype out_dtype, void* out,
                                   la_stream_t stream);

/*
 * lora_attn_decode_static_scratch -- lora_attn_decode for callers that cannot
 * give the library device memory.
 *
 * The pages have no counterpart to this entry point: it exists for callers
 * that cannot allocate device memory.  Examples are a plugin running inside a
 * serving runtime whose allocator owns every device allocation, and a process
 * that sizes its device memory once at start-up.
 *
 * It computes exactly what lora_attn_decode computes, with the same arguments
 * and errors, but it takes no workspace and allocates nothing.  The split-K
 * scratch (per-split partials and arrival counters) lives in one device array
 * of LA_STATIC_SCRATCH_BYTES that the library holds on every device that loads
 * it, until the process exits.
 *   - Each call looks up the array's device address on the current device
 *     (a host-side query) and allocates nothing.
 *   - An empty batch (n_seqs = 0) returns LA_OK and launches nothing; invalid
 *     arguments return the status lora_attn_decode would return.
 *   - Every call shares the one array, which keeps what the last call left
 *     in it; each call first clears, on `stream`, the part that must start at
 *     zero.  Calls whose work overlaps on the GPU (other streams, other host
 *     threads) race on the array: serialise them, e.g. on one stream.
 *   - If these arguments need more scratch than LA_STATIC_SCRATCH_BYTES
 *     (lora_attn_decode_workspace_bytes(args) > LA_STATIC_SCRATCH_BYTES), it
 *     returns LA_ERR_SCRATCH_LIMIT before launching anything.
 */
/*
 * lora_query_expand -- query-side LoRA and RoPE (the qkvo setting: LoRA on
 * the query, key, value and output projections; LRAgent summary App. D.1
 * "Ablation on LoRA Application"), producing the rotated per-agent queries
 * that lora_attn_prefill / lora_attn_decode take:
 *   q_out[q][a][j][h][:] = RoPE_pos( q_base[q][a][j][h][:]
 *                                    + s * lr_q[q][a][j][:] B_q[a][:, h*d:(h+1)*d] )
 * at position pos = pos_end[q] - n_tok + j (decode: pos_end = kv_len; prefill:
 * q_pos0 + n_tok), RoPE as for the keys.  The delta joins the projection
 * before the rotation.
 *
 *   q_base  [n_seqs][n_agents][n_tok][n_q_heads][d], X^a W_q of the base model,
 *           not yet rotated, contiguous.
 *   lr_q    [n_seqs][n_agents][n_tok][r], X^a A_q (unscaled), contiguous.
 *   B_q     [n_agents][r][n_q_heads * d], contiguous.
 *   q_out   layout of q_base; may be q_base itself (each element is read
 *           before it is written, by the same thread).
 *   pos_end device int32 [n_seqs].
 * All of dtype dt; fp32 accumulation.  Errors: LA_ERR_INVALID_ARG (null or
 * misaligned pointer, non-positive size), LA_ERR_UNSUPPORTED (head_dim not 64
 * or 128, r not in {8,16,32,64}, grid limits).
 */
la_status lora_query_expand(const void* q_base, const void* lr_q, const void* B_q, void* q_out,
                            int32_t n_seqs, int32_t n_agents, int32_t n_tok, int32_t n_q_heads,
                            int32_t head_dim, int32_t r, float lora_scale, double rope_base,
                            const int32_t* pos_end, la_dtype dt, la_stream_t stream);

/*
 * lora_output_delta -- output-side LoRA of the qkvo setting (LRAgent summary
 * App. D.1), added to the base model's output projection:
 *   y[q][a][j][:] += s * ( o[q][a][j][:] A_o[a] ) B_o[a]
 * so that y = O W_o + s (O A_o) B_o^a when y holds O W_o on entry.
 *
 *   o     [n_seqs][n_agents][n_tok][d_in], the attention outputs, contiguous.
 *   A_o   [d_in][r]; agent a's at A_o + a * a_agent_stride elements
 *         (a_agent_stride = 0: one A_o shared by every agent, shared-A).
 *   B_o   [n_agents][r][d_out], contiguous.
 *   y     [n_seqs][n_agents][n_tok][d_out], read and written.
 * All of dtype dt; fp32 accumulation.  Errors: LA_ERR_INVALID_ARG (null or
 * misaligned pointer, non-positive size, negative stride),
 * LA_ERR_UNSUPPORTED (r not in {8,16,32,64}, d_out not a multiple of 8,
 * grid limits).
 */
la_status lora_output_delta(const void* o, const void* A_o, int64_t a_agent_stride, const void* B_o,
                            void* y, int32_t n_seqs, int32_t n_agents, int32_t n_tok, int32_t d_in,
                            int32_t d_out, int32_t r, float lora_scale, la_dtype dt,
                            la_stream_t stream);

/*
 * lora_materialize_agent_kv -- the non-shared baseline's caches.
 *
 * Writes every agent's full keys and values
 *   K^a_t = K_base_t + RoPE_t(s LRk_t B_k^a),  V^a_t = V_base_t + s LRv_t B_v^a
 * for positions [0, max_kv_len) of every sequence and KV head: what a system
 * without cache sharing keeps per agent (LRAgent summary §3, Non-Shared).
 * Attention over them (lora_attn_decode with n_seqs * n_agents sequences of
 * one agent and B = 0) reads n_agents times the base cache; the library's
 * shared path never writes these.  It exists to measure that baseline.
 *
 * args: as for lora_attn_decode (q, out and the workspace are not used).
 * k_out, v_out: device, [n_seqs][n_agents][n_kv_heads][L_max][head_dim],
 *   contiguous, io_dtype; rows at or past max_kv_len are not written.
 * Errors: as lora_attn_decode's argument errors, and LA_ERR_INVALID_ARG for
 * a null or misaligned k_out / v_out.
 */
la_status lora_materialize_agent_kv(const la_attn_args* args, void* k_out, void* v_out,
                                    la_stream_t stream);

#define LA_STATIC_SCRATCH_BYTES ((size_t)4 << 20)
la_status lora_attn_decode_static_scratch(const la_attn_args* args, la_stream_t stream);

/*
 * la_device_check -- synchronises the current device, then reads and clears
 * the library's device error word.  Returns LA_OK, LA_ERR_DEVICE_CHECK if a
 * kernel's own check fired since the last call, or LA_ERR_CUDA.
 *
 * la_device_check_word -- the same, and writes the word's bits to *word
 * (host pointer; 0 when nothing fired):
 *   LA_DEV_KV_LEN     a decode kv_len[q] outside [1, max_kv_len]
 *   LA_DEV_PIPE_WAIT  a tensor-core kernel's wait on its copy/MMA pipeline
 *                     gave up after its iteration limit (the CTA skipped its
 *                     output and, holding TMEM, freed it)
 *   LA_DEV_MERGE_WAIT the split merge of a decode unit failed: a wait for
 *                     another split of the unit gave up after its iteration
 *                     limit (about a second), or the unit's arrival counter
 *                     held a value no call leaves there (a workspace not
 *                     zero-filled before its first use); that unit's output
 *                     is not to be trusted and may be left unwritten
 * No check traps: every kernel returns and the context stays usable.
 */
#define LA_DEV_KV_LEN 1
#define LA_DEV_PIPE_WAIT 2
#define LA_DEV_MERGE_WAIT 4
la_status la_device_check(void);
la_status la_device_check_word(int32_t* word);

#ifdef __cplusplus
}
#endif

#endif /* LORA_ATTN_H_ */
