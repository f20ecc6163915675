"""fp64 CPU oracle for Flash-LoRA-Attention and the low-rank cache append.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  The library's
product path never calls it, and it shares no code with the CUDA kernels.

What it computes, and from which passage:

* Cache decomposition Y = Y_base + dY with Y_base = X W_0 and
  dY = X dW = (X A) B -- LRAgent summary (paperlayer.ai/abs/2602.01053v2),
  App. A.3 "Cosine Similarity Bound" definitions; LRAgent explainer
  (gist.science/pt/paper/2602.01053), Resumo Tecnico, Metodologia 1
  "Decomposicao de Cache".
* One low-rank (LR) cache X A shared by every agent because A is shared
  (BaseLRShared) -- LRAgent summary §3 "BaseLRShared"; explainer,
  Metodologia 2 "BaseLRShared".  Filled once per new context chunk
  (PreLRShared precompute) -- PReCache abstract (ai.info/it, PReCache
  paper page), PReCache blog (rit.work).
* Keys carry LoRA too (the qkvo ablation): the key delta is rebuilt in head
  dimension and rotated by RoPE, because the position-dependent rotation
  blocks the associativity trick -- LRAgent summary App. D.1 "Ablation on
  LoRA Application".  So K^a_t = K_base,t + RoPE_t(s LRk_t B_k^a),
  V^a_t = V_base,t + s LRv_t B_v^a, with s = alpha / r.
* Attention of one head over accumulated length L = L_p + L_c with a causal
  mask -- LRAgent summary App. B "Flash-LoRA-Attention".
* Optionally one LR cache per agent, X A_a, when every agent owns its own
  down-projection A_a (BaseShared: only the base cache is shared) -- LRAgent
  summary §3 "BaseShared"; LRAgent explainer, "Esquemas de Compartilhamento",
  BaseShared.  PreLRShared fills every agent's cache when a chunk first passes
  through the model -- PReCache blog (rit.work), how PReCache precomputes each
  role's cache.
* A decode split over devices by key slices (no passage on the pages: the
  decode's split-K merge of partial softmax results, taken across devices):
  ``decode_slice`` and ``combine_slices``, pinned by the merge reproducing
  the whole decode.

The oracle MATERIALISES every agent's full K^a and V^a and runs a naive
two-pass softmax (max, then exp / sum).  It does not use the reordered value
path (P V_lr) B that the kernels use; the tests check that identity
separately.

Readings where the pages are silent (each is also listed in the design notes):
* RoPE: half-split pairing (i, i + d/2), theta_i = base^(-2i/d), angle
  t * theta_i, positions 0-based; no frequency rescaling.
* Queries arrive already rotated at their own position.
* s multiplies the LR product on both the key and the value side; the LR
  cache stores the unscaled X A, K part first: row = [X A_k | X A_v].
* GQA: query head h reads KV head floor(h / g), g = n_q / n_kv.  Columns
  [j d, (j + 1) d) of B_k^a / B_v^a belong to KV head j.
* Decode: the one query sits at position kv_len - 1 and sees keys [0, kv_len).
  Prefill: query j sits at position q_pos0 + j and sees keys [0, q_pos0 + j].
"""
from __future__ import annotations

import numpy as np

f64 = np.float64


def _np64(x) -> np.ndarray:
    """Any tensor-like (torch CPU tensor of any float dtype, numpy array) -> fp64 ndarray."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch  # local: only to upcast bf16, which numpy lacks
        x = x.to(torch.float64).numpy()
    return np.asarray(x, dtype=f64)


# ----------------------------------------------------------------------------
# RoPE (LRAgent summary App. D.1 names the rotation; convention: see header)
# ----------------------------------------------------------------------------
def rope_inv_freq(head_dim: int, rope_base: float) -> np.ndarray:
    """theta_i = base^(-2 i / d) for i in [0, d/2), fp64."""
    i = np.arange(head_dim // 2, dtype=f64)
    return np.power(f64(rope_base), -2.0 * i / head_dim)


def rope(x, positions, rope_base: float) -> np.ndarray:
    """Rotate rows of x [..., T, d] by their positions [T] (half-split pairs)."""
    x = _np64(x)
    d = x.shape[-1]
    h = d // 2
    ang = np.asarray(positions, dtype=f64)[:, None] * rope_inv_freq(d, rope_base)[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., :h], x[..., h:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


# ----------------------------------------------------------------------------
# LR cache append (PreLRShared precompute)
# ----------------------------------------------------------------------------
def lr_cache_rows(X, A_kv) -> np.ndarray:
    """LR rows for a chunk: X [.., n, H] @ A_kv [H, 2r] -> [.., n, 2r] = [X A_k | X A_v].

    Unscaled (s is applied when the rows are used) and unrotated.
    """
    return _np64(X) @ _np64(A_kv)


def lr_cache_append(lr_cache, X, A_kv, pos0: int) -> np.ndarray:
    """Return a copy of lr_cache [n_seqs, L_max, 2r] with rows pos0..pos0+n-1 replaced
    by X [n_seqs, n, H] @ A_kv.  Every other row is left as it was."""
    out = _np64(lr_cache).copy()
    rows = lr_cache_rows(X, A_kv)
    n = rows.shape[-2]
    out[:, pos0:pos0 + n, :] = rows
    return out


def lr_cache_append_agents(lr_caches, X, A_kv_agents, pos0: int) -> np.ndarray:
    """Every agent's own LR cache (BaseShared, filled by PreLRShared): a copy of
    lr_caches [n_agents, n_seqs, L_max, 2r] whose agent a has rows
    pos0..pos0+n-1 replaced by X @ A_kv_agents[a] ([H, 2r])."""
    return np.stack([lr_cache_append(lr_caches[a], X, A_kv_agents[a], pos0)
                     for a in range(len(A_kv_agents))])


# ----------------------------------------------------------------------------
# Base cache from hidden states (used only where the inputs are hidden states)
# ----------------------------------------------------------------------------
def base_cache_from_hidden(X, W_k, W_v, n_kv_heads: int, rope_base: float):
    """K_base = RoPE_t(X_t W_k) per KV head, V_base = X W_v.

    X [n_seqs, L, H]; W_k, W_v [H, n_kv*d].  Returns k_base, v_base with layout
    [n_seqs, n_kv, L, d] in fp64.
    """
    X = _np64(X)
    n_seqs, L, _ = X.shape
    kp = X @ _np64(W_k)
    vp = X @ _np64(W_v)
    d = kp.shape[-1] // n_kv_heads
    kp = kp.reshape(n_seqs, L, n_kv_heads, d).transpose(0, 2, 1, 3)
    vp = vp.reshape(n_seqs, L, n_kv_heads, d).transpose(0, 2, 1, 3)
    k_base = rope(kp, np.arange(L), rope_base)
    return k_base, vp


# ----------------------------------------------------------------------------
# LoRA on the query and output projections (the qkvo setting of LRAgent
# summary App. D.1 "Ablation on LoRA Application"; Y = X W_0 + (X A) B as in
# App. A.3)
# ----------------------------------------------------------------------------
def lora_queries(q_base, lr_q, B_q, lora_scale: float, positions, rope_base: float) -> np.ndarray:
    """Agent queries with a query-side LoRA, rotated at their positions:
    q^a_t = RoPE_t(X_t W_q + s (X_t A_q) B_q^a), head by head.

    q_base [n_tok, n_q, d]: the base projection X W_q, not yet rotated;
    lr_q [n_tok, r]: X A_q, unscaled; B_q [r, n_q*d]: the agent's up-projection.
    The delta joins the projection before RoPE (RoPE rotates what the
    projection produces).  Returns [n_tok, n_q, d]."""
    qb = _np64(q_base)
    n_tok, n_q, d = qb.shape
    delta = lora_scale * (_np64(lr_q) @ _np64(B_q))            # [n_tok, n_q*d]
    pre = qb + delta.reshape(n_tok, n_q, d)
    return rope(pre.transpose(1, 0, 2), positions, rope_base).transpose(1, 0, 2)


def lora_output(y_base, o, A_o, B_o, lora_scale: float) -> np.ndarray:
    """Output projection with LoRA: y^a = O W_o + s (O A_o) B_o^a, given the
    base part y_base = O W_o.  o [n_tok, D_in]; A_o [D_in, r]; B_o [r, D_out]."""
    return _np64(y_base) + lora_scale * ((_np64(o) @ _np64(A_o)) @ _np64(B_o))


# ----------------------------------------------------------------------------
# Per-agent keys and values (materialised)
# ----------------------------------------------------------------------------
def agent_keys(k_base_h, lr_k, B_k_h, lora_scale: float, positions, rope_base: float):
    """K^a = K_base + RoPE_t(s * LRk_t B_k^a[:, head]) for one KV head.

    k_base_h [L, d], lr_k [L, r], B_k_h [r, d]."""
    delta = lora_scale * (_np64(lr_k) @ _np64(B_k_h))
    return _np64(k_base_h) + rope(delta, positions, rope_base)


def agent_values(v_base_h, lr_v, B_v_h, lora_scale: float):
    """V^a = V_base + s * LRv B_v^a[:, head] for one KV head."""
    return _np64(v_base_h) + lora_scale * (_np64(lr_v) @ _np64(B_v_h))


# ----------------------------------------------------------------------------
# Naive two-pass softmax attention
# ----------------------------------------------------------------------------
def attention_probs(q, K, softmax_scale: float, q_positions, k_positions) -> np.ndarray:
    """P = softmax(q K^T * scale) with keys after the query's position masked out.

    q [n, d], K [L, d] -> P [n, L]; every row has at least one visible key."""
    s = (_np64(q) @ _np64(K).T) * softmax_scale
    visible = np.asarray(k_positions)[None, :] <= np.asarray(q_positions)[:, None]
    s = np.where(visible, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.where(visible, np.exp(s - m), 0.0)
    return e / e.sum(axis=1, keepdims=True)


def attention(q, K, V, softmax_scale: float, q_positions, k_positions) -> np.ndarray:
    return attention_probs(q, K, softmax_scale, q_positions, k_positions) @ _np64(V)


# ----------------------------------------------------------------------------
# Flash-LoRA-Attention, defined by materialisation
# ----------------------------------------------------------------------------
def query_positions(kv_len: int, n_q_tokens: int, mode: str, q_pos0: int = None):
    if mode == "decode":
        assert n_q_tokens == 1
        return np.array([kv_len - 1])
    q_pos0 = kv_len - n_q_tokens if q_pos0 is None else q_pos0
    return q_pos0 + np.arange(n_q_tokens)


def lora_attention_unit(k_base, v_base, lr, B_k, B_v, q, *, seq: int, agent: int,
                        kv_head: int, kv_len: int, q_positions, lora_scale: float,
                        softmax_scale: float, rope_base: float, q_heads=None,
                        q_tokens=None) -> np.ndarray:
    """Outputs of one (sequence, agent, KV head): every query head of its GQA group.

    Shapes as in ``lora_attention``.  Returns [n_tok_sel, g_sel, d] for the
    selected query tokens (default all) and query heads (default the group)."""
    d = k_base.shape[-1]
    r = lr.shape[-1] // 2
    n_q = q.shape[3]
    g = n_q // k_base.shape[1]
    L = int(kv_len)
    kpos = np.arange(L)
    # the agent's own LR cache (BaseShared), or the one shared by all agents
    lr_s = _np64(lr[agent, seq, :L] if lr.ndim == 4 else lr[seq, :L])
    cols = slice(kv_head * d, (kv_head + 1) * d)
    Ka = agent_keys(k_base[seq, kv_head, :L], lr_s[:, :r], _np64(B_k[agent])[:, cols],
                    lora_scale, kpos, rope_base)
    Va = agent_values(v_base[seq, kv_head, :L], lr_s[:, r:], _np64(B_v[agent])[:, cols],
                      lora_scale)
    q_positions = np.asarray(q_positions)
    toks = np.arange(len(q_positions)) if q_tokens is None else np.asarray(q_tokens)
    heads = range(kv_head * g, (kv_head + 1) * g) if q_heads is None else q_heads
    out = np.empty((len(toks), len(heads), d), dtype=f64)
    for hi, h in enumerate(heads):
        assert h // g == kv_head
        qh = _np64(q[seq, agent, :, h])[toks]
        out[:, hi] = attention(qh, Ka, Va, softmax_scale, q_positions[toks], kpos)
    return out


def lora_attention(k_base, v_base, lr, B_k, B_v, q, kv_len, *, lora_scale: float,
                   softmax_scale: float, rope_base: float, mode: str,
                   q_pos0: int = None) -> np.ndarray:
    """Every agent's attention output over the shared base and LR caches.

    k_base, v_base [n_seqs, n_kv, L_max, d]; lr [n_seqs, L_max, 2r] shared by
    every agent, or [n_agents, n_seqs, L_max, 2r], one cache per agent;
    B_k, B_v [n_agents, r, n_kv*d]; q [n_seqs, n_agents, n_tok, n_q, d];
    kv_len [n_seqs].  Returns out [n_seqs, n_agents, n_tok, n_q, d] in fp64.
    """
    n_seqs, n_kv = k_base.shape[0], k_base.shape[1]
    n_agents, n_tok, n_q, d = q.shape[1], q.shape[2], q.shape[3], q.shape[4]
    g = n_q // n_kv
    out = np.empty((n_seqs, n_agents, n_tok, n_q, d), dtype=f64)
    kv_len = [int(x) for x in _np64(kv_len).reshape(-1)]
    for s_ in range(n_seqs):
        qpos = query_positions(kv_len[s_], n_tok, mode, q_pos0)
        for a in range(n_agents):
            for j in range(n_kv):
                out[s_, a, :, j * g:(j + 1) * g] = lora_attention_unit(
                    k_base, v_base, lr, B_k, B_v, q, seq=s_, agent=a, kv_head=j,
                    kv_len=kv_len[s_], q_positions=qpos, lora_scale=lora_scale,
                    softmax_scale=softmax_scale, rope_base=rope_base)
    return out


# ----------------------------------------------------------------------------
# Sequence-sharded decode: one slice of the keys, and the merge of slices
# ----------------------------------------------------------------------------
# The pages show no multi-device step.  A device holding keys [lo, hi) of a
# sequence decodes over those keys alone; the attention over all keys is the
# merge of the slices' results by the online-softmax rescale (the same merge
# that combines the splits of one device's decode).
def decode_slice(k_base, v_base, lr, B_k, B_v, q, *, seq: int, agent: int, kv_head: int,
                 lo: int, hi: int, lora_scale: float, softmax_scale: float, rope_base: float):
    """Decode of one (sequence, agent, KV head) over keys [lo, hi) only, at
    their own positions lo .. hi - 1.  Returns (out [g, d], M [g], L [g]):
    out = softmax over the slice's keys times V^a, M = max_t (q . K^a_t) *
    softmax_scale * log2(e), L = sum_t 2^((q . K^a_t) * softmax_scale *
    log2(e) - M); an empty slice gives out 0, M = -inf, L = 0."""
    d = k_base.shape[-1]
    r = lr.shape[-1] // 2
    g = q.shape[3] // k_base.shape[1]
    heads = range(kv_head * g, (kv_head + 1) * g)
    if hi <= lo:
        return np.zeros((g, d)), np.full(g, -np.inf), np.zeros(g)
    kpos = np.arange(lo, hi)
    lr_s = _np64(lr[agent, seq, lo:hi] if lr.ndim == 4 else lr[seq, lo:hi])
    cols = slice(kv_head * d, (kv_head + 1) * d)
    Ka = agent_keys(k_base[seq, kv_head, lo:hi], lr_s[:, :r], _np64(B_k[agent])[:, cols],
                    lora_scale, kpos, rope_base)
    Va = agent_values(v_base[seq, kv_head, lo:hi], lr_s[:, r:], _np64(B_v[agent])[:, cols],
                      lora_scale)
    qh = _np64(q[seq, agent, 0])[list(heads)]             # [g, d]
    z = (qh @ Ka.T) * softmax_scale * np.log2(np.e)        # scores in log2 units
    M = z.max(axis=1)
    e = np.exp2(z - M[:, None])
    L = e.sum(axis=1)
    return (e / L[:, None]) @ Va, M, L


def combine_slices(outs, Ms, Ls) -> np.ndarray:
    """Merge of slice results of the same rows: outs [n, rows, d], Ms, Ls
    [n, rows].  w_p = 2^(M_p - M*) L_p with M* = max_p M_p;
    out = sum_p w_p out_p / sum_p w_p (0 where no slice has keys)."""
    outs, Ms, Ls = _np64(outs), _np64(Ms), _np64(Ls)
    Mx = Ms.max(axis=0)
    w = np.where(Ls > 0, np.exp2(Ms - np.where(np.isfinite(Mx), Mx, 0.0)[None]) * Ls, 0.0)
    tot = w.sum(axis=0)
    return np.where(tot[..., None] > 0, (w[..., None] * outs).sum(axis=0) / np.where(tot > 0, tot, 1.0)[..., None], 0.0)
