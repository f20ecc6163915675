"""Pins for the fp64 oracle, each against something other than the oracle itself.

* closed forms of RoPE (identity at position 0, exact angle t on the first pair,
  theta_1 = base^(-2/d)) and an independent complex-number formulation of it;
* B^a = 0 reduces Flash-LoRA-Attention to plain GQA attention over the base
  cache (the FullShared case of LRAgent §4) -- checked against PyTorch's
  fp64 CPU scaled_dot_product_attention;
* brute force: per-agent caches built directly from merged weights
  W + s A B^a (dW = A B, LRAgent App. A.3), rotated by the complex-form RoPE,
  then attended with PyTorch SDPA, must equal the oracle's decomposed path;
* reordering identity P (V_base + s V_lr B) = P V_base + s (P V_lr) B
  (LRAgent explainer, Metodologia 3 "Flash-LoRA-Attention");
* softmax rows sum to one, one visible key returns that key's value, agent
  permutation permutes outputs, future keys do not change a prefill row;
* the LR append against a pure-Python triple loop with guard rows;
* planted mistakes: each plausible bug, planted in the oracle on the CPU, makes
  at least one of these pins fail.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F


from oracle import impl


# ---------------------------------------------------------------- helpers ---
def complex_rope(x, positions, base):
    """RoFormer-style rotation written with complex numbers: pair (x_i, x_{i+d/2})
    is the complex number x_i + j x_{i+d/2}, multiplied by exp(j t theta_i)."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    h = d // 2
    theta = 1.0 / (float(base) ** (np.arange(0, d, 2, dtype=np.float64) / d))
    z = x[..., :h] + 1j * x[..., h:]
    z = z * np.exp(1j * np.asarray(positions, dtype=np.float64)[:, None] * theta[None, :])
    return np.concatenate([z.real, z.imag], axis=-1)


def sdpa_gqa(q, K, V, scale, q_pos, k_pos):
    """torch fp64 SDPA; q [n_q, n_tok, d], K/V [n_kv, L, d]; GQA by repeat_interleave."""
    n_q, n_kv = q.shape[0], K.shape[0]
    g = n_q // n_kv
    Kt = torch.from_numpy(np.repeat(K, g, axis=0))
    Vt = torch.from_numpy(np.repeat(V, g, axis=0))
    mask = torch.from_numpy(np.asarray(k_pos)[None, :] <= np.asarray(q_pos)[:, None])
    return F.scaled_dot_product_attention(torch.from_numpy(q), Kt, Vt, attn_mask=mask,
                                          scale=scale).numpy()


def tiny_problem(seed=0, n_seqs=2, n_agents=3, n_q=4, n_kv=2, d=8, H=16, r=2, L=7,
                 n_tok=3, alpha=6.0, base=100.0):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((n_seqs, L, H))
    W_k = rng.standard_normal((H, n_kv * d)) / math.sqrt(H)
    W_v = rng.standard_normal((H, n_kv * d)) / math.sqrt(H)
    A_k = rng.standard_normal((H, r)) / math.sqrt(H)
    A_v = rng.standard_normal((H, r)) / math.sqrt(H)
    B_k = rng.standard_normal((n_agents, r, n_kv * d))
    B_v = rng.standard_normal((n_agents, r, n_kv * d))
    q = rng.standard_normal((n_seqs, n_agents, n_tok, n_q, d))
    return dict(X=X, W_k=W_k, W_v=W_v, A_k=A_k, A_v=A_v, B_k=B_k, B_v=B_v, q=q,
                s=alpha / r, base=base, n_kv=n_kv, d=d, L=L, n_tok=n_tok)


def brute_force(p, mode):
    """Per-agent caches from merged weights, complex RoPE, torch SDPA."""
    X, q = p["X"], p["q"]
    n_seqs, n_agents, n_tok, n_q, d = q.shape
    n_kv, L = p["n_kv"], p["L"]
    out = np.empty(q.shape)
    kpos = np.arange(L)
    qpos = np.array([L - 1]) if mode == "decode" else np.arange(L - n_tok, L)
    for s_ in range(n_seqs):
        for a in range(n_agents):
            Wk = p["W_k"] + p["s"] * p["A_k"] @ p["B_k"][a]
            Wv = p["W_v"] + p["s"] * p["A_v"] @ p["B_v"][a]
            K = (X[s_] @ Wk).reshape(L, n_kv, d).transpose(1, 0, 2)
            V = (X[s_] @ Wv).reshape(L, n_kv, d).transpose(1, 0, 2)
            K = complex_rope(K, kpos, p["base"])
            qa = q[s_, a].transpose(1, 0, 2)  # [n_q, n_tok, d]
            o = sdpa_gqa(qa, K, V, 1 / math.sqrt(d), qpos, kpos)
            out[s_, a] = o.transpose(1, 0, 2)
    return out


def oracle_from_hidden(p, mode):
    k_base, v_base = impl.base_cache_from_hidden(p["X"], p["W_k"], p["W_v"], p["n_kv"],
                                                   p["base"])
    lr = impl.lr_cache_rows(p["X"], np.concatenate([p["A_k"], p["A_v"]], axis=1))
    kv_len = np.full(p["X"].shape[0], p["L"])
    q = p["q"] if mode == "prefill" else p["q"][:, :, -1:]
    return impl.lora_attention(k_base, v_base, lr, p["B_k"], p["B_v"], q, kv_len,
                                 lora_scale=p["s"], softmax_scale=1 / math.sqrt(p["d"]),
                                 rope_base=p["base"], mode=mode)


def brute_force_error(mode="prefill", seed=0, **kw):
    p = tiny_problem(seed=seed, **kw)
    ref = brute_force(p if mode == "prefill" else dict(p, q=p["q"][:, :, -1:]), mode)
    got = oracle_from_hidden(p, mode)
    return np.abs(got - ref).max() / np.abs(ref).max()


def b_zero_error(seed=1, mode="prefill"):
    """Oracle with B = 0 against fp64 SDPA over the base cache (FullShared)."""
    rng = np.random.default_rng(seed)
    n_seqs, n_agents, n_q, n_kv, d, L, r, n_tok = 2, 2, 6, 2, 16, 11, 4, 4
    k_base = rng.standard_normal((n_seqs, n_kv, L, d))
    v_base = rng.standard_normal((n_seqs, n_kv, L, d))
    lr = rng.standard_normal((n_seqs, L, 2 * r))
    B0 = np.zeros((n_agents, r, n_kv * d))
    if mode == "decode":
        n_tok = 1
    q = rng.standard_normal((n_seqs, n_agents, n_tok, n_q, d))
    kv_len = np.full(n_seqs, L)
    scale = 0.3
    got = impl.lora_attention(k_base, v_base, lr, B0, B0, q, kv_len, lora_scale=2.0,
                                softmax_scale=scale, rope_base=10000.0, mode=mode)
    qpos = np.arange(L - n_tok, L)
    err = 0.0
    for s_ in range(n_seqs):
        for a in range(n_agents):
            ref = sdpa_gqa(q[s_, a].transpose(1, 0, 2), k_base[s_], v_base[s_], scale, qpos,
                           np.arange(L)).transpose(1, 0, 2)
            err = max(err, np.abs(got[s_, a] - ref).max() / np.abs(ref).max())
    return err


# ------------------------------------------------------------------ RoPE ----
def test_rope_closed_forms():
    d, base = 8, 10000.0
    x = np.arange(1.0, 9.0)[None, :]
    # position 0 is the identity
    np.testing.assert_array_equal(impl.rope(x, [0], base), x)
    # theta_0 = 1: the first pair (x_0, x_4) turns by exactly t radians
    t = 3.0
    y = impl.rope(x, [t], base)
    assert y[0, 0] == pytest.approx(1 * math.cos(t) - 5 * math.sin(t), abs=1e-14)
    assert y[0, 4] == pytest.approx(5 * math.cos(t) + 1 * math.sin(t), abs=1e-14)
    # theta_1 = base^(-2/d): the second pair (x_1, x_5) turns by t * 10000^(-1/4) = t / 10
    a = t / 10.0
    assert y[0, 1] == pytest.approx(2 * math.cos(a) - 6 * math.sin(a), abs=1e-14)
    assert y[0, 5] == pytest.approx(6 * math.cos(a) + 2 * math.sin(a), abs=1e-14)
    np.testing.assert_allclose(impl.rope_inv_freq(8, 10000.0),
                               [1.0, 0.1, 0.01, 0.001], rtol=1e-15)


def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((5, 3, 16))
    pos = np.array([[0, 1, 2], [5, 17, 33], [100, 4096, 8191], [9000, 32768, 65535],
                    [131069, 131070, 131071]])
    for base in (10000.0, 500000.0):
        for row in range(5):
            np.testing.assert_allclose(impl.rope(x[row], pos[row], base),
                                       complex_rope(x[row], pos[row], base), atol=1e-12)


def test_rope_norm_and_relative_position():
    rng = np.random.default_rng(4)
    qv, kv = rng.standard_normal((1, 32)), rng.standard_normal((1, 32))
    for m, n in [(5, 2), (1000, 17), (70000, 3)]:
        a = impl.rope(qv, [m], 500000.0) @ impl.rope(kv, [n], 500000.0).T
        b = impl.rope(qv, [m + 123], 500000.0) @ impl.rope(kv, [n + 123], 500000.0).T
        assert a[0, 0] == pytest.approx(b[0, 0], rel=1e-9, abs=1e-9)
        assert np.linalg.norm(impl.rope(qv, [m], 500000.0)) == pytest.approx(
            np.linalg.norm(qv), rel=1e-13)


# ------------------------------------------------------------ attention -----
@pytest.mark.parametrize("mode", ["prefill", "decode"])
def test_b_zero_is_plain_gqa_attention(mode):
    assert b_zero_error(mode=mode) < 1e-12


@pytest.mark.parametrize("mode", ["prefill", "decode"])
@pytest.mark.parametrize("seed", [0, 1])
def test_brute_force_merged_weights(mode, seed):
    assert brute_force_error(mode=mode, seed=seed) < 1e-12


def test_brute_force_llama_like_rope_base():
    assert brute_force_error(seed=2, d=16, r=4, L=9, n_tok=4, base=500000.0) < 1e-12


# ------------------------------------------------ one LR cache per agent ----
def per_agent_problem(seed=3, **kw):
    """The tiny problem with a down-projection A_a of its own for every agent
    (BaseShared: only the base cache is shared)."""
    p = tiny_problem(seed=seed, **kw)
    rng = np.random.default_rng(100 + seed)
    n_agents, H, r = p["B_k"].shape[0], p["X"].shape[-1], p["B_k"].shape[1]
    p["A_k"] = rng.standard_normal((n_agents, H, r)) / math.sqrt(H)
    p["A_v"] = rng.standard_normal((n_agents, H, r)) / math.sqrt(H)
    return p


def per_agent_brute_force_error(mode="prefill", seed=3, **kw):
    """Per-agent merged weights W + s A_a B_a against the oracle fed every agent's
    own LR cache X A_a (filled by the per-agent append)."""
    p = per_agent_problem(seed=seed, **kw)
    n_agents = p["B_k"].shape[0]
    q = p["q"] if mode == "prefill" else p["q"][:, :, -1:]
    ref = np.empty(q.shape)
    for a in range(n_agents):
        pa = dict(p, A_k=p["A_k"][a], A_v=p["A_v"][a], B_k=p["B_k"][a:a + 1],
                  B_v=p["B_v"][a:a + 1], q=q[:, a:a + 1])
        ref[:, a:a + 1] = brute_force(pa, mode)
    k_base, v_base = impl.base_cache_from_hidden(p["X"], p["W_k"], p["W_v"], p["n_kv"], p["base"])
    A_kv = np.concatenate([p["A_k"], p["A_v"]], axis=2)       # [n_agents, H, 2r]
    n_seqs, L = p["X"].shape[0], p["L"]
    lr = impl.lr_cache_append_agents(np.zeros((n_agents, n_seqs, L, A_kv.shape[2])), p["X"], A_kv, 0)
    got = impl.lora_attention(k_base, v_base, lr, p["B_k"], p["B_v"], q, np.full(n_seqs, L),
                              lora_scale=p["s"], softmax_scale=1 / math.sqrt(p["d"]),
                              rope_base=p["base"], mode=mode)
    return np.abs(got - ref).max() / np.abs(ref).max()


@pytest.mark.parametrize("mode", ["prefill", "decode"])
def test_brute_force_per_agent_down_projections(mode):
    assert per_agent_brute_force_error(mode=mode) < 1e-12


def test_per_agent_caches_all_equal_reduce_to_the_shared_cache():
    rng = np.random.default_rng(7)
    n_seqs, n_agents, n_q, n_kv, d, L, r = 2, 3, 4, 2, 8, 9, 2
    k_base = rng.standard_normal((n_seqs, n_kv, L, d))
    v_base = rng.standard_normal((n_seqs, n_kv, L, d))
    lr = rng.standard_normal((n_seqs, L, 2 * r))
    B_k, B_v = rng.standard_normal((2, n_agents, r, n_kv * d))
    q = rng.standard_normal((n_seqs, n_agents, 3, n_q, d))
    kw = dict(lora_scale=1.5, softmax_scale=0.3, rope_base=100.0, mode="prefill")
    shared = impl.lora_attention(k_base, v_base, lr, B_k, B_v, q, np.full(n_seqs, L), **kw)
    each = impl.lora_attention(k_base, v_base, np.stack([lr] * n_agents), B_k, B_v, q,
                               np.full(n_seqs, L), **kw)
    np.testing.assert_array_equal(shared, each)


def test_per_agent_append_against_python_loops():
    rng = np.random.default_rng(8)
    n_agents, n_seqs, L, H, r, n, pos0 = 2, 2, 6, 5, 2, 3, 2
    X = rng.standard_normal((n_seqs, n, H))
    A = rng.standard_normal((n_agents, H, 2 * r))
    old = rng.standard_normal((n_agents, n_seqs, L, 2 * r))
    got = impl.lr_cache_append_agents(old, X, A, pos0)
    for a in range(n_agents):
        for q in range(n_seqs):
            for t in range(L):
                for c in range(2 * r):
                    if pos0 <= t < pos0 + n:
                        want = sum(X[q, t - pos0, k] * A[a, k, c] for k in range(H))
                    else:
                        want = old[a, q, t, c]
                    assert abs(got[a, q, t, c] - want) <= 1e-12 * (1 + abs(want))


def _bad_unit_first_agents_cache(k_base, v_base, lr, B_k, B_v, q, **kw):
    # reads agent 0's LR cache for every agent
    lr2 = np.asarray(impl._np64(lr))
    if lr2.ndim == 4:
        lr2 = np.stack([lr2[0]] * lr2.shape[0])
    return _orig_unit(k_base, v_base, lr2, B_k, B_v, q, **kw)


def test_planted_per_agent_cache_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(impl, "lora_attention_unit", _bad_unit_first_agents_cache)
    assert per_agent_brute_force_error(mode="prefill") > 1e-6


# --------------------------------------- query- and output-side LoRA ----
def qo_problem(seed=11, n_tok=5, H=12, n_q=4, d=8, r=3, D_out=10, alpha=4.5):
    rng = np.random.default_rng(seed)
    return dict(X=rng.standard_normal((n_tok, H)), W_q=rng.standard_normal((H, n_q * d)),
                A_q=rng.standard_normal((H, r)), B_q=rng.standard_normal((r, n_q * d)),
                W_o=rng.standard_normal((n_q * d, D_out)), A_o=rng.standard_normal((n_q * d, r)),
                B_o=rng.standard_normal((r, D_out)), s=alpha / r, n_q=n_q, d=d,
                pos=np.arange(7, 7 + n_tok))


def query_lora_error(seed=11, base=100.0):
    """Merged weights W_q + s A_q B_q, projected and rotated with the complex
    RoPE, against the decomposed oracle."""
    p = qo_problem(seed)
    n_tok = p["X"].shape[0]
    merged = (p["X"] @ (p["W_q"] + p["s"] * p["A_q"] @ p["B_q"])).reshape(n_tok, p["n_q"], p["d"])
    ref = complex_rope(merged.transpose(1, 0, 2), p["pos"], base).transpose(1, 0, 2)
    got = impl.lora_queries((p["X"] @ p["W_q"]).reshape(n_tok, p["n_q"], p["d"]),
                            p["X"] @ p["A_q"], p["B_q"], p["s"], p["pos"], base)
    return np.abs(got - ref).max() / np.abs(ref).max()


def test_query_lora_against_merged_weights():
    assert query_lora_error() < 1e-12
    assert query_lora_error(seed=12, base=500000.0) < 1e-12


def test_output_lora_against_merged_weights():
    p = qo_problem(13)
    o = p["X"] @ p["W_q"]                                   # any [n_tok, n_q*d] attention output
    ref = o @ (p["W_o"] + p["s"] * p["A_o"] @ p["B_o"])
    got = impl.lora_output(o @ p["W_o"], o, p["A_o"], p["B_o"], p["s"])
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def _bad_queries_delta_after_rope(q_base, lr_q, B_q, lora_scale, positions, rope_base):
    qb = impl._np64(q_base)
    n_tok, n_q, d = qb.shape
    rot = impl.rope(qb.transpose(1, 0, 2), positions, rope_base).transpose(1, 0, 2)
    return rot + lora_scale * (impl._np64(lr_q) @ impl._np64(B_q)).reshape(n_tok, n_q, d)


def test_planted_query_lora_mistake_is_caught(monkeypatch):
    monkeypatch.setattr(impl, "lora_queries", _bad_queries_delta_after_rope)
    assert query_lora_error() > 1e-6


def test_reordered_value_path_identity():
    rng = np.random.default_rng(5)
    L, d, r, s = 13, 16, 4, 2.0
    q, K = rng.standard_normal((3, d)), rng.standard_normal((L, d))
    Vb, Vlr, B = rng.standard_normal((L, d)), rng.standard_normal((L, r)), rng.standard_normal((r, d))
    P = impl.attention_probs(q, K, 0.25, np.array([L - 1] * 3), np.arange(L))
    full = P @ impl.agent_values(Vb, Vlr, B, s)
    reordered = P @ Vb + s * (P @ Vlr) @ B
    np.testing.assert_allclose(full, reordered, rtol=1e-12, atol=1e-12)


def test_softmax_rows_sum_to_one():
    rng = np.random.default_rng(6)
    q, K = rng.standard_normal((7, 8)) * 5, rng.standard_normal((20, 8)) * 5
    qpos = np.array([0, 3, 5, 10, 19, 19, 2])
    P = impl.attention_probs(q, K, 1.0, qpos, np.arange(20))
    assert (P >= 0).all()
    assert np.abs(P.sum(axis=1) - 1).max() < 1e-14
    assert (P[np.arange(20)[None, :] > qpos[:, None]] == 0).all()


def test_single_visible_key_returns_its_value():
    p = tiny_problem(seed=7, L=1, n_tok=1)
    out = oracle_from_hidden(p, "decode")
    k_base, v_base = impl.base_cache_from_hidden(p["X"], p["W_k"], p["W_v"], p["n_kv"], p["base"])
    lr = impl.lr_cache_rows(p["X"], np.concatenate([p["A_k"], p["A_v"]], 1))
    d, g = p["d"], p["q"].shape[3] // p["n_kv"]
    for s_ in range(out.shape[0]):
        for a in range(out.shape[1]):
            for h in range(out.shape[3]):
                j = h // g
                Va = impl.agent_values(v_base[s_, j], lr[s_, :, 2:], p["B_v"][a][:, j * d:(j + 1) * d], p["s"])
                np.testing.assert_allclose(out[s_, a, 0, h], Va[0], rtol=1e-12, atol=1e-12)


def test_agent_permutation_permutes_outputs():
    p = tiny_problem(seed=8)
    out = oracle_from_hidden(p, "prefill")
    perm = [2, 0, 1]
    pp = dict(p, B_k=p["B_k"][perm], B_v=p["B_v"][perm], q=p["q"][:, perm])
    np.testing.assert_allclose(oracle_from_hidden(pp, "prefill"), out[:, perm], rtol=1e-13, atol=1e-13)


def test_prefill_rows_ignore_future_keys():
    p = tiny_problem(seed=9, L=9, n_tok=4)
    out = oracle_from_hidden(p, "prefill")
    X2 = p["X"].copy()
    X2[:, -1] += 10.0  # changes the last token's key, value and LR rows
    out2 = oracle_from_hidden(dict(p, X=X2), "prefill")
    np.testing.assert_array_equal(out[:, :, :-1], out2[:, :, :-1])
    assert np.abs(out[:, :, -1] - out2[:, :, -1]).max() > 1e-3


def test_decode_equals_last_prefill_row():
    p = tiny_problem(seed=10)
    pre = oracle_from_hidden(p, "prefill")
    dec = oracle_from_hidden(p, "decode")
    np.testing.assert_allclose(dec[:, :, 0], pre[:, :, -1], rtol=1e-13, atol=1e-13)


# ------------------------------------------------------------- LR append ----
def test_lr_append_against_python_loops():
    rng = np.random.default_rng(11)
    n_seqs, n, H, r, L_max, pos0 = 2, 3, 5, 2, 8, 4
    X = rng.standard_normal((n_seqs, n, H))
    A = rng.standard_normal((H, 2 * r))
    cache = np.full((n_seqs, L_max, 2 * r), -7.25)
    out = impl.lr_cache_append(cache, X, A, pos0)
    for s_ in range(n_seqs):
        for t in range(L_max):
            for c in range(2 * r):
                if pos0 <= t < pos0 + n:
                    acc = 0.0
                    for k in range(H):
                        acc += X[s_, t - pos0, k] * A[k, c]
                    assert out[s_, t, c] == pytest.approx(acc, rel=1e-13, abs=1e-13)
                else:
                    assert out[s_, t, c] == -7.25


# ------------------------------------------------------- planted mistakes ---
def _bad_rope_sign(x, positions, rope_base):
    x = impl._np64(x)
    h = x.shape[-1] // 2
    ang = np.asarray(positions, dtype=np.float64)[:, None] * impl.rope_inv_freq(x.shape[-1], rope_base)
    c, s = np.cos(ang), np.sin(ang)
    return np.concatenate([x[..., :h] * c + x[..., h:] * s, x[..., h:] * c - x[..., :h] * s], -1)


def _bad_rope_adjacent_pairs(x, positions, rope_base):
    x = impl._np64(x)
    d = x.shape[-1]
    ang = np.asarray(positions, dtype=np.float64)[:, None] * impl.rope_inv_freq(d, rope_base)
    c, s = np.cos(ang), np.sin(ang)
    y = x.copy()
    y[..., 0::2] = x[..., 0::2] * c - x[..., 1::2] * s
    y[..., 1::2] = x[..., 1::2] * c + x[..., 0::2] * s
    return y


def _bad_inv_freq(head_dim, rope_base):
    i = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(np.float64(rope_base), -1.0 * i / head_dim)


def _bad_values_no_scale(v_base_h, lr_v, B_v_h, lora_scale):
    return impl._np64(v_base_h) + impl._np64(lr_v) @ impl._np64(B_v_h)


def _bad_keys_unrotated_delta(k_base_h, lr_k, B_k_h, lora_scale, positions, rope_base):
    return impl._np64(k_base_h) + lora_scale * (impl._np64(lr_k) @ impl._np64(B_k_h))


def _bad_mask_strict(q, K, softmax_scale, q_positions, k_positions):
    s = (impl._np64(q) @ impl._np64(K).T) * softmax_scale
    vis = np.asarray(k_positions)[None, :] < np.maximum(np.asarray(q_positions)[:, None], 1)
    s = np.where(vis, s, -np.inf)
    e = np.where(vis, np.exp(s - s.max(1, keepdims=True)), 0.0)
    return e / e.sum(1, keepdims=True)


def _bad_lr_swapped(X, A_kv):
    rows = impl._np64(X) @ impl._np64(A_kv)
    r = rows.shape[-1] // 2
    return np.concatenate([rows[..., r:], rows[..., :r]], -1)


_orig_unit = impl.lora_attention_unit


def _bad_gqa_mapping(k_base, v_base, lr, B_k, B_v, q, **kw):
    # reads KV head (h mod n_kv) instead of floor(h / g): swap the group's heads
    n_kv = k_base.shape[1]
    kw = dict(kw)
    kw["kv_head"] = (kw["kv_head"] + 1) % n_kv if n_kv > 1 else kw["kv_head"]
    q2 = np.asarray(impl._np64(q))
    g = q2.shape[3] // n_kv
    j = kw["kv_head"]
    q3 = q2.copy()
    src = (j - 1) % n_kv
    q3[:, :, :, j * g:(j + 1) * g] = q2[:, :, :, src * g:(src + 1) * g]
    return _orig_unit(k_base, v_base, lr, B_k, B_v, q3, **kw)


MUTATIONS = {
    "rope_sign": ("rope", _bad_rope_sign),
    "rope_adjacent_pairs": ("rope", _bad_rope_adjacent_pairs),
    "inv_freq_exponent": ("rope_inv_freq", _bad_inv_freq),
    "values_drop_scale": ("agent_values", _bad_values_no_scale),
    "keys_delta_unrotated": ("agent_keys", _bad_keys_unrotated_delta),
    "mask_strict": ("attention_probs", _bad_mask_strict),
    "lr_parts_swapped": ("lr_cache_rows", _bad_lr_swapped),
    "gqa_mapping": ("lora_attention_unit", _bad_gqa_mapping),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, bad = MUTATIONS[name]
    monkeypatch.setattr(impl, attr, bad)
    errs = [brute_force_error(mode="prefill", seed=0), brute_force_error(mode="decode", seed=1),
            b_zero_error(mode="prefill")]
    try:
        test_rope_closed_forms()
        rope_ok = True
    except AssertionError:
        rope_ok = False
    assert max(errs) > 1e-6 or not rope_ok, f"mistake {name} slipped through: {errs}"
