"""Pins of the oracle's sequence-sharded decode (decode_slice, combine_slices).

Merging the slices' (out, M, L) must give the decode over all keys, which the
other oracle pins tie to the pages' definition; a single key gives the closed
form; planted mistakes (natural exp in the merge, slice positions from 0)
break the identity.
"""
import numpy as np
import pytest
import torch

from oracle import lora_attn_oracle as O


def _inputs(seed=3, n_seqs=2, n_agents=2, n_kv=2, g=2, d=16, r=4, L=37):
    gen = torch.Generator().manual_seed(seed)
    rn = lambda *shape, sc=1.0: torch.randn(*shape, generator=gen, dtype=torch.float64) * sc
    return dict(k_base=rn(n_seqs, n_kv, L, d), v_base=rn(n_seqs, n_kv, L, d), lr=rn(n_seqs, L, 2 * r),
                B_k=rn(n_agents, r, n_kv * d, sc=0.3), B_v=rn(n_agents, r, n_kv * d, sc=0.3),
                q=rn(n_seqs, n_agents, 1, n_kv * g, d))


KW = dict(lora_scale=2.0, softmax_scale=0.25, rope_base=10000.0)


def _full_unit(inp, seq, agent, j, L):
    return O.lora_attention_unit(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"], inp["q"],
                                 seq=seq, agent=agent, kv_head=j, kv_len=L, q_positions=[L - 1], **KW)[0]


def _sliced(inp, seq, agent, j, cuts, slice_fn=O.decode_slice, combine=O.combine_slices):
    parts = [slice_fn(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"], inp["q"], seq=seq,
                      agent=agent, kv_head=j, lo=lo, hi=hi, **KW) for lo, hi in zip(cuts[:-1], cuts[1:])]
    outs = np.stack([p_[0] for p_ in parts])
    Ms = np.stack([p_[1] for p_ in parts])
    Ls = np.stack([p_[2] for p_ in parts])
    return combine(outs, Ms, Ls)


@pytest.mark.parametrize("cuts", [(0, 37), (0, 10, 37), (0, 5, 5, 20, 36, 37), (0, 1, 2, 37), (0, 30, 37, 37)])
def test_slices_merge_to_the_whole_decode(cuts):
    """Every cut of [0, L) into slices (empty ones included) merges back to the
    decode over all keys, for every sequence, agent and KV head."""
    inp = _inputs()
    for seq in range(2):
        for agent in range(2):
            for j in range(2):
                ref = _full_unit(inp, seq, agent, j, 37)
                got = _sliced(inp, seq, agent, j, list(cuts))
                np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_single_key_slice_closed_form():
    """One key t: M is its scaled score in log2 units, L = 1, out = V^a_t."""
    inp = _inputs(seed=5)
    t, seq, agent, j, g, d, r = 17, 1, 0, 1, 2, 16, 4
    out, M, L = O.decode_slice(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"], inp["q"],
                               seq=seq, agent=agent, kv_head=j, lo=t, hi=t + 1, **KW)
    cols = slice(j * d, (j + 1) * d)
    delta = KW["lora_scale"] * (inp["lr"][seq, t, :r].numpy() @ inp["B_k"][agent][:, cols].numpy())
    k = inp["k_base"][seq, j, t].numpy() + O.rope(delta[None], [t], KW["rope_base"])[0]
    v = inp["v_base"][seq, j, t].numpy() + KW["lora_scale"] * (inp["lr"][seq, t, r:].numpy() @ inp["B_v"][agent][:, cols].numpy())
    qh = inp["q"][seq, agent, 0, j * g:(j + 1) * g].numpy()
    np.testing.assert_allclose(M, qh @ k * KW["softmax_scale"] * np.log2(np.e), rtol=1e-13)
    np.testing.assert_allclose(L, np.ones(g))
    np.testing.assert_allclose(out, np.stack([v, v]), rtol=1e-13)


def test_empty_slice():
    inp = _inputs()
    out, M, L = O.decode_slice(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"], inp["q"],
                               seq=0, agent=0, kv_head=0, lo=9, hi=9, **KW)
    assert np.all(out == 0) and np.all(np.isneginf(M)) and np.all(L == 0)


def test_planted_mistakes_break_the_merge():
    """A merge with natural exp instead of exp2, or slice keys RoPE'd from
    position 0 instead of lo, no longer reproduce the whole decode."""
    inp = _inputs(seed=7)
    cuts = [0, 12, 25, 37]
    ref = _full_unit(inp, 0, 1, 0, 37)

    def combine_e(outs, Ms, Ls):
        Mx = Ms.max(axis=0)
        w = np.exp(Ms - Mx[None]) * Ls
        return (w[..., None] * outs).sum(axis=0) / w.sum(axis=0)[..., None]

    def slice_pos0(k_base, v_base, lr, B_k, B_v, q, *, seq, agent, kv_head, lo, hi, **kw):
        # the slice as if it started at position 0
        sl = lambda x: x[:, :, lo:hi]
        return O.decode_slice(sl(k_base), sl(v_base), lr[:, lo:hi], B_k, B_v, q, seq=seq, agent=agent,
                              kv_head=kv_head, lo=0, hi=hi - lo, **kw)

    assert np.allclose(_sliced(inp, 0, 1, 0, cuts), ref, rtol=1e-12, atol=1e-12)
    assert not np.allclose(_sliced(inp, 0, 1, 0, cuts, combine=combine_e), ref, rtol=1e-6, atol=1e-6)
    assert not np.allclose(_sliced(inp, 0, 1, 0, cuts, slice_fn=slice_pos0), ref, rtol=1e-6, atol=1e-6)
