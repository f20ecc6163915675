"""Property-based pin of the oracle: the merged-weight brute force against the
oracle's decomposed path on random small shapes (hypothesis).  Kept apart from
the other pins so that, where hypothesis is not installed, only this test is
skipped."""
import pytest

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import given, settings, strategies as st  # noqa: E402

from tests.test_oracle_pins import brute_force_error  # noqa: E402


@settings(max_examples=30, deadline=None, derandomize=True)
@given(seed=st.integers(0, 2**31 - 1), n_agents=st.integers(1, 4), n_kv=st.integers(1, 3),
       g=st.integers(1, 3), half_d=st.sampled_from([2, 4, 8]), r=st.sampled_from([1, 2, 4]),
       L=st.integers(1, 9), n_tok_frac=st.floats(0.0, 1.0), base=st.sampled_from([50.0, 1e4]),
       mode=st.sampled_from(["decode", "prefill"]))
def test_brute_force_on_random_shapes(seed, n_agents, n_kv, g, half_d, r, L, n_tok_frac, base,
                                      mode):
    """The merged-weight brute force and the oracle's decomposed path agree on
    random small shapes: GQA group sizes, head widths, ranks, lengths down to
    one key, chunks from one query to the whole sequence."""
    n_tok = max(1, round(n_tok_frac * L))
    err = brute_force_error(mode, seed=seed, n_seqs=1, n_agents=n_agents, n_q=n_kv * g,
                            n_kv=n_kv, d=2 * half_d, H=8, r=r, L=L, n_tok=n_tok,
                            alpha=2.0 * r, base=base)
    assert err <= 1e-12


@settings(max_examples=25, deadline=None, derandomize=True)
@given(seed=st.integers(0, 2**31 - 1), L=st.integers(1, 40), n_cuts=st.integers(0, 5),
       g=st.integers(1, 3), half_d=st.sampled_from([2, 4, 8]), r=st.sampled_from([1, 2, 4]),
       data=st.data())
def test_slice_merge_on_random_cuts(seed, L, n_cuts, g, half_d, r, data):
    """The sequence-sharded decode's merge (decode_slice per slice, then
    combine_slices) equals the oracle's decode over all keys for random cut
    points, empty slices included, on random small shapes."""
    import numpy as np
    import torch

    from oracle import impl as O
    cuts = sorted(data.draw(st.lists(st.integers(0, L), min_size=n_cuts, max_size=n_cuts)))
    cuts = [0] + cuts + [L]
    d, n_kv, n_agents = 2 * half_d, 2, 2
    gen = torch.Generator().manual_seed(seed)
    rn = lambda *shape, sc=1.0: torch.randn(*shape, generator=gen, dtype=torch.float64) * sc
    inp = dict(k_base=rn(1, n_kv, L, d), v_base=rn(1, n_kv, L, d), lr=rn(1, L, 2 * r),
               B_k=rn(n_agents, r, n_kv * d, sc=0.3), B_v=rn(n_agents, r, n_kv * d, sc=0.3),
               q=rn(1, n_agents, 1, n_kv * g, d))
    kw = dict(lora_scale=1.5, softmax_scale=0.3, rope_base=500.0)
    for agent in range(n_agents):
        for j in range(n_kv):
            ref = O.lora_attention_unit(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"],
                                        inp["q"], seq=0, agent=agent, kv_head=j, kv_len=L,
                                        q_positions=[L - 1], **kw)[0]
            parts = [O.decode_slice(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"], inp["q"],
                                    seq=0, agent=agent, kv_head=j, lo=lo, hi=hi, **kw)
                     for lo, hi in zip(cuts[:-1], cuts[1:])]
            got = O.combine_slices(np.stack([p_[0] for p_ in parts]), np.stack([p_[1] for p_ in parts]),
                                   np.stack([p_[2] for p_ in parts]))
            np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-11)
