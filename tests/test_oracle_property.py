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
