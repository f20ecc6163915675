"""The KV-cache memory accounting of the sharing schemes, pinned twice: to the
sizes of the buffers the library actually reads (the workload's caches and
the non-shared baseline's materialised K^a, V^a), and to the pages' closed
forms for the fraction of non-shared caching (tests/golden/memory_ratios.txt,
LRAgent summary §3 Methodology, BaseShared and BaseLRShared)."""
import os
from fractions import Fraction

import pytest

import bench
from rank_attention_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "memory_ratios.txt")

SHAPES = [W.LLAMA8B_DECODE_8K, W.llama8b_sweep(32768), W.llama8b_stack_decode(0),
          W.LLAMA8B_DECODE_8K.replace(n_agents=5, r=64, n_seqs=3)]


def golden_fractions():
    out = {}
    for line in open(GOLDEN):
        line = line.strip()
        if line and not line.startswith("#"):
            scheme, expr = line.split(None, 1)
            out[scheme] = expr
    return out


def nbytes(t):
    return t.numel() * t.element_size()


def test_golden_lists_both_shared_schemes():
    assert set(golden_fractions()) == {"base_shared", "base_lr_shared"}


@pytest.mark.parametrize("s", SHAPES, ids=lambda s: s.name)
def test_fractions_match_the_pages_closed_forms(s):
    ns = bench.kv_cache_bytes(s, "non_shared")
    env = {"N": Fraction(s.n_agents), "r": Fraction(s.r),
           "d_out": Fraction(s.n_kv_heads * s.head_dim)}
    for scheme, expr in golden_fractions().items():
        want = eval(expr, {"__builtins__": {}}, env)
        assert Fraction(bench.kv_cache_bytes(s, scheme), ns) == want, scheme


def test_llama8b_three_agents_values():
    # N = 3, r = 16, d_out = 8 * 128: 1/3 + 1/64 and 1/3 + 1/192
    rep = bench.kv_cache_report(W.LLAMA8B_DECODE_8K)["vs_non_shared"]
    assert rep["non_shared"] == 1.0
    assert rep["base_shared"] == pytest.approx(1 / 3 + 1 / 64, rel=1e-15)
    assert rep["base_lr_shared"] == pytest.approx(1 / 3 + 1 / 192, rel=1e-15)


@pytest.mark.parametrize("per_agent", [False, True])
def test_counts_equal_the_buffers_the_library_reads(per_agent):
    from rank_attention_b200 import lora_attn as la
    s = W.LLAMA8B_DECODE_8K.replace(kv_len=256, n_seqs=2, lr_per_agent=per_agent)
    inp = W.direct_cache_inputs(s)
    shared = nbytes(inp["k_base"]) + nbytes(inp["v_base"]) + nbytes(inp["lr"])
    scheme = "base_shared" if per_agent else "base_lr_shared"
    assert bench.kv_cache_bytes(s, scheme) == shared
    # the non-shared baseline's per-agent caches, as its setup allocates them
    # (argument marshalling and allocation only: nothing is launched)
    mat, _, _ = bench.non_shared_setup(la, s, inp, "cpu")
    kout, vout = mat.keep[0], mat.keep[1]
    assert bench.kv_cache_bytes(s, "non_shared") == nbytes(kout) + nbytes(vout)
