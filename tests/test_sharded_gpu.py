"""Sequence-sharded decode on one GPU: every sequence's keys cut into slices,
each slice decoded on its own (key_pos0 = the slice's first position,
row_stats filled), and the slices merged by lora_attn_decode_combine.  Across
devices each slice would sit on its own GPU and the outputs and stats would be
all-gathered first; the arithmetic is this.  The merge must match the oracle's
decode over all keys, and each slice's (M, L) the oracle's slice statistics.
"""
import numpy as np
import pytest
import torch

from oracle import impl as oracle
from rank_attention_b200 import workloads as W
from tests.helpers import assert_parity, oracle_decode, to_device, to_np

DEV = "cuda"


@pytest.fixture(scope="module")
def la():
    from rank_attention_b200 import lora_attn
    return lora_attn


def _run_slices(la, s, d, kv_lens, cuts, out_dtype=torch.float32):
    """Decode every slice [cuts[i], cuts[i+1]) of the caches in d; returns the
    per-slice outputs [n, ...], stats [n, n_seqs, n_agents, n_q, 2] and the merge."""
    n_parts = len(cuts) - 1
    q = d["q"]
    outs = torch.full((n_parts,) + tuple(q.shape), float("nan"), dtype=out_dtype, device=DEV)
    stats = torch.full((n_parts, q.shape[0], q.shape[1], q.shape[3], 2), float("nan"), device=DEV)
    keep = []
    for pi, (lo, hi) in enumerate(zip(cuts[:-1], cuts[1:])):
        kvl = torch.tensor([min(max(k - lo, 0), hi - lo) for k in kv_lens], dtype=torch.int32, device=DEV)
        lr = d["lr"][..., lo:hi, :]
        args = la.make_args(d["k_base"][:, :, lo:hi], d["v_base"][:, :, lo:hi], lr, d["B_k"], d["B_v"], q,
                            outs[pi], lora_scale=s.lora_scale, rope_base=s.rope_base, kv_len=kvl,
                            max_kv_len=hi - lo, key_pos0=lo, row_stats=stats[pi])
        ws = la.decode_workspace(args, DEV)
        la.lora_attn_decode(args, ws)
        keep.append((kvl, ws))
    out = torch.empty(tuple(q.shape), dtype=out_dtype, device=DEV)
    la.lora_attn_decode_combine(outs, stats, out)
    torch.cuda.synchronize()
    assert la.la_device_check() == la.LA_OK
    return outs, stats, out


def _check_stats(s, inp, stats, cuts, kv_lens, units):
    """Each slice's (M, L) against the oracle's, on sampled (seq, agent, KV head)."""
    g = s.n_q_heads // s.n_kv_heads
    st = stats.cpu().double().numpy()
    for seq, agent, j in units:
        for pi, (lo, hi) in enumerate(zip(cuts[:-1], cuts[1:])):
            hi_q = min(hi, kv_lens[seq])
            _, M, L = oracle.decode_slice(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"],
                                          inp["q"], seq=seq, agent=agent, kv_head=j, lo=lo, hi=hi_q,
                                          lora_scale=s.lora_scale, softmax_scale=s.softmax_scale,
                                          rope_base=s.rope_base)
            gM, gL = st[pi, seq, agent, j * g:(j + 1) * g, 0], st[pi, seq, agent, j * g:(j + 1) * g, 1]
            if hi_q <= lo:   # no keys of this sequence in the slice
                assert np.all(np.isneginf(gM)) and np.all(gL == 0)
                continue
            assert np.all(np.abs(gM - M) <= 0.05 + 1e-2 * np.abs(M)), (gM, M)
            assert np.all(np.abs(gL - L) <= 2e-2 * L), (gL, L)


@pytest.mark.gpu
@pytest.mark.parametrize("r,n_agents", [(16, 3), (32, 3), (64, 1)])
def test_sharded_decode_merges_to_the_oracle(la, r, n_agents):
    """Two sequences of 2048 and 1000 keys cut at 640 and 1280: the second
    sequence has no keys in the last slice (kv_len 0 there)."""
    s = W.LLAMA8B_DECODE_8K.replace(kv_len=2048, n_seqs=2, r=r, n_agents=n_agents, seed=53)
    inp = W.direct_cache_inputs(s)
    kv_lens = [2048, 1000]
    inp["kv_len"] = torch.tensor(kv_lens, dtype=torch.int32)
    cuts = [0, 640, 1280, 2048]
    _, stats, out = _run_slices(la, s, to_device(inp), kv_lens, cuts)
    assert_parity(to_np(out), oracle_decode(inp, s), s.dtype)
    _check_stats(s, inp, stats, cuts, kv_lens, [(0, 0, 0), (1, n_agents - 1, 7), (0, n_agents - 1, 3)])


@pytest.mark.gpu
def test_sharded_llama8b_decode_8k_four_slices(la):
    """The 8192-token, 3-agent, r = 16 layer in four slices of 2048 keys (as on
    four GPUs), fp32 and bf16 outputs: the merge matches the oracle and the
    unsharded decode."""
    s = W.LLAMA8B_DECODE_8K
    inp = W.direct_cache_inputs(s)
    d = to_device(inp)
    kv_lens = [s.kv_len] * s.n_seqs
    cuts = [0, 2048, 4096, 6144, 8192]
    ref = oracle_decode(inp, s)
    whole = torch.empty(d["q"].shape, device=DEV)
    args = la.make_args(d["k_base"], d["v_base"], d["lr"], d["B_k"], d["B_v"], d["q"], whole,
                        lora_scale=s.lora_scale, rope_base=s.rope_base, kv_len=d["kv_len"],
                        max_kv_len=s.kv_len)
    la.lora_attn_decode(args, la.decode_workspace(args, DEV))
    for dt in (torch.float32, torch.bfloat16):
        _, stats, out = _run_slices(la, s, d, kv_lens, cuts, out_dtype=dt)
        assert_parity(to_np(out), ref, s.dtype)
        assert_parity(to_np(out), to_np(whole), s.dtype)
    _check_stats(s, inp, stats, cuts, kv_lens, [(0, 0, 0), (0, 2, 5)])


@pytest.mark.gpu
def test_combine_of_one_slice_is_the_identity(la):
    """One slice holding every key: the merge returns that slice's output."""
    s = W.LLAMA8B_DECODE_8K.replace(kv_len=1024, seed=59)
    inp = W.direct_cache_inputs(s)
    outs, _, out = _run_slices(la, s, to_device(inp), [1024], [0, 1024])
    torch.testing.assert_close(out, outs[0], rtol=1e-6, atol=0.0)
    assert_parity(to_np(out), oracle_decode(inp, s), s.dtype)
