"""CUDA path vs the fp64 oracle, element by element, through the C ABI.

Small cases run the oracle on every output; the LLaMA-shaped cases run the
CUDA path at full size and compare every output the oracle can afford
(all of the 8k decode; sampled (agent, KV head, token) units elsewhere)."""
import math

import numpy as np
import pytest
import torch

from oracle import impl as oracle
from rank_attention_b200 import workloads as W
from tests.helpers import (assert_parity, bf16_ulp, errors, oracle_decode, to_device, to_np)

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module")
def la():
    from rank_attention_b200 import lora_attn
    return lora_attn


# ------------------------------------------------------------- LR append ----
def _append_case(la, n_seqs, n, H, r, dtype, L_max, pos0, seed):
    inp = W.append_inputs(n, H, r, dtype, seed, n_seqs=n_seqs)
    sentinel = -123.5
    lr = torch.full((n_seqs, L_max, 2 * r), sentinel, dtype=dtype, device=DEV)
    la.lr_cache_append(inp["X"].to(DEV), inp["A_kv"].to(DEV), lr, pos0)
    torch.cuda.synchronize()
    got = lr.cpu()
    ref = oracle.lr_cache_rows(inp["X"], inp["A_kv"])
    # rows outside [pos0, pos0 + n) untouched, bit for bit
    outside = torch.ones(L_max, dtype=torch.bool)
    outside[pos0:pos0 + n] = False
    assert (got[:, outside] == sentinel).all()
    rows = to_np(got[:, pos0:pos0 + n])
    if dtype == torch.float32:
        mx, _ = errors(rows, ref)
        assert mx <= 1e-5
    else:
        # the fp64 value rounded to bf16, within one bf16 ulp (fp32 accumulation order)
        bound = np.maximum(bf16_ulp(ref),
                           1e-6 * (np.abs(to_np(inp["X"])) @ np.abs(to_np(inp["A_kv"]))))
        assert (np.abs(rows - ref) <= bound).all(), np.abs(rows - ref).max()


def test_append_fp32_tiny(la):
    s = W.TINY_FP32
    _append_case(la, 1, s.kv_len, s.hidden, s.r, torch.float32, 300, 20, seed=0)


@pytest.mark.parametrize("r", [8, 16, 32, 64])
def test_append_bf16_ragged(la, r):
    _append_case(la, 2, 333, 4096, r, torch.bfloat16, 1000, 501, seed=r)


def test_append_bf16_single_row_and_last_slot(la):
    _append_case(la, 1, 1, 4096, 16, torch.bfloat16, 8192, 8191, seed=5)


def test_append_bf16_stack_chunk(la):
    # 4096-token chunk through r=64 shared A (one layer of the 32-layer stack)
    _append_case(la, 1, 4096, 4096, 64, torch.bfloat16, 4096 + 64, 37, seed=6)


def test_append_empty_is_noop(la):
    lr = torch.full((1, 8, 16), 3.0, device=DEV)
    X = torch.zeros((1, 0, 256), device=DEV)
    A = torch.zeros((256, 16), device=DEV)
    la.lr_cache_append(X, A, lr, 8)
    torch.cuda.synchronize()
    assert (lr == 3.0).all()


# ----------------------------------------------------- tiny fp32 (exact) ----
def _tiny_caches(shape, L_max=None):
    w = W.hidden_layer_weights(shape)
    kb, vb = oracle.base_cache_from_hidden(w["X"], w["W_k"], w["W_v"], shape.n_kv_heads,
                                           shape.rope_base)
    L = shape.kv_len
    L_max = L if L_max is None else L_max
    k_base = torch.zeros((shape.n_seqs, shape.n_kv_heads, L_max, shape.head_dim))
    v_base = torch.zeros_like(k_base)
    k_base[:, :, :L] = torch.from_numpy(kb).float()
    v_base[:, :, :L] = torch.from_numpy(vb).float()
    return w, k_base, v_base


def _run(la, shape, k_base, v_base, lr, B_k, B_v, q, kv_len=None, mode=None, out_dtype=None):
    mode = mode or shape.mode
    out = torch.empty(q.shape, dtype=out_dtype or torch.float32, device=DEV)
    if mode == "decode":
        args = la.make_args(k_base, v_base, lr, B_k, B_v, q, out, lora_scale=shape.lora_scale,
                            rope_base=shape.rope_base, kv_len=kv_len,
                            max_kv_len=int(kv_len.max().item()))
        ws = la.decode_workspace(args, DEV)
        la.lora_attn_decode(args, ws)
    else:
        args = la.make_args(k_base, v_base, lr, B_k, B_v, q, out, lora_scale=shape.lora_scale,
                            rope_base=shape.rope_base, q_pos0=shape.q_pos0)
        la.lora_attn_prefill(args)
    torch.cuda.synchronize()
    assert la.la_device_check() == 0
    return out


def test_tiny_fp32_decode_step_from_hidden(la):
    """Full step: GPU appends LR = X A, then decodes; oracle works from X in fp64."""
    s = W.TINY_FP32
    w, k_base, v_base = _tiny_caches(s)
    lr = torch.zeros((1, s.kv_len, 2 * s.r), device=DEV)
    la.lr_cache_append(w["X"].to(DEV), w["A_kv"].to(DEV), lr, 0)
    kv_len = torch.tensor([s.kv_len], dtype=torch.int32, device=DEV)
    got = _run(la, s, k_base.to(DEV), v_base.to(DEV), lr, w["B_k"].to(DEV), w["B_v"].to(DEV),
               w["q"].to(DEV), kv_len)
    kb, vb = oracle.base_cache_from_hidden(w["X"], w["W_k"], w["W_v"], s.n_kv_heads, s.rope_base)
    ref = oracle.lora_attention(kb, vb, oracle.lr_cache_rows(w["X"], w["A_kv"]), w["B_k"],
                                w["B_v"], w["q"], [s.kv_len], lora_scale=s.lora_scale,
                                softmax_scale=s.softmax_scale, rope_base=s.rope_base,
                                mode="decode")
    assert_parity(to_np(got), ref, torch.float32)


@pytest.mark.parametrize("kv_len", [1, 2, 31, 33, 200, 256])
def test_tiny_fp32_decode_lengths(la, kv_len):
    s = W.TINY_FP32
    w, k_base, v_base = _tiny_caches(s)
    lr = torch.from_numpy(oracle.lr_cache_rows(w["X"], w["A_kv"])).float()
    kvl = torch.tensor([kv_len], dtype=torch.int32)
    got = _run(la, s, k_base.to(DEV), v_base.to(DEV), lr.to(DEV), w["B_k"].to(DEV),
               w["B_v"].to(DEV), w["q"].to(DEV), kvl.to(DEV))
    ref = oracle.lora_attention(k_base, v_base, lr, w["B_k"], w["B_v"], w["q"], kvl,
                                lora_scale=s.lora_scale, softmax_scale=s.softmax_scale,
                                rope_base=s.rope_base, mode="decode")
    assert_parity(to_np(got), ref, torch.float32)


@pytest.mark.parametrize("n_tok", [1, 40, 77])
def test_tiny_fp32_prefill(la, n_tok):
    s = W.TINY_FP32.replace(n_q_tokens=n_tok, mode="prefill")
    w, k_base, v_base = _tiny_caches(s)
    lr = torch.from_numpy(oracle.lr_cache_rows(w["X"], w["A_kv"])).float()
    got = _run(la, s, k_base.to(DEV), v_base.to(DEV), lr.to(DEV), w["B_k"].to(DEV),
               w["B_v"].to(DEV), w["q"].to(DEV))
    ref = oracle.lora_attention(k_base, v_base, lr, w["B_k"], w["B_v"], w["q"], [s.kv_len],
                                lora_scale=s.lora_scale, softmax_scale=s.softmax_scale,
                                rope_base=s.rope_base, mode="prefill")
    assert_parity(to_np(got), ref, torch.float32)


# ----------------------------------------------------------- bf16 decode ----
def test_llama8b_decode_8k_full(la):
    """The 8192-token, 3-agent, r=16 decode: every output against the oracle."""
    s = W.LLAMA8B_DECODE_8K
    inp = W.direct_cache_inputs(s)
    d = to_device(inp)
    got = _run(la, s, d["k_base"], d["v_base"], d["lr"], d["B_k"], d["B_v"], d["q"], d["kv_len"])
    ref = oracle_decode(inp, s)
    assert_parity(to_np(got), ref, s.dtype)
    # the LoRA terms matter at this scale: dropping them would fail the bar
    no_lora = oracle.lora_attention(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"] * 0,
                                    inp["B_v"] * 0, inp["q"], inp["kv_len"],
                                    lora_scale=s.lora_scale, softmax_scale=s.softmax_scale,
                                    rope_base=s.rope_base, mode="decode")
    assert errors(no_lora, ref)[0] > 20 * 1e-2


@pytest.mark.parametrize("r,n_agents,d,lens", [
    (16, 3, 128, [1, 37, 1000]),
    (32, 5, 128, [64, 65, 129]),
    (64, 2, 128, [513, 2, 300]),
    (8, 4, 128, [100, 7, 1024]),
    (16, 3, 64, [1024, 500, 33]),
])
def test_bf16_decode_ragged(la, r, n_agents, d, lens):
    s = W.LLAMA8B_DECODE_8K.replace(n_seqs=len(lens), n_agents=n_agents, head_dim=d, r=r,
                                    alpha=2.0 * r, kv_len=max(lens), seed=11 + r)
    inp = W.direct_cache_inputs(s, L_max=max(lens) + 16)
    inp["kv_len"] = torch.tensor(lens, dtype=torch.int32)
    dd = to_device(inp)
    got = _run(la, s, dd["k_base"], dd["v_base"], dd["lr"], dd["B_k"], dd["B_v"], dd["q"],
               dd["kv_len"])
    assert_parity(to_np(got), oracle_decode(inp, s), s.dtype)


@pytest.mark.parametrize("r,n_agents,n_q,L,n_seqs,out_bf16", [
    (16, 5, 32, 3000, 1, False),   # groups of 3 + 2 agents, keys split over CTAs
    (64, 4, 32, 2000, 1, True),    # r = 64: one agent per CTA, four groups
    (32, 7, 16, 1500, 2, False),   # g = 2: groups of 3 + 3 + 1, two sequences
])
def test_bf16_decode_agent_groups(la, r, n_agents, n_q, L, n_seqs, out_bf16):
    """More agents than one CTA holds: the agents are split into groups that run
    side by side, each with its own split merge."""
    s = W.LLAMA8B_DECODE_8K.replace(n_seqs=n_seqs, n_agents=n_agents, n_q_heads=n_q, r=r,
                                    alpha=2.0 * r, kv_len=L, seed=90 + n_agents)
    inp = W.direct_cache_inputs(s)
    dd = to_device(inp)
    got = _run(la, s, dd["k_base"], dd["v_base"], dd["lr"], dd["B_k"], dd["B_v"], dd["q"],
               dd["kv_len"], out_dtype=torch.bfloat16 if out_bf16 else None)
    assert_parity(to_np(got.float()), oracle_decode(inp, s), s.dtype)


def test_bf16_decode_token_major_layout(la):
    """Base cache stored [seq][token][head][d]: same result as head-major."""
    s = W.LLAMA8B_DECODE_8K.replace(kv_len=777, n_seqs=2, seed=21)
    inp = W.direct_cache_inputs(s)
    dd = to_device(inp)
    kt = dd["k_base"].permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
    vt = dd["v_base"].permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
    a = _run(la, s, dd["k_base"], dd["v_base"], dd["lr"], dd["B_k"], dd["B_v"], dd["q"],
             dd["kv_len"])
    b = _run(la, s, kt, vt, dd["lr"], dd["B_k"], dd["B_v"], dd["q"], dd["kv_len"])
    assert torch.equal(a, b)
    assert_parity(to_np(b), oracle_decode(inp, s), s.dtype)


def test_decode_workspace_reuse_is_deterministic(la):
    s = W.LLAMA8B_DECODE_8K.replace(kv_len=3000, seed=22)
    dd = to_device(W.direct_cache_inputs(s))
    out1 = torch.empty(dd["q"].shape, device=DEV)
    out2 = torch.empty_like(out1)
    a1 = la.make_args(dd["k_base"], dd["v_base"], dd["lr"], dd["B_k"], dd["B_v"], dd["q"], out1,
                      lora_scale=s.lora_scale, rope_base=s.rope_base, kv_len=dd["kv_len"],
                      max_kv_len=s.kv_len)
    a2 = la.make_args(dd["k_base"], dd["v_base"], dd["lr"], dd["B_k"], dd["B_v"], dd["q"], out2,
                      lora_scale=s.lora_scale, rope_base=s.rope_base, kv_len=dd["kv_len"],
                      max_kv_len=s.kv_len)
    ws = la.decode_workspace(a1, DEV)
    la.lora_attn_decode(a1, ws)
    la.lora_attn_decode(a2, ws)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2)


def test_decode_kv_len_beyond_bound_is_reported(la):
    """kv_len above max_kv_len: the kernel's own check skips that sequence and
    raises the device error word; the other sequence is still computed."""
    s = W.LLAMA8B_DECODE_8K.replace(kv_len=500, n_seqs=2, seed=23)
    inp = W.direct_cache_inputs(s, L_max=600)
    dd = to_device(inp)
    dd["kv_len"] = torch.tensor([500, 550], dtype=torch.int32, device=DEV)
    out = torch.full(dd["q"].shape, 7.0, device=DEV)
    args = la.make_args(dd["k_base"], dd["v_base"], dd["lr"], dd["B_k"], dd["B_v"], dd["q"], out,
                        lora_scale=s.lora_scale, rope_base=s.rope_base, kv_len=dd["kv_len"],
                        max_kv_len=500)
    la.lora_attn_decode(args, la.decode_workspace(args, DEV))
    assert la.la_device_check() == la.LA_ERR_DEVICE_CHECK
    assert la.la_device_check() == 0
    assert (out[1] == 7.0).all()
    ref = oracle_decode(dict(inp, kv_len=torch.tensor([500, 500])), s)
    assert_parity(to_np(out[0]), ref[0], s.dtype)


def test_decode_merge_wait_runs_out_and_is_reported(la):
    """The in-launch split merge of the r = 64 decode waits, bounded, for every
    split of its unit to arrive on the unit's counter in the workspace.  A
    workspace whose counters start at -1 (all bytes 0xFF, never zero-filled)
    never reaches the split count: every CTA's wait gives up, the launch still
    ends, the merge bit of the device error word is set, and the same context
    then computes a correct decode on a zeroed workspace."""
    # r = 64: the decode whose split merge counts arrivals in the workspace
    s = W.llama8b_stack_decode(0).replace(kv_len=4096, seed=29)
    inp = W.direct_cache_inputs(s)
    dd = to_device(inp)
    out = torch.zeros(dd["q"].shape, device=DEV)
    args = la.make_args(dd["k_base"], dd["v_base"], dd["lr"], dd["B_k"], dd["B_v"], dd["q"], out,
                        lora_scale=s.lora_scale, rope_base=s.rope_base, kv_len=dd["kv_len"],
                        max_kv_len=s.kv_len)
    ws = la.decode_workspace(args, DEV)
    assert la.la_device_check() == 0
    ws.fill_(0xFF)
    la.lora_attn_decode(args, ws)
    st, word = la.la_device_check_word()
    assert st == la.LA_ERR_DEVICE_CHECK
    assert word == la.LA_DEV_MERGE_WAIT
    assert la.la_device_check_word() == (0, 0)
    ws.zero_()
    la.lora_attn_decode(args, ws)
    assert la.la_device_check_word() == (0, 0)
    assert_parity(to_np(out), oracle_decode(inp, s), s.dtype)


@pytest.mark.parametrize("kv_lens,per_agent,packed", [
    ((8192,), False, False),          # the LLaMA-8B decode step: one sequence, shared A
    ((8192,), False, True),           # the same with x, q, kv_len back to back: one copy
    ((700, 650, 700), False, True),   # unequal lengths: one append per sequence
    ((640, 640), True, False),        # BaseShared: every agent's own A_a and LR cache
])
def test_decode_step_from_host_equals_device_step(la, kv_lens, per_agent, packed):
    """lora_decode_step_host (copies in, the step, copy out) gives the same LR
    rows and outputs, bit for bit, as lora_attn_decode_step on device buffers.
    The new rows are X A within one bf16 ulp of the oracle's fp64 rows (fp32
    accumulation order), every other row is untouched, and the outputs match
    the oracle over the updated caches."""
    n_seqs, L_max = len(kv_lens), max(kv_lens)
    s = W.LLAMA8B_DECODE_8K.replace(kv_len=L_max, n_seqs=n_seqs, seed=37, lr_per_agent=per_agent)
    inp = W.direct_cache_inputs(s, L_max=L_max)
    inp["kv_len"] = torch.tensor(kv_lens, dtype=torch.int32)
    x = W.append_inputs(1, s.hidden, s.r, s.dtype, seed=41, n_seqs=n_seqs)["X"]
    if per_agent:
        A_kv = torch.stack([W.append_inputs(1, s.hidden, s.r, s.dtype, seed=43 + a)["A_kv"]
                            for a in range(s.n_agents)])
    else:
        A_kv = W.append_inputs(1, s.hidden, s.r, s.dtype, seed=43)["A_kv"]
    outs, lrs = [], []
    for from_host in (False, True):
        dd = to_device(inp)
        out = torch.zeros(dd["q"].shape, device=DEV)
        x_dev, A_dev = x.to(DEV), A_kv.to(DEV)
        h_x, h_q, h_len = x.pin_memory(), inp["q"].pin_memory(), inp["kv_len"].pin_memory()
        if from_host and packed:
            _, x_dev, dd["q"], dd["kv_len"] = la.packed_step_inputs(
                x.shape, inp["q"].shape, n_seqs, s.dtype, DEV)
            _, h_x, h_q, h_len = la.packed_step_inputs(x.shape, inp["q"].shape, n_seqs, s.dtype,
                                                       "cpu", pin=True)
            h_x.copy_(x)
            h_q.copy_(inp["q"])
            h_len.copy_(inp["kv_len"])
        step = la.DecodeStep(dd["k_base"], dd["v_base"], dd["lr"], dd["B_k"], dd["B_v"], dd["q"],
                             out, dd["kv_len"], lora_scale=s.lora_scale, rope_base=s.rope_base,
                             max_kv_len=L_max, A_kv=A_dev, x_new=x_dev)
        if from_host:
            x_dev.zero_()
            dd["q"].zero_()
            dd["kv_len"].zero_()
            out_host = torch.full(out.shape, 7.0).pin_memory()
            step.from_host(h_x, h_q, h_len, out_host)
            torch.cuda.synchronize()
            outs.append(out_host.clone())
        else:
            step()
            torch.cuda.synchronize()
            outs.append(out.cpu())
        lrs.append(dd["lr"].cpu())
    assert la.la_device_check() == 0
    assert torch.equal(lrs[0], lrs[1])
    assert torch.equal(outs[0], outs[1])
    # the new rows, and nothing else, changed
    got = lrs[1] if per_agent else lrs[1][None]
    before = inp["lr"] if per_agent else inp["lr"][None]
    A_list = [A_kv[a] for a in range(s.n_agents)] if per_agent else [A_kv]
    for l, A in enumerate(A_list):
        ref = oracle.lr_cache_rows(x, A)[:, 0]                      # [n_seqs, 2r]
        for q, n in enumerate(kv_lens):
            row = to_np(got[l, q, n - 1])
            bound = np.maximum(bf16_ulp(ref[q]), 1e-6 * (np.abs(to_np(x[q, 0])) @ np.abs(to_np(A))))
            assert (np.abs(row - ref[q]) <= bound).all(), np.abs(row - ref[q]).max()
            keep = torch.ones(got.shape[2], dtype=torch.bool)
            keep[n - 1] = False
            assert torch.equal(got[l, q, keep], before[l, q, keep])
    assert_parity(to_np(outs[1]), oracle_decode(inp, s, lr=lrs[1].double()), s.dtype)


@pytest.mark.parametrize("r,n_agents,per_agent", [(16, 3, False), (32, 5, False), (16, 3, True),
                                                  (64, 4, False)])
def test_decode_step_equals_append_then_decode(la, r, n_agents, per_agent):
    """The step (a row-append kernel at the device's kv_len, then the decode)
    against lr_cache_append at host positions followed by lora_attn_decode:
    the rows agree within one bf16 ulp (different summation orders), the
    outputs within the parity bar."""
    kv_lens = (1000, 777)
    s = W.LLAMA8B_DECODE_8K.replace(kv_len=1000, n_seqs=2, r=r, alpha=2.0 * r, n_agents=n_agents,
                                    seed=48 + r, lr_per_agent=per_agent)
    inp = W.direct_cache_inputs(s)
    inp["kv_len"] = torch.tensor(kv_lens, dtype=torch.int32)
    x = W.append_inputs(1, s.hidden, r, s.dtype, seed=49, n_seqs=2)["X"]
    A_kv = (torch.stack([W.append_inputs(1, s.hidden, r, s.dtype, seed=50 + a)["A_kv"]
                         for a in range(n_agents)]) if per_agent
            else W.append_inputs(1, s.hidden, r, s.dtype, seed=50)["A_kv"])
    res = []
    for fused in (True, False):
        dd = to_device(inp)
        out = torch.zeros(dd["q"].shape, device=DEV)
        x_dev, A_dev = x.to(DEV), A_kv.to(DEV)
        step = la.DecodeStep(dd["k_base"], dd["v_base"], dd["lr"], dd["B_k"], dd["B_v"], dd["q"],
                             out, dd["kv_len"], lora_scale=s.lora_scale, rope_base=s.rope_base,
                             max_kv_len=1000, A_kv=A_dev, x_new=x_dev)
        if fused:
            step()
        else:
            for q, n in enumerate(kv_lens):
                if per_agent:
                    la.lr_cache_append_agents(x_dev[q:q + 1], A_dev, dd["lr"][:, q:q + 1], n - 1)
                else:
                    la.lr_cache_append(x_dev[q:q + 1], A_dev, dd["lr"][q:q + 1], n - 1)
            la.lora_attn_decode(step.args, step.workspace)
        torch.cuda.synchronize()
        assert la.la_device_check() == 0
        res.append((to_np(out), to_np(dd["lr"])))
    (o1, l1), (o2, l2) = res
    assert (np.abs(l1 - l2) <= 2 * bf16_ulp(l2)).all()
    assert_parity(o1, o2, s.dtype)
    assert_parity(o1, oracle_decode(inp, s, lr=torch.from_numpy(l1)), s.dtype)


# ---------------------------------------------------------- bf16 prefill ----
@pytest.mark.parametrize("L,n_tok,r,n_agents", [
    (300, 77, 16, 3),
    (129, 129, 32, 2),
    (1000, 256, 64, 4),
    (65, 1, 8, 1),
])
def test_bf16_prefill_small(la, L, n_tok, r, n_agents):
    s = W.LLAMA8B_PREFILL_16K.replace(kv_len=L, n_q_tokens=n_tok, r=r, alpha=2.0 * r,
                                      n_agents=n_agents, seed=31 + L)
    inp = W.direct_cache_inputs(s)
    dd = to_device(inp)
    got = _run(la, s, dd["k_base"], dd["v_base"], dd["lr"], dd["B_k"], dd["B_v"], dd["q"])
    ref = oracle.lora_attention(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"],
                                inp["q"], inp["kv_len"], lora_scale=s.lora_scale,
                                softmax_scale=s.softmax_scale, rope_base=s.rope_base,
                                mode="prefill")
    assert_parity(to_np(got), ref, s.dtype)


def _prefill_vs_oracle(la, s, inp, out_dtype=None):
    dd = to_device(inp)
    got = _run(la, s, dd["k_base"], dd["v_base"], dd["lr"], dd["B_k"], dd["B_v"], dd["q"],
               out_dtype=out_dtype)
    ref = oracle.lora_attention(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"],
                                inp["q"], inp["kv_len"], lora_scale=s.lora_scale,
                                softmax_scale=s.softmax_scale, rope_base=s.rope_base,
                                mode="prefill")
    return assert_parity(to_np(got.float()), ref, s.dtype)


@pytest.mark.parametrize("n_q,n_kv,L,n_tok,n_seqs,r", [
    (32, 8, 200, 200, 1, 16),     # g = 4, self-attention of a fresh chunk (q_pos0 = 0), ragged block
    (32, 8, 600, 300, 1, 32),     # r = 32
    (32, 8, 700, 200, 1, 64),     # r = 64: one V stage
    (32, 4, 700, 45, 2, 16),      # g = 8: 16 tokens per block, two sequences
    (8, 8, 390, 260, 1, 16),      # g = 1: 128 tokens per block, chunk over a prefix
    (16, 8, 129, 64, 1, 16),      # g = 2, one key past a tile
    (32, 8, 100, 1, 1, 16),       # one query token, one partial tile
    (4, 1, 512, 512, 1, 16),      # few CTAs: key halves on CTA pairs; blocks of one tile leave half 1 empty
    (32, 8, 600, 224, 1, 16),     # 168 CTAs: 6 blocks whole, the last one as key halves (two launches)
])
def test_bf16_prefill_tensor_core_shapes(la, n_q, n_kv, L, n_tok, n_seqs, r):
    """The tcgen05 prefill (r = 16, 32, 64): GQA groups 1..8, blocks cut by the
    chunk's end, keys cut inside a tile, several sequences."""
    s = W.LLAMA8B_PREFILL_16K.replace(n_q_heads=n_q, n_kv_heads=n_kv, kv_len=L, n_q_tokens=n_tok,
                                      n_seqs=n_seqs, r=r, alpha=2.0 * r, seed=400 + L)
    _prefill_vs_oracle(la, s, W.direct_cache_inputs(s))


def test_bf16_prefill_bf16_output(la):
    s = W.LLAMA8B_PREFILL_16K.replace(kv_len=333, n_q_tokens=96, seed=77)
    _prefill_vs_oracle(la, s, W.direct_cache_inputs(s), out_dtype=torch.bfloat16)


def _ramped_keys(s, inp, lo, hi):
    ramp = torch.linspace(lo, hi, s.kv_len).view(1, 1, -1, 1)
    inp["k_base"] = (inp["k_base"].float() * ramp).to(torch.bfloat16)
    return inp


def test_bf16_prefill_growing_scores(la):
    """Keys whose scale grows tenfold along the sequence move every row's
    maximum up by many units of log2: the lazy rescale of O and l engages
    repeatedly.  Exact oracle."""
    s = W.LLAMA8B_PREFILL_16K.replace(kv_len=1200, n_q_tokens=128, seed=78)
    _prefill_vs_oracle(la, s, _ramped_keys(s, W.direct_cache_inputs(s), 0.25, 2.5))


def test_bf16_prefill_growing_scores_thirtyfold(la):
    """A thirtyfold ramp (keys up to six times the configs' scale): the
    maximum of every row keeps moving, and the key operand of the score MMA,
    K^a = K_base + RoPE(s LRk B_k^a) rounded once (to fp16), must stay close
    enough at |K| six times larger.  Exact oracle."""
    s = W.LLAMA8B_PREFILL_16K.replace(kv_len=1200, n_q_tokens=128, seed=79)
    _prefill_vs_oracle(la, s, _ramped_keys(s, W.direct_cache_inputs(s), 0.2, 6.0))


def _sampled_units(la, s, inp, got, units, tokens):
    """Compare sampled (seq, agent, kv head) x query tokens against the oracle."""
    g = s.group
    refs, gots = [], []
    for (seq, agent, kvh) in units:
        kvl = int(inp["kv_len"][seq])
        qpos = oracle.query_positions(kvl, s.n_q_tokens, s.mode, s.q_pos0 if s.mode == "prefill"
                                      else None)
        ref = oracle.lora_attention_unit(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"],
                                         inp["B_v"], inp["q"], seq=seq, agent=agent, kv_head=kvh,
                                         kv_len=kvl, q_positions=qpos, lora_scale=s.lora_scale,
                                         softmax_scale=s.softmax_scale, rope_base=s.rope_base,
                                         q_tokens=tokens)
        refs.append(ref)
        gots.append(to_np(got[seq, agent][tokens][:, kvh * g:(kvh + 1) * g]))
    return assert_parity(np.stack(gots), np.stack(refs), s.dtype)


def test_llama8b_prefill_16k_sampled(la):
    s = W.LLAMA8B_PREFILL_16K
    inp = W.direct_cache_inputs(s)
    dd = to_device(inp)
    got = _run(la, s, dd["k_base"], dd["v_base"], dd["lr"], dd["B_k"], dd["B_v"], dd["q"]).cpu()
    tokens = np.array([0, 1, 63, 64, 127, 500, 1000, 1022, 1023])
    _sampled_units(la, s, inp, got, [(0, 0, 0), (0, 1, 3), (0, 2, 7)], tokens)


@pytest.mark.parametrize("layer", [0, 15, 31])
def test_llama8b_stack_prefill_sampled(la, layer):
    """Layers 0, 15 and 31 of the 32-layer stack (each its own seeded inputs):
    a 4096-token chunk over a 32768-token prefix, 4 agents, r = 64 (the
    tensor-core prefill with one V stage).  Every agent and KV head is
    sampled across the layers, at tokens on tile and block edges and the last."""
    s = W.llama8b_stack_prefill(layer)
    inp = W.direct_cache_inputs(s, device=DEV)
    got = _run(la, s, inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"],
               inp["q"]).cpu()
    tokens = np.array([0, 1, 31, 32, 127, 128, 1000, 2047, 2048, 3071, 4094, 4095])
    units = [((0, (layer + k) % s.n_agents, (3 * layer + 5 * k) % s.n_kv_heads)) for k in range(4)]
    _sampled_units(la, s, inp, got, units, tokens)


@pytest.mark.parametrize("layer", [0, 15, 31])
def test_llama8b_stack_decode_full(la, layer):
    """The stack's decode over the 36864 cached keys (prefix + chunk), 4 agents,
    r = 64, layers 0, 15 and 31: every output against the oracle."""
    s = W.llama8b_stack_decode(layer)
    inp = W.direct_cache_inputs(s, device=DEV)
    got = _run(la, s, inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"], inp["q"],
               inp["kv_len"])
    assert_parity(to_np(got), oracle_decode(inp, s), s.dtype)


@pytest.mark.parametrize("layer", [0, 15, 31])
def test_llama8b_stack_layer_append_and_decode_steps(la, layer):
    """Layers 0, 15 and 31 of the 32-layer stack as the bench runs them: the
    chunk's LR rows appended (X A), then every one of the decode steps appends
    its token's row and attends over prefix + chunk + the steps so far.  The
    oracle forms the LR rows from X and A itself (fp64); two (agent, KV head)
    units are checked at every step, every agent and head over the steps."""
    import bench
    L = bench.StackLayer(layer, DEV)
    s = L.shape
    L.append()
    outs = []
    for t in range(bench.STACK_STEPS):
        L.decode_step(t)
        outs.append(L.dec_out[t].clone())
    torch.cuda.synchronize()
    assert la.la_device_check() == 0
    lr = oracle.lr_cache_append(L.inp["lr"][:, :s.kv_len].cpu(), L.chunk["X"].cpu(),
                                L.chunk["A_kv"].cpu(), L.n_pre)
    steps = oracle.lr_cache_rows(L.xs.cpu(), L.chunk["A_kv"].cpu())      # [1, steps, 2r]
    lr = np.concatenate([lr, steps], axis=1)
    kb, vb = L.inp["k_base"].cpu(), L.inp["v_base"].cpu()
    g = s.group
    gots, refs = [], []
    for t in range(bench.STACK_STEPS):
        kvl = s.kv_len + t + 1
        q = L.q_dec[t].cpu()
        for u in range(2):
            agent = (t + 2 * u + layer) % s.n_agents
            kvh = (3 * t + 5 * u + layer) % s.n_kv_heads
            refs.append(oracle.lora_attention_unit(kb, vb, lr, L.inp["B_k"].cpu(), L.inp["B_v"].cpu(),
                                                   q, seq=0, agent=agent, kv_head=kvh, kv_len=kvl,
                                                   q_positions=[kvl - 1], lora_scale=s.lora_scale,
                                                   softmax_scale=s.softmax_scale,
                                                   rope_base=s.rope_base))
            gots.append(to_np(outs[t][0, agent][:, kvh * g:(kvh + 1) * g]))
    assert_parity(np.stack(gots), np.stack(refs), s.dtype)


@pytest.mark.parametrize("ctx", W.SWEEP_CTX)
def test_llama8b_sweep_decode_sampled(la, ctx):
    """The batched long-context decode (16 requests x 5 agents, r = 32) at
    32768, 65536 and 131072 keys; inputs drawn on the device, sampled
    (sequence, agent, KV head) units copied to the host for the oracle."""
    s = W.llama8b_sweep(ctx)
    inp = W.direct_cache_inputs(s, device=DEV)
    got = _run(la, s, inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"], inp["q"],
               inp["kv_len"]).cpu()
    _sampled_units(la, s, inp, got, [(0, 0, 0), (5, 4, 7), (15, 2, 3), (9, 3, 1)], np.array([0]))
    del inp
    torch.cuda.empty_cache()


@pytest.mark.parametrize("ctx,n_agents,r", [(131072, 5, 32), (36864, 4, 64)])
def test_decode_dominated_by_the_last_keys(la, ctx, n_agents, r):
    """The largest positions decide the output: the LR rows of the last 200
    keys are scaled fourfold, so their rotated key deltas lead the scores and
    their values the output.  A rotation off by one position at the tail then
    moves the outputs by about 5e-2 of their maximum (1e-2 rad of drift by
    about 5e-3), where with unscaled rows it would be averaged away over the
    131072 keys (3e-3)."""
    s = W.llama8b_sweep(ctx).replace(n_seqs=1, n_agents=n_agents, r=r, alpha=2.0 * r,
                                     seed=ctx + r)
    inp = W.direct_cache_inputs(s, device=DEV)
    inp["lr"][:, ctx - 200:] *= 4
    got = _run(la, s, inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"], inp["q"],
               inp["kv_len"])
    assert_parity(to_np(got), oracle_decode(inp, s), s.dtype)


# ------------------------------------------------------ non-shared baseline ----
def test_materialized_agent_caches_and_non_shared_decode(la):
    """The non-shared baseline: every agent's K^a, V^a written out equal the
    oracle's materialised caches (one bf16 rounding), and plain attention over
    them gives the shared path's outputs."""
    import bench
    s = W.LLAMA8B_DECODE_8K.replace(kv_len=700, n_seqs=2, seed=55)
    inp = W.direct_cache_inputs(s)
    dd = to_device(inp)
    mat, dec, out_ns = bench.non_shared_setup(la, s, dd, DEV)
    mat()
    kout, vout = mat.keep[0].cpu(), mat.keep[1].cpu()
    d, r = s.head_dim, s.r
    kpos = np.arange(s.kv_len)
    for seq in range(s.n_seqs):
        lr = to_np(inp["lr"][seq])
        for a in range(s.n_agents):
            for j in (0, s.n_kv_heads - 1):
                cols = slice(j * d, (j + 1) * d)
                Ka = oracle.agent_keys(inp["k_base"][seq, j], lr[:, :r], to_np(inp["B_k"][a])[:, cols],
                                       s.lora_scale, kpos, s.rope_base)
                Va = oracle.agent_values(inp["v_base"][seq, j], lr[:, r:], to_np(inp["B_v"][a])[:, cols],
                                         s.lora_scale)
                for got, ref in ((kout[seq, a, j, :s.kv_len], Ka), (vout[seq, a, j, :s.kv_len], Va)):
                    err = np.abs(to_np(got) - ref)
                    assert (err <= bf16_ulp(ref) + 1e-3 * np.abs(ref).max()).all(), err.max()
    dec()
    torch.cuda.synchronize()
    assert la.la_device_check() == 0
    shared = _run(la, s, dd["k_base"], dd["v_base"], dd["lr"], dd["B_k"], dd["B_v"], dd["q"],
                  dd["kv_len"])
    assert_parity(to_np(out_ns), oracle_decode(inp, s), s.dtype)
    assert_parity(to_np(out_ns), to_np(shared), s.dtype)


# ------------------------------ one LR cache per agent (BaseShared) ----
# Each agent owns its down-projection A_a and reads its own LR cache X A_a
# beside the shared base cache (LRAgent summary §3 "BaseShared"); the LR
# tensor is [n_agents, n_seqs, L_max, 2r] and la_attn_args.lr_agent_stride
# points each agent at its own.
@pytest.mark.parametrize("n_q,n_kv,L,n_tok,n_seqs,r,n_agents", [
    (32, 8, 600, 300, 1, 16, 3),     # tensor-core prefill, r = 16
    (32, 8, 700, 200, 1, 64, 4),     # r = 64: one V stage
    (8, 8, 390, 260, 2, 32, 2),      # g = 1, two sequences
    (4, 1, 512, 512, 1, 16, 3),      # few CTAs: key halves on CTA pairs
])
def test_base_shared_prefill_tensor_cores(la, n_q, n_kv, L, n_tok, n_seqs, r, n_agents):
    s = W.LLAMA8B_PREFILL_16K.replace(n_q_heads=n_q, n_kv_heads=n_kv, kv_len=L, n_q_tokens=n_tok,
                                      n_seqs=n_seqs, r=r, alpha=2.0 * r, n_agents=n_agents,
                                      seed=600 + L, lr_per_agent=True)
    _prefill_vs_oracle(la, s, W.direct_cache_inputs(s))


@pytest.mark.parametrize("kv_len,n_seqs,n_agents,r,n_kv", [
    (1500, 1, 3, 16, 8),     # the 3-agent layer: 3 agents a CTA, each with its own LR tiles
    (900, 1, 5, 16, 8),      # groups of 3 + 2 agents
    (650, 2, 3, 16, 4),      # g = 8: 24 rows, three row tiles
    (700, 2, 5, 32, 8),      # the batched sweep's agents and rank, short: one agent a CTA
    (300, 1, 4, 64, 8),      # the stack's rank
])
def test_base_shared_decode_tensor_cores(la, kv_len, n_seqs, n_agents, r, n_kv):
    s = W.LLAMA8B_DECODE_8K.replace(kv_len=kv_len, n_seqs=n_seqs, n_agents=n_agents, r=r,
                                    alpha=2.0 * r, seed=700 + kv_len, lr_per_agent=True,
                                    n_kv_heads=n_kv)
    inp = W.direct_cache_inputs(s)
    dd = to_device(inp)
    got = _run(la, s, dd["k_base"], dd["v_base"], dd["lr"], dd["B_k"], dd["B_v"], dd["q"],
               dd["kv_len"])
    assert_parity(to_np(got), oracle_decode(inp, s), s.dtype)


@pytest.mark.parametrize("mode,n_tok", [("decode", 1), ("prefill", 37)])
def test_base_shared_fp32_generic_kernel(la, mode, n_tok):
    s = W.TINY_FP32.replace(kv_len=200, n_q_tokens=n_tok, mode=mode, n_agents=3, seed=71,
                            lr_per_agent=True)
    inp = W.direct_cache_inputs(s)
    dd = to_device(inp)
    got = _run(la, s, dd["k_base"], dd["v_base"], dd["lr"], dd["B_k"], dd["B_v"], dd["q"],
               dd["kv_len"])
    ref = oracle.lora_attention(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"],
                                inp["q"], inp["kv_len"], lora_scale=s.lora_scale,
                                softmax_scale=s.softmax_scale, rope_base=s.rope_base, mode=mode)
    assert_parity(to_np(got), ref, s.dtype)


@pytest.mark.parametrize("dtype,r", [(torch.bfloat16, 16), (torch.bfloat16, 64), (torch.float32, 8)])
def test_append_agents_equals_one_append_per_agent(la, dtype, r):
    """Every agent's cache X A_a: bit-identical to one single-A append per agent,
    rows outside the chunk untouched, and within one rounding of the oracle."""
    n_agents, n_seqs, n, H, L_max, pos0 = 3, 2, 45, 512, 64, 7
    g = torch.Generator().manual_seed(90 + r)
    X = torch.randn(n_seqs, n, H, generator=g).to(dtype)
    A = (0.05 * torch.randn(n_agents, H, 2 * r, generator=g)).to(dtype)
    guard = torch.full((n_agents, n_seqs, L_max, 2 * r), 7.0, dtype=dtype)
    lr = guard.to(DEV)
    la.lr_cache_append_agents(X.to(DEV), A.to(DEV), lr, pos0)
    one = guard.to(DEV)
    for a in range(n_agents):
        la.lr_cache_append(X.to(DEV), A[a].to(DEV), one[a], pos0)
    torch.cuda.synchronize()
    assert torch.equal(lr.cpu(), one.cpu())
    got = lr.cpu()
    assert torch.equal(got[:, :, :pos0], guard[:, :, :pos0])
    assert torch.equal(got[:, :, pos0 + n:], guard[:, :, pos0 + n:])
    ref = oracle.lr_cache_append_agents(guard.to(torch.float64).numpy(), X, A, pos0)
    err = np.abs(to_np(got) - ref)
    tol = bf16_ulp(ref) if dtype == torch.bfloat16 else 1e-5 * (1 + np.abs(ref))
    assert (err <= tol).all(), err.max()


def test_base_shared_materialized_caches(la):
    """The non-shared baseline over per-agent LR caches: agent a's K^a, V^a are
    built from its own LR rows."""
    import bench
    s = W.LLAMA8B_DECODE_8K.replace(kv_len=400, n_seqs=1, seed=57, lr_per_agent=True)
    inp = W.direct_cache_inputs(s)
    dd = to_device(inp)
    mat, dec, out_ns = bench.non_shared_setup(la, s, dd, DEV)
    mat()
    torch.cuda.synchronize()
    kout, vout = mat.keep[0].cpu(), mat.keep[1].cpu()
    d, r = s.head_dim, s.r
    kpos = np.arange(s.kv_len)
    for a in range(s.n_agents):
        lr = to_np(inp["lr"][a, 0])
        j = a % s.n_kv_heads
        cols = slice(j * d, (j + 1) * d)
        Ka = oracle.agent_keys(inp["k_base"][0, j], lr[:, :r], to_np(inp["B_k"][a])[:, cols],
                               s.lora_scale, kpos, s.rope_base)
        Va = oracle.agent_values(inp["v_base"][0, j], lr[:, r:], to_np(inp["B_v"][a])[:, cols],
                                 s.lora_scale)
        for got, ref in ((kout[0, a, j, :s.kv_len], Ka), (vout[0, a, j, :s.kv_len], Va)):
            err = np.abs(to_np(got) - ref)
            assert (err <= bf16_ulp(ref) + 1e-3 * np.abs(ref).max()).all(), err.max()
    dec()
    torch.cuda.synchronize()
    assert la.la_device_check() == 0
    assert_parity(to_np(out_ns), oracle_decode(inp, s), s.dtype)


# --------------------------- query- and output-side LoRA (qkvo setting) ----
def _qo_inputs(n_seqs, n_agents, n_tok, n_q, d, r, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    q_base = (W.CACHE_STD * torch.randn(n_seqs, n_agents, n_tok, n_q, d, generator=g)).to(dtype)
    lr_q = (W.CACHE_STD * torch.randn(n_seqs, n_agents, n_tok, r, generator=g)).to(dtype)
    B_q = (0.02 * torch.randn(n_agents, r, n_q * d, generator=g)).to(dtype)
    return q_base, lr_q, B_q


@pytest.mark.parametrize("dtype,n_seqs,n_agents,n_tok,n_q,d,r,in_place", [
    (torch.bfloat16, 1, 3, 1, 32, 128, 16, False),    # one decode step of the 3-agent layer
    (torch.bfloat16, 2, 2, 37, 32, 128, 64, True),    # a ragged prefill chunk, in place
    (torch.float32, 2, 3, 5, 4, 64, 8, False),        # the tiny fp32 shape
    (torch.bfloat16, 1, 3, 1024, 32, 128, 16, False), # the 1024-token chunk of the 3-agent layer
    (torch.bfloat16, 1, 2, 20, 8, 64, 32, True),      # head_dim 64, r = 32, ragged, in place
    (torch.bfloat16, 2, 1, 17, 4, 128, 8, False),     # r = 8, fewer heads than threads
])
def test_query_expand_against_oracle(la, dtype, n_seqs, n_agents, n_tok, n_q, d, r, in_place):
    q_base, lr_q, B_q = _qo_inputs(n_seqs, n_agents, n_tok, n_q, d, r, dtype, 300 + r)
    pos_end = torch.tensor([5000 + 977 * i for i in range(n_seqs)], dtype=torch.int32)
    s, base = 2.0, 500000.0
    qb = q_base.to(DEV)
    out = qb if in_place else torch.empty_like(qb)
    la.lora_query_expand(qb, lr_q.to(DEV), B_q.to(DEV), out, pos_end.to(DEV), lora_scale=s,
                         rope_base=base)
    torch.cuda.synchronize()
    ref = np.empty(q_base.shape)
    for q in range(n_seqs):
        pos = int(pos_end[q]) - n_tok + np.arange(n_tok)
        for a in range(n_agents):
            ref[q, a] = oracle.lora_queries(q_base[q, a], lr_q[q, a], B_q[a], s, pos, base)
    assert_parity(to_np(out), ref, dtype)


@pytest.mark.parametrize("dtype,n_seqs,n_agents,n_tok,r,per_agent_A,zero_base", [
    (torch.bfloat16, 1, 3, 1, 16, False, False),     # a decode step, shared A_o
    (torch.bfloat16, 2, 2, 19, 64, True, False),     # ragged token blocks, per-agent A_o
    (torch.float32, 1, 2, 9, 8, False, False),
    # y = 0 on entry: the bf16 delta alone against the oracle (tensor-core shrink)
    (torch.bfloat16, 1, 3, 1024, 16, False, True),   # the 1024-token chunk of the 3-agent layer
    (torch.bfloat16, 2, 2, 19, 64, True, True),
    (torch.bfloat16, 1, 2, 33, 8, False, True),
    (torch.bfloat16, 1, 1, 16, 32, True, True),
])
def test_output_delta_against_oracle(la, dtype, n_seqs, n_agents, n_tok, r, per_agent_A, zero_base):
    d_in, d_out = 4096, 4096
    g = torch.Generator().manual_seed(400 + r)
    o = torch.randn(n_seqs, n_agents, n_tok, d_in, generator=g).to(dtype)
    A_shape = (n_agents, d_in, r) if per_agent_A else (d_in, r)
    A_o = (0.02 * torch.randn(*A_shape, generator=g)).to(dtype)
    B_o = (0.02 * torch.randn(n_agents, r, d_out, generator=g)).to(dtype)
    y0 = torch.randn(n_seqs, n_agents, n_tok, d_out, generator=g).to(dtype)
    if zero_base:
        y0.zero_()
    y = y0.to(DEV)
    s = 2.0
    la.lora_output_delta(o.to(DEV), A_o.to(DEV), B_o.to(DEV), y, lora_scale=s)
    torch.cuda.synchronize()
    ref = np.empty(y0.shape)
    for q in range(n_seqs):
        for a in range(n_agents):
            Aa = A_o[a] if per_agent_A else A_o
            ref[q, a] = oracle.lora_output(y0[q, a], o[q, a], Aa, B_o[a], s)
    assert_parity(to_np(y), ref, dtype)
    if dtype == torch.float32:   # the delta alone too (fp32 keeps it exact enough to isolate)
        assert_parity(to_np(y) - to_np(y0), ref - to_np(y0), dtype)


def test_query_expand_then_decode(la):
    """The decode step with a query-side LoRA: expanded queries feed the
    attention; the oracle rotates its own q^a and attends."""
    s = W.LLAMA8B_DECODE_8K.replace(kv_len=900, seed=61)
    inp = W.direct_cache_inputs(s)
    q_base, lr_q, B_q = _qo_inputs(s.n_seqs, s.n_agents, 1, s.n_q_heads, s.head_dim, s.r,
                                   s.dtype, 62)
    dd = to_device(inp)
    q = torch.empty_like(dd["q"])
    la.lora_query_expand(q_base.to(DEV), lr_q.to(DEV), B_q.to(DEV), q, dd["kv_len"],
                         lora_scale=s.lora_scale, rope_base=s.rope_base)
    got = _run(la, s, dd["k_base"], dd["v_base"], dd["lr"], dd["B_k"], dd["B_v"], q, dd["kv_len"])
    qa = np.stack([oracle.lora_queries(q_base[0, a], lr_q[0, a], B_q[a], s.lora_scale,
                                       [s.kv_len - 1], s.rope_base) for a in range(s.n_agents)])
    inp_q = dict(inp, q=torch.from_numpy(qa[None]).to(s.dtype))   # the kernel's queries are bf16
    assert_parity(to_np(got), oracle_decode(inp_q, s), s.dtype)


# -------------------- value side: reordered vs rebuilt per tile (ablation) ----
def _run_path(la, s, dd, value_path):
    out = torch.empty(dd["q"].shape, dtype=torch.float32, device=DEV)
    if s.mode == "decode":
        args = la.make_args(dd["k_base"], dd["v_base"], dd["lr"], dd["B_k"], dd["B_v"], dd["q"], out,
                            lora_scale=s.lora_scale, rope_base=s.rope_base, kv_len=dd["kv_len"],
                            max_kv_len=s.kv_len, value_path=value_path)
        la.lora_attn_decode(args, la.decode_workspace(args, DEV))
    else:
        args = la.make_args(dd["k_base"], dd["v_base"], dd["lr"], dd["B_k"], dd["B_v"], dd["q"], out,
                            lora_scale=s.lora_scale, rope_base=s.rope_base, q_pos0=s.q_pos0,
                            value_path=value_path)
        la.lora_attn_prefill(args)
    torch.cuda.synchronize()
    assert la.la_device_check() == 0
    return out


@pytest.mark.parametrize("shape", [
    W.LLAMA8B_DECODE_8K.replace(kv_len=700, seed=81),
    W.LLAMA8B_PREFILL_16K.replace(kv_len=300, n_q_tokens=45, seed=82),
    W.LLAMA8B_DECODE_8K.replace(kv_len=500, seed=83, lr_per_agent=True),
    W.TINY_FP32.replace(kv_len=150, seed=84),
    W.LLAMA8B_PREFILL_16K.replace(kv_len=2000, n_q_tokens=300, seed=85),
])
@pytest.mark.parametrize("value_path", [1, 2, 3])
def test_value_paths_match_the_oracle(la, shape, value_path):
    """The reordered value side on the generic kernel (1) and V^a rebuilt per
    tile (2: on the tensor-core prefill for the bf16 r = 16 prefills, several
    query blocks, key tiles and a ragged tail in the larger one; 3: on the
    generic kernel) all equal the oracle, which materialises V^a."""
    inp = W.direct_cache_inputs(shape)
    got = _run_path(la, shape, to_device(inp), value_path)
    ref = oracle.lora_attention(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"],
                                inp["q"], inp["kv_len"], lora_scale=shape.lora_scale,
                                softmax_scale=shape.softmax_scale, rope_base=shape.rope_base,
                                mode=shape.mode)
    assert_parity(to_np(got), ref, shape.dtype)
