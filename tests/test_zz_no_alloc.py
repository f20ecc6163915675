"""lora_attn_decode_static_scratch: decode for callers that cannot allocate.

A plugin inside a serving runtime whose allocator owns all device memory, or a
process that fixes its device memory at start-up, cannot hand the library a
workspace.  This entry point keeps the decode's split scratch in the library's
own device array instead.  These tests call it through the C ABI and check that
two calls in a row give what lora_attn_decode gives with a caller workspace.

The file sorts last so that a run stopping at its first failure has already run
every other test; it also passes on its own in a fresh process.
"""
import ctypes

import pytest
import torch

from rank_attention_b200 import workloads as W
from tests.helpers import assert_parity, oracle_decode, to_np

DEV = "cuda"
FAKE = 0x10000  # 16-byte aligned, never dereferenced


@pytest.fixture(scope="module")
def la():
    from rank_attention_b200 import lora_attn
    return lora_attn


def _compare(la, s, inp):
    d = {k: v.to(DEV) for k, v in inp.items()}
    out_ws = torch.empty(d["q"].shape, device=DEV)
    args = la.make_args(d["k_base"], d["v_base"], d["lr"], d["B_k"], d["B_v"], d["q"], out_ws,
                        lora_scale=s.lora_scale, rope_base=s.rope_base, kv_len=d["kv_len"],
                        max_kv_len=int(inp["kv_len"].max()))
    need = la.lora_attn_decode_workspace_bytes(args)
    assert 0 < need <= la.LA_STATIC_SCRATCH_BYTES
    la.lora_attn_decode(args, la.decode_workspace(args, DEV))
    torch.cuda.synchronize()
    ref = out_ws.cpu()
    for _ in range(2):  # two calls in a row share (and reuse) the static scratch
        out = torch.full(d["q"].shape, float("nan"), device=DEV)
        a2 = la.make_args(d["k_base"], d["v_base"], d["lr"], d["B_k"], d["B_v"], d["q"], out,
                          lora_scale=s.lora_scale, rope_base=s.rope_base, kv_len=d["kv_len"],
                          max_kv_len=int(inp["kv_len"].max()))
        st = la.lib.lora_attn_decode_static_scratch(ctypes.byref(a2),
                                                    torch.cuda.current_stream().cuda_stream)
        assert st == la.LA_OK, la.status_string(st)
        torch.cuda.synchronize()
        assert la.la_device_check() == la.LA_OK
        assert_parity(to_np(out), to_np(ref), s.dtype)
    assert_parity(to_np(out), oracle_decode(inp, s), s.dtype)   # and the oracle itself


@pytest.mark.gpu
def test_static_scratch_matches_workspace_decode_bf16(la):
    """The LLaMA-shaped 8192-token decode (r = 16) and the stack's r = 64 decode,
    both with split partials and arrival counters in the scratch."""
    s = W.LLAMA8B_DECODE_8K
    _compare(la, s, W.direct_cache_inputs(s))
    s = W.llama8b_stack_decode(0).replace(kv_len=4096, seed=17)
    _compare(la, s, W.direct_cache_inputs(s))


@pytest.mark.gpu
def test_static_scratch_matches_workspace_decode_fp32(la):
    """The fp32 generic kernel, whose split merge also uses arrival counters."""
    s = W.TINY_FP32
    inp = W.direct_cache_inputs(s.replace(dtype=torch.float32))
    _compare(la, s, inp)


@pytest.mark.gpu
def test_static_scratch_after_a_larger_call_clears_its_counters(la):
    """Two shapes in a row: the second decode's arrival counters sit inside the
    bytes where the first left its split partials (nonzero floats), so the
    call must clear them before it launches.  Checked against the oracle."""
    from tests.helpers import oracle_decode
    big = W.llama8b_stack_decode(0).replace(kv_len=8192)
    small = W.llama8b_stack_decode(0).replace(kv_len=300, seed=91)
    outs = []
    for s in (big, small):
        inp = W.direct_cache_inputs(s)
        d = {k: v.to(DEV) for k, v in inp.items()}
        out = torch.full(d["q"].shape, float("nan"), device=DEV)
        a = la.make_args(d["k_base"], d["v_base"], d["lr"], d["B_k"], d["B_v"], d["q"], out,
                         lora_scale=s.lora_scale, rope_base=s.rope_base, kv_len=d["kv_len"],
                         max_kv_len=s.kv_len)
        # d stays referenced: the arguments hold raw pointers into its tensors
        outs.append((s, inp, out, a, la.lora_attn_decode_workspace_bytes(a), d))
    (_, _, _, a_big, need_big, _), (_, _, _, a_small, _, _) = outs
    # the small decode's counters start before the big decode's scratch ends
    assert need_big > 0 and la.lora_attn_decode_workspace_bytes(a_small) < need_big
    for s, inp, out, a, _, _ in outs:
        st = la.lib.lora_attn_decode_static_scratch(ctypes.byref(a),
                                                    torch.cuda.current_stream().cuda_stream)
        assert st == la.LA_OK, la.status_string(st)
    torch.cuda.synchronize()
    assert la.la_device_check() == la.LA_OK
    for s, inp, out, _, _, _ in outs:
        assert_parity(to_np(out), oracle_decode(inp, s), s.dtype)


def test_static_scratch_empty_batch_is_ok(la):
    """n_seqs = 0 is a valid, empty batch: LA_OK with nothing launched, as for
    lora_attn_decode (whose workspace is 0 bytes and may be NULL)."""
    a = la.AttnArgs()
    a.n_seqs, a.n_agents, a.n_q_heads, a.n_kv_heads, a.head_dim, a.r = 0, 3, 32, 8, 128, 16
    a.lora_scale, a.softmax_scale, a.rope_base = 2.0, 0.088, 500000.0
    a.L_max = 8192
    a.k_base = a.v_base = a.lr_cache = a.B_k = a.B_v = a.q = a.out = a.kv_len = FAKE
    a.kv_seq_stride, a.kv_head_stride, a.kv_tok_stride = 8 * 8192 * 128, 8192 * 128, 128
    a.lr_seq_stride = 8192 * 32
    a.max_kv_len = 8192
    a.n_q_tokens = 1
    a.io_dtype = a.out_dtype = la.LA_BF16
    assert la.lora_attn_decode_workspace_bytes(a) == 0
    assert la.lib.lora_attn_decode_static_scratch(ctypes.byref(a), None) == la.LA_OK
    assert la.lib.lora_attn_decode(ctypes.byref(a), None, 0, None) == la.LA_OK
    bad = la.AttnArgs()
    ctypes.memmove(ctypes.byref(bad), ctypes.byref(a), ctypes.sizeof(a))
    bad.r = 12
    assert la.lib.lora_attn_decode_static_scratch(ctypes.byref(bad), None) == la.LA_ERR_UNSUPPORTED
    bad.r, bad.k_base = 16, 0
    assert la.lib.lora_attn_decode_static_scratch(ctypes.byref(bad), None) == la.LA_ERR_INVALID_ARG


def test_static_scratch_rejects_oversized_request(la):
    """Arguments needing more scratch than the array are refused before any
    launch (the fake pointers are never touched)."""
    a = la.AttnArgs()
    a.n_seqs, a.n_agents, a.n_q_heads, a.n_kv_heads, a.head_dim, a.r = 1, 16, 4, 1, 128, 64
    a.lora_scale, a.softmax_scale, a.rope_base = 2.0, 0.088, 10000.0
    a.L_max = 1 << 20
    a.k_base = a.v_base = a.lr_cache = a.B_k = a.B_v = a.q = a.out = a.kv_len = FAKE
    a.kv_seq_stride, a.kv_head_stride, a.kv_tok_stride = (1 << 20) * 128, (1 << 20) * 128, 128
    a.lr_seq_stride = (1 << 20) * 128
    a.max_kv_len = 1 << 20
    a.n_q_tokens = 1
    a.io_dtype = a.out_dtype = la.LA_F32
    assert la.lora_attn_decode_workspace_bytes(a) > la.LA_STATIC_SCRATCH_BYTES
    st = la.lib.lora_attn_decode_static_scratch(ctypes.byref(a), None)
    assert st == la.LA_ERR_SCRATCH_LIMIT
    assert "LA_ERR_SCRATCH_LIMIT" in la.status_string(st)
    bad = la.AttnArgs()
    ctypes.memmove(ctypes.byref(bad), ctypes.byref(a), ctypes.sizeof(a))
    bad.head_dim = 96
    assert la.lib.lora_attn_decode_static_scratch(ctypes.byref(bad), None) == la.LA_ERR_UNSUPPORTED
