"""Host-side checks of the C ABI: the library loads on a machine without a GPU,
exports every entry point include/lora_attn.h declares, its struct layout
matches the binding, and invalid arguments are rejected before any launch.

Every call below carries at least one invalid argument, so none of them can
reach a kernel launch (the fake pointers are never dereferenced)."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

from rank_attention_b200 import lora_attn as la

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lora_attn.h")
FAKE = 0x10000  # 16-byte aligned, never dereferenced


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"#define.*", "", text)
    return sorted(set(re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", text)) -
                  {"sizeof", "defined"})


def test_every_declared_symbol_is_exported():
    names = declared_functions()
    assert set(names) == set(la.EXPORTED), names
    lib = ctypes.CDLL(la.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings():
    for s in range(8):
        assert la.status_string(s).startswith("LA_")
    assert "unknown" in la.status_string(99)


def test_struct_layout_matches_header(tmp_path):
    fields = [f[0] for f in la.AttnArgs._fields_]
    src = tmp_path / "layout.c"
    body = "\n".join(f'printf("{f} %zu\\n", offsetof(la_attn_args, {f}));' for f in fields)
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "lora_attn.h"\n'
                   "int main(void){" + body +
                   'printf("sizeof %zu\\n", sizeof(la_attn_args)); return 0;}\n')
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", os.path.join(ROOT, "include"), str(src), "-o",
                    str(exe)], check=True)
    out = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True,
                                                        text=True, check=True).stdout.split("\n")
               if line)
    for f in fields:
        assert int(out[f]) == getattr(la.AttnArgs, f).offset, f
    assert int(out["sizeof"]) == ctypes.sizeof(la.AttnArgs)


def _append(**kw):
    a = dict(X=FAKE, ldx=256, n=4, H=256, A=FAKE, r=8, lr=FAKE, L_max=16, pos0=0, n_seqs=1,
             sx=0, slr=0, dt=la.LA_F32)
    a.update(kw)
    return la.lib.lr_cache_append(a["X"], a["ldx"], a["n"], a["H"], a["A"], a["r"], a["lr"],
                                  a["L_max"], a["pos0"], a["n_seqs"], a["sx"], a["slr"], a["dt"],
                                  None)


@pytest.mark.parametrize("kw,status", [
    (dict(X=0), la.LA_ERR_INVALID_ARG),
    (dict(A=0), la.LA_ERR_INVALID_ARG),
    (dict(lr=0), la.LA_ERR_INVALID_ARG),
    (dict(X=FAKE + 4), la.LA_ERR_INVALID_ARG),
    (dict(r=12), la.LA_ERR_UNSUPPORTED),
    (dict(dt=7), la.LA_ERR_INVALID_ARG),
    (dict(ldx=100), la.LA_ERR_INVALID_ARG),
    (dict(ldx=258), la.LA_ERR_INVALID_ARG),
    (dict(pos0=13), la.LA_ERR_CAPACITY),
    (dict(pos0=-1), la.LA_ERR_CAPACITY),
    (dict(n=-1), la.LA_ERR_INVALID_ARG),
    (dict(H=0), la.LA_ERR_INVALID_ARG),
])
def test_append_rejects(kw, status):
    assert _append(**kw) == status


def _args(**kw):
    a = la.AttnArgs()
    a.n_seqs, a.n_agents, a.n_q_heads, a.n_kv_heads, a.head_dim, a.r = 1, 2, 4, 2, 64, 8
    a.lora_scale, a.softmax_scale, a.rope_base = 2.0, 0.125, 10000.0
    a.L_max = 256
    a.k_base = a.v_base = a.lr_cache = a.B_k = a.B_v = a.q = a.out = a.kv_len = FAKE
    a.kv_seq_stride, a.kv_head_stride, a.kv_tok_stride = 2 * 256 * 64, 256 * 64, 64
    a.lr_seq_stride = 256 * 16
    a.max_kv_len = 256
    a.q_pos0, a.n_q_tokens = 0, 1
    a.io_dtype = a.out_dtype = la.LA_F32
    for k, v in kw.items():
        setattr(a, k, v)
    return a


BAD_ATTN = [
    (dict(head_dim=96), la.LA_ERR_UNSUPPORTED),
    (dict(r=24), la.LA_ERR_UNSUPPORTED),
    (dict(n_q_heads=5), la.LA_ERR_INVALID_ARG),
    (dict(n_agents=0), la.LA_ERR_INVALID_ARG),
    (dict(k_base=0), la.LA_ERR_INVALID_ARG),
    (dict(out=FAKE + 8), la.LA_ERR_INVALID_ARG),
    (dict(kv_tok_stride=32), la.LA_ERR_INVALID_ARG),
    (dict(kv_head_stride=3), la.LA_ERR_INVALID_ARG),
    (dict(lr_seq_stride=100), la.LA_ERR_INVALID_ARG),
    (dict(softmax_scale=0.0), la.LA_ERR_INVALID_ARG),
    (dict(softmax_scale=float("nan")), la.LA_ERR_INVALID_ARG),
    (dict(rope_base=0.5), la.LA_ERR_INVALID_ARG),
    (dict(io_dtype=3), la.LA_ERR_INVALID_ARG),
    (dict(n_agents=40), la.LA_ERR_UNSUPPORTED),
    (dict(lr_agent_stride=-4096), la.LA_ERR_INVALID_ARG),
    (dict(lr_agent_stride=4097), la.LA_ERR_INVALID_ARG),   # not a multiple of 16 bytes
    (dict(lr_agent_stride=2048), la.LA_ERR_INVALID_ARG),   # overlaps the next agent's cache
    (dict(value_path=4), la.LA_ERR_INVALID_ARG),
    (dict(value_path=-1), la.LA_ERR_INVALID_ARG),
]


@pytest.mark.parametrize("kw,status", BAD_ATTN + [
    (dict(n_q_tokens=2), la.LA_ERR_INVALID_ARG),
    (dict(kv_len=0), la.LA_ERR_INVALID_ARG),
    (dict(max_kv_len=0), la.LA_ERR_INVALID_ARG),
    (dict(max_kv_len=257), la.LA_ERR_CAPACITY),
])
def test_decode_rejects(kw, status):
    a = _args(**kw)
    assert la.lib.lora_attn_decode(ctypes.byref(a), FAKE, 1 << 20, None) == status
    assert la.lib.lora_attn_decode_workspace_bytes(ctypes.byref(a)) == 0


def test_decode_rejects_small_workspace():
    a = _args()
    need = la.lib.lora_attn_decode_workspace_bytes(ctypes.byref(a))
    assert need > 0
    assert la.lib.lora_attn_decode(ctypes.byref(a), FAKE, need - 1, None) == la.LA_ERR_WORKSPACE
    assert la.lib.lora_attn_decode(ctypes.byref(a), 0, need, None) == la.LA_ERR_WORKSPACE
    assert la.lib.lora_attn_decode(ctypes.byref(a), FAKE + 16, need, None) == la.LA_ERR_WORKSPACE


@pytest.mark.parametrize("kw,status", BAD_ATTN + [
    (dict(q_pos0=250, n_q_tokens=7), la.LA_ERR_CAPACITY),
    (dict(q_pos0=-1), la.LA_ERR_INVALID_ARG),
    (dict(n_q_tokens=-1), la.LA_ERR_INVALID_ARG),
])
def test_prefill_rejects(kw, status):
    a = _args(**kw)
    assert la.lib.lora_attn_prefill(ctypes.byref(a), None) == status


def test_per_agent_lr_stride_accepted():
    # one LR cache per agent, laid out back to back: a valid plan
    a = _args(lr_agent_stride=256 * 16)
    assert la.lib.lora_attn_decode_workspace_bytes(ctypes.byref(a)) > 0


def test_per_agent_lr_too_large_for_the_generic_kernel():
    # fp32 runs on the generic kernel, which stages every agent's LR tile:
    # 16 agents at r = 64, d = 128 exceed its shared memory, refused before launch
    a = _args(n_agents=16, head_dim=128, r=64, lr_seq_stride=256 * 128,
              kv_seq_stride=2 * 256 * 128, kv_head_stride=256 * 128, kv_tok_stride=128,
              lr_agent_stride=256 * 128)
    assert la.lib.lora_attn_decode(ctypes.byref(a), FAKE, 1 << 26, None) == la.LA_ERR_UNSUPPORTED
    a.n_q_tokens = 1
    assert la.lib.lora_attn_prefill(ctypes.byref(a), None) == la.LA_ERR_UNSUPPORTED


def _append_agents(**kw):
    a = dict(X=FAKE, ldx=256, n=4, H=256, A=FAKE, na=2, r=8, lr=FAKE, ls=16 * 16, L_max=16,
             pos0=0, n_seqs=1, sx=0, slr=0, dt=la.LA_F32)
    a.update(kw)
    return la.lib.lr_cache_append_agents(a["X"], a["ldx"], a["n"], a["H"], a["A"], a["na"],
                                         a["r"], a["lr"], a["ls"], a["L_max"], a["pos0"],
                                         a["n_seqs"], a["sx"], a["slr"], a["dt"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(na=0), la.LA_ERR_INVALID_ARG),
    (dict(ls=101), la.LA_ERR_INVALID_ARG),       # not a multiple of 16 bytes
    (dict(ls=16), la.LA_ERR_INVALID_ARG),        # overlaps the next agent's cache
    (dict(X=0), la.LA_ERR_INVALID_ARG),
    (dict(r=12), la.LA_ERR_UNSUPPORTED),
    (dict(pos0=13), la.LA_ERR_CAPACITY),
])
def test_append_agents_rejects(kw, status):
    assert _append_agents(**kw) == status


def _qexp(**kw):
    a = dict(qb=FAKE, lr=FAKE, B=FAKE, qo=FAKE, n=1, na=3, nt=1, nq=32, d=128, r=16, s=2.0,
             base=500000.0, pe=FAKE, dt=la.LA_BF16)
    a.update(kw)
    return la.lib.lora_query_expand(a["qb"], a["lr"], a["B"], a["qo"], a["n"], a["na"], a["nt"],
                                    a["nq"], a["d"], a["r"], a["s"], a["base"], a["pe"], a["dt"],
                                    None)


@pytest.mark.parametrize("kw,status", [
    (dict(qb=0), la.LA_ERR_INVALID_ARG),
    (dict(pe=0), la.LA_ERR_INVALID_ARG),
    (dict(qo=FAKE + 2), la.LA_ERR_INVALID_ARG),
    (dict(nt=0), la.LA_ERR_INVALID_ARG),
    (dict(base=1.0), la.LA_ERR_INVALID_ARG),
    (dict(d=96), la.LA_ERR_UNSUPPORTED),
    (dict(r=12), la.LA_ERR_UNSUPPORTED),
    (dict(dt=5), la.LA_ERR_INVALID_ARG),
])
def test_query_expand_rejects(kw, status):
    assert _qexp(**kw) == status


def _odelta(**kw):
    a = dict(o=FAKE, A=FAKE, As=0, B=FAKE, y=FAKE, n=1, na=3, nt=1, di=4096, do=4096, r=16,
             s=2.0, dt=la.LA_BF16)
    a.update(kw)
    return la.lib.lora_output_delta(a["o"], a["A"], a["As"], a["B"], a["y"], a["n"], a["na"],
                                    a["nt"], a["di"], a["do"], a["r"], a["s"], a["dt"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(y=0), la.LA_ERR_INVALID_ARG),
    (dict(A=FAKE + 4), la.LA_ERR_INVALID_ARG),
    (dict(As=-1), la.LA_ERR_INVALID_ARG),
    (dict(As=4100), la.LA_ERR_INVALID_ARG),      # agents' A_o not 16-byte aligned
    (dict(di=0), la.LA_ERR_INVALID_ARG),
    (dict(r=3), la.LA_ERR_UNSUPPORTED),
    (dict(do=4100), la.LA_ERR_UNSUPPORTED),
    (dict(s=float("inf")), la.LA_ERR_INVALID_ARG),
])
def test_output_delta_rejects(kw, status):
    assert _odelta(**kw) == status


def test_null_args():
    assert la.lib.lora_attn_prefill(None, None) == la.LA_ERR_INVALID_ARG
    assert la.lib.lora_attn_decode(None, FAKE, 1 << 20, None) == la.LA_ERR_INVALID_ARG
    assert la.lib.lora_attn_decode_workspace_bytes(None) == 0
    assert la.lib.lora_decode_step_host(None, FAKE, 1 << 20, FAKE, 64, FAKE, FAKE, FAKE, FAKE,
                                        FAKE, None) == la.LA_ERR_INVALID_ARG


def _step(a=None, ws_bytes=1 << 20, A_kv=FAKE, hidden=64, x_dev=FAKE, x_host=FAKE, q_host=FAKE,
          kv_len=(5,), out_host=FAKE):
    a = a if a is not None else _args()
    kv = (ctypes.c_int32 * len(kv_len))(*kv_len) if kv_len is not None else None
    return la.lib.lora_decode_step_host(ctypes.byref(a), FAKE, ws_bytes, A_kv, hidden, x_dev,
                                        x_host, q_host, kv, out_host, None)


@pytest.mark.parametrize("kw,status", [
    (dict(kv_len=(0,)), la.LA_ERR_INVALID_ARG),        # no key: the new token has no row
    (dict(kv_len=(257,)), la.LA_ERR_INVALID_ARG),      # above max_kv_len
    (dict(kv_len=None), la.LA_ERR_INVALID_ARG),
    (dict(x_host=0), la.LA_ERR_INVALID_ARG),
    (dict(q_host=0), la.LA_ERR_INVALID_ARG),
    (dict(out_host=0), la.LA_ERR_INVALID_ARG),
    (dict(x_dev=0), la.LA_ERR_INVALID_ARG),
    (dict(x_dev=FAKE + 8), la.LA_ERR_INVALID_ARG),     # staging not 16-byte aligned
    (dict(A_kv=0), la.LA_ERR_INVALID_ARG),
    (dict(hidden=0), la.LA_ERR_INVALID_ARG),
    (dict(hidden=6), la.LA_ERR_INVALID_ARG),           # 24-byte rows
    (dict(ws_bytes=16), la.LA_ERR_WORKSPACE),
] + [(dict(a=_args(**kw)), st) for kw, st in BAD_ATTN])
def test_decode_step_host_rejects(kw, status):
    """Every check of the host-buffer step runs before anything is queued."""
    assert _step(**kw) == status


def test_decode_step_host_second_sequence_checked():
    # the second sequence's length is checked too, before any copy
    a = _args(n_seqs=2)
    assert _step(a=a, kv_len=(5, 300)) == la.LA_ERR_INVALID_ARG


def test_packed_step_inputs_back_to_back():
    """The helper's views sit in the order and with no gap that let
    lora_decode_step_host move a step's inputs in one copy."""
    import torch
    buf, x, q, kv = la.packed_step_inputs((2, 1, 64), (2, 3, 1, 4, 64), 2, torch.bfloat16, "cpu")
    assert x.data_ptr() == buf.data_ptr()
    assert q.data_ptr() == x.data_ptr() + x.numel() * 2
    assert kv.data_ptr() == q.data_ptr() + q.numel() * 2
    assert kv.dtype == torch.int32 and kv.numel() == 2
    assert buf.numel() == (x.numel() + q.numel()) * 2 + 8


@pytest.mark.parametrize("kw,status", [
    (dict(key_pos0=-1), la.LA_ERR_INVALID_ARG),
    (dict(row_stats=FAKE + 4), la.LA_ERR_INVALID_ARG),
    # the generic fp32 decode does not take the sharded decode's inputs
    (dict(key_pos0=128), la.LA_ERR_UNSUPPORTED),
    (dict(row_stats=FAKE), la.LA_ERR_UNSUPPORTED),
])
def test_sharded_decode_inputs_checked(kw, status):
    a = _args(**kw)
    assert la.lib.lora_attn_decode(ctypes.byref(a), FAKE, 1 << 20, None) == status


@pytest.mark.parametrize("kw", [dict(key_pos0=128), dict(row_stats=FAKE)])
def test_sharded_inputs_refused_outside_the_decode(kw):
    a = _args(**kw)
    assert la.lib.lora_attn_prefill(ctypes.byref(a), None) == la.LA_ERR_UNSUPPORTED
    assert la.lib.lora_materialize_agent_kv(ctypes.byref(a), FAKE, FAKE, None) == la.LA_ERR_UNSUPPORTED


@pytest.mark.parametrize("kw,status", [
    (dict(outs=0), la.LA_ERR_INVALID_ARG),
    (dict(stats=0), la.LA_ERR_INVALID_ARG),
    (dict(out=0), la.LA_ERR_INVALID_ARG),
    (dict(n_parts=0), la.LA_ERR_INVALID_ARG),
    (dict(rows=-1), la.LA_ERR_INVALID_ARG),
    (dict(d=6), la.LA_ERR_INVALID_ARG),
    (dict(dt=3), la.LA_ERR_INVALID_ARG),
    (dict(outs=FAKE + 8), la.LA_ERR_INVALID_ARG),         # fp32 rows read four at a time
    (dict(stats=FAKE + 4), la.LA_ERR_INVALID_ARG),
    (dict(rows=0), la.LA_OK),                             # nothing to merge, nothing launched
])
def test_combine_checks(kw, status):
    a = dict(outs=FAKE, stats=FAKE, n_parts=2, rows=8, d=128, dt=la.LA_F32, out=FAKE)
    a.update(kw)
    assert la.lib.lora_attn_decode_combine(a["outs"], a["stats"], a["n_parts"], a["rows"], a["d"],
                                           a["dt"], a["out"], None) == status
