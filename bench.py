#!/usr/bin/env python
"""Benchmark of the Flash-LoRA-Attention hot path on B200.

One step = one decode step of the LLaMA-3.1-8B-shaped layer with three agents
over an 8192-token shared context (hidden 4096, 32 query / 8 KV heads,
head_dim 128, LoRA rank 16, alpha 32, bf16 caches, fp32 accumulation):
  1. lr_cache_append of the new token's row X_t [A_k | A_v];
  2. lora_attn_decode of every agent's query over the shared base and LR caches.
value = agent-tokens per second over all ranks (3 per step per rank).

The working set of one step is 34 MB, which fits in the 126 MB L2, so the
steps rotate over enough independent cache sets (each a full synthetic
problem) that consecutive steps never find their inputs in L2.

--impl reference times the fp64 CPU oracle on the same workload (rank 0 only).
Multi-GPU: one process per GPU, each serving its own independent requests
(weak scaling); the only collective is the timing barrier / max.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Flash-LoRA-Attn decode agent-tokens/s & % HBM peak; prefill TFLOP/s & % TC peak"
UNIT = "agent-tokens/s"
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", nargs="?", const="decode",
                    choices=["decode", "prefill", "append", "qkvo"],
                    help="a short deterministic run of one kernel for profilers "
                         "(decode: the 8192-token decode five times; prefill: the "
                         "16384 + 1024-token prefill three times); prints nothing")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


NOMINAL_HBM_GBS = 8000.0      # B200 HBM3e, nominal (7.7 TB/s in the HGX figure)
NOMINAL_BF16_TFLOPS = 2250.0  # B200 dense bf16 tensor cores, nominal


def tc_peak():
    """Dense bf16 tensor-core peak (TFLOP/s) for a kernel timed on its own."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured cuBLAS bf16 burst"
    except Exception:
        return 1590.0, "fallback"


def prefill_flops(s):
    """4 d flops per unmasked (query, key) pair (Q K^T and P V), plus the
    LoRA-inclusive count: 2 r per pair for P LR_v, 2 r d per (agent, KV head,
    key) for the key delta, 2 r d per query row for the epilogue."""
    pairs = s.n_agents * s.n_q_heads * sum(s.q_pos0 + j + 1 for j in range(s.n_q_tokens))
    base = 4 * s.head_dim * pairs
    keys = s.n_agents * s.n_kv_heads * (s.q_pos0 + s.n_q_tokens)
    lora = 2 * s.r * pairs + 2 * s.r * s.head_dim * keys + \
        2 * s.r * s.head_dim * s.n_agents * s.n_q_heads * s.n_q_tokens
    return base, base + lora


def non_shared_setup(la, s, inp, dev):
    """The non-shared baseline of one decode step: every agent's K^a, V^a
    materialised (lora_materialize_agent_kv), then plain attention over the
    per-agent caches -- the same decode kernel with n_seqs * n_agents
    sequences of one agent and B = 0, so it reads n_agents x the base cache.
    Returns (materialise, decode, outputs [n_seqs, n_agents, 1, n_q, d])."""
    import torch
    n, na, nkv, d, r = s.n_seqs, s.n_agents, s.n_kv_heads, s.head_dim, s.r
    L = inp["k_base"].shape[2]
    kout = torch.empty((n, na, nkv, L, d), dtype=inp["k_base"].dtype, device=dev)
    vout = torch.empty_like(kout)
    q = inp["q"]
    out = torch.empty(q.shape, dtype=torch.float32, device=dev)
    margs = la.make_args(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"], q, out,
                         lora_scale=s.lora_scale, rope_base=s.rope_base, kv_len=inp["kv_len"],
                         max_kv_len=int(s.kv_len))
    zlr = torch.zeros((n * na, L, 2 * r), dtype=inp["lr"].dtype, device=dev)
    zb = torch.zeros((1, r, nkv * d), dtype=inp["B_k"].dtype, device=dev)
    kv_len = inp["kv_len"].repeat_interleave(na)
    q1 = q.reshape(n * na, 1, q.shape[2], q.shape[3], d)
    out1 = out.view(n * na, 1, q.shape[2], q.shape[3], d)
    dargs = la.make_args(kout.view(n * na, nkv, L, d), vout.view(n * na, nkv, L, d), zlr, zb, zb,
                         q1, out1, lora_scale=s.lora_scale, rope_base=s.rope_base, kv_len=kv_len,
                         max_kv_len=int(s.kv_len))
    ws = la.decode_workspace(dargs, dev)
    keep = (kout, vout, zlr, zb, kv_len, q1, out1, ws)

    def materialise(stream=None):
        la.lora_materialize_agent_kv(margs, kout, vout, stream)

    def decode(stream=None):
        la.lora_attn_decode(dargs, ws, stream)

    materialise.keep = keep
    return materialise, decode, out


def time_non_shared(dev, shared_decode_us, reps=5):
    """Time the non-shared baseline on the decode workload (L2 flushed before
    each timed launch) and report its bytes beside the shared path's."""
    import torch
    from rank_attention_b200 import lora_attn as la
    from rank_attention_b200 import workloads as W
    s = W.LLAMA8B_DECODE_8K
    inp = W.direct_cache_inputs(s, device=dev)
    mat, dec, _ = non_shared_setup(la, s, inp, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    mat()
    dec()
    torch.cuda.synchronize()

    def timed(fn):
        ts = []
        for _ in range(reps):
            flush.fill_(1)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts) * 1e3

    mat_us, dec_us = timed(mat), timed(dec)
    if la.la_device_check() != 0:
        raise RuntimeError("non-shared baseline device check failed")
    shared = decode_bytes(s)
    e = 2
    ns_bytes = (2 * s.n_seqs * s.n_agents * s.n_kv_heads * s.kv_len * s.head_dim * e
                + s.n_seqs * s.n_agents * s.n_q_heads * s.head_dim * (e + 4))
    return {"workload": s.name, "decode_us": dec_us, "materialise_us": mat_us,
            "bytes_per_decode": ns_bytes, "shared_bytes_per_decode": shared,
            "bytes_saved_frac": 1.0 - shared / ns_bytes,
            "shared_speedup": dec_us / shared_decode_us,
            "what": "per-agent K^a, V^a materialised once (materialise_us, not per step), then "
                    "attention over n_agents separate caches (decode_us): the same decode kernel "
                    "with B = 0"}


def time_prefill(dev, reps=5, warmup=3, s=None, value_path=0):
    """A chunked prefill workload (default: 16384-token prefix + 1024-token
    chunk per agent, 3 agents, r = 16): one lora_attn_prefill per launch, CUDA
    events around each launch, L2 flushed (256 MB written) before each."""
    import torch
    from rank_attention_b200 import lora_attn as la
    from rank_attention_b200 import workloads as W
    s = s or W.LLAMA8B_PREFILL_16K
    inp = W.direct_cache_inputs(s, device=dev)
    out = torch.empty(inp["q"].shape, dtype=torch.bfloat16, device=dev)
    args = la.make_args(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"],
                        inp["q"], out, lora_scale=s.lora_scale, rope_base=s.rope_base,
                        q_pos0=s.q_pos0, value_path=value_path)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        la.lora_attn_prefill(args)
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        la.lora_attn_prefill(args)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    if la.la_device_check() != 0:
        raise RuntimeError("prefill device check failed")
    ms = statistics.median(times)
    base, lora = prefill_flops(s)
    peak, kind = tc_peak()
    tf = base / (ms / 1e3) / 1e12
    return {"workload": s.name, "value": tf, "unit": "TFLOP/s", "ms": ms,
            "flops_per_launch": base, "lora_inclusive_tflops": lora / (ms / 1e3) / 1e12,
            "peak": peak, "peak_kind": kind, "frac": tf / peak,
            "frac_of_nominal": tf / NOMINAL_BF16_TFLOPS, "out_dtype": "bf16",
            "timing": f"median of {reps} launches, CUDA events, L2 flushed before each"}


def time_decode_shape(dev, s, reps=5, warmup=3, value_path=0):
    """One lora_attn_decode launch of a decode workload, CUDA events around
    each launch, L2 flushed before each; HBM roofline on its algorithmic bytes."""
    import torch
    from rank_attention_b200 import lora_attn as la
    from rank_attention_b200 import workloads as W
    inp = W.direct_cache_inputs(s, device=dev)
    out = torch.empty(inp["q"].shape, dtype=torch.bfloat16, device=dev)
    args = la.make_args(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"],
                        inp["q"], out, lora_scale=s.lora_scale, rope_base=s.rope_base,
                        kv_len=inp["kv_len"], max_kv_len=s.kv_len, value_path=value_path)
    ws = la.decode_workspace(args, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        la.lora_attn_decode(args, ws)
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        la.lora_attn_decode(args, ws)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    if la.la_device_check() != 0:
        raise RuntimeError("decode device check failed")
    ms = statistics.median(times)
    hbm, kind = peaks()
    b = decode_bytes(s)
    gbs = b / (ms / 1e3) / 1e9
    return {"workload": s.name, "kind": "decode", "us": ms * 1e3,
            "agent_tokens_per_s": s.n_seqs * s.n_agents / (ms / 1e3),
            "algorithmic_bytes": b, "GB/s": gbs, "peak": hbm, "frac": gbs / hbm,
            "timing": f"median of {reps} launches, CUDA events, L2 flushed before each"}


def time_value_ablation(dev, prefill_reordered=None):
    """The reordering of the value side, each pair of arms on one kernel.
    Prefill (tensor cores, the chunked-prefill workload): O_lr = P LRv with
    B_v^a once per row (reordered, the product path) against dV = LRv B_v^a
    on the tensor cores, V^a = V_base + s dV rebuilt over V_base in shared
    memory per key tile, then O += P V^a (per tile).  Decode (the generic
    CUDA-core kernel, the 8192-key decode): the same two arms; the
    tensor-core decode (reordered) timed alike, for context."""
    from rank_attention_b200 import workloads as W
    pre_re = prefill_reordered or time_prefill(dev)
    pre_pt = time_prefill(dev, value_path=2)
    s = W.LLAMA8B_DECODE_8K
    reord = time_decode_shape(dev, s, value_path=1)
    naive = time_decode_shape(dev, s, value_path=3)
    tc = time_decode_shape(dev, s, value_path=0)
    return {"prefill": {"workload": pre_re["workload"], "reordered_ms": pre_re["ms"],
                        "per_tile_ms": pre_pt["ms"], "reordering_gain": pre_pt["ms"] / pre_re["ms"],
                        "kernels": "both tcgen05 (prefill_tc_kernel, per-tile arm: VT)"},
            "decode_generic": {"workload": s.name, "reordered_us": reord["us"],
                               "per_tile_us": naive["us"], "reordering_gain": naive["us"] / reord["us"],
                               "tensor_core_reordered_us": tc["us"]},
            "what": "value side reordered (P LRv, B_v once per row) against V^a rebuilt in head "
                    "dimension per key tile, same kernel and tiling per pair; the pages report "
                    "1.24x (BaseShared) / 1.35x (BaseLRShared) for their kernel, end to end, on "
                    "other hardware",
            "timing": reord["timing"]}


def time_base_shared(dev):
    """The decode workload with one LR cache per agent (each agent's own A_a,
    BaseShared) beside the same decode over one shared LR cache, both timed
    alike (single launches, L2 flushed), with the caches' sizes."""
    from rank_attention_b200 import workloads as W
    s = W.LLAMA8B_DECODE_8K
    own = time_decode_shape(dev, s.replace(lr_per_agent=True))
    shared = time_decode_shape(dev, s)
    lr_one = s.n_seqs * s.kv_len * 2 * s.r * 2
    base = 2 * s.n_seqs * s.n_kv_heads * s.kv_len * s.head_dim * 2
    return {"workload": s.name + "_lr_per_agent", "decode_us": own["us"], "GB/s": own["GB/s"],
            "frac": own["frac"], "algorithmic_bytes": own["algorithmic_bytes"],
            "shared_lr_decode_us": shared["us"],
            "cache_bytes": {"base": base, "lr_per_agent_total": s.n_agents * lr_one,
                            "lr_shared": lr_one},
            "what": "each agent reads its own LR cache X A_a beside the shared base cache "
                    "(at r = 16 up to three agents a CTA, each stage holding every agent's LR "
                    "tile); shared_lr_decode_us: the same decode with one LR cache (shared A), "
                    "timed the same way",
            "timing": own["timing"]}


def _time_launches(fn, flush, reps=5, warmup=3):
    """Median CUDA-event time (ms) of single launches, L2 flushed before each."""
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return statistics.median(times)


def time_qkvo(dev):
    """Query- and output-side LoRA (the qkvo setting) on the 3-agent layer: one
    decode token per agent, and a 1024-token chunk per agent.  HBM roofline on
    the bytes each kernel must move (inputs once, outputs once)."""
    import torch
    from rank_attention_b200 import lora_attn as la
    from rank_attention_b200 import workloads as W
    s = W.LLAMA8B_DECODE_8K
    na, nq, d, r, e = s.n_agents, s.n_q_heads, s.head_dim, s.r, 2
    D = nq * d
    hbm, _ = peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(5)
    res = {}
    for n_tok in (1, 1024):
        qb = torch.randn(1, na, n_tok, nq, d, generator=g, device=dev).to(torch.bfloat16)
        lrq = torch.randn(1, na, n_tok, r, generator=g, device=dev).to(torch.bfloat16)
        Bq = (0.02 * torch.randn(na, r, D, generator=g, device=dev)).to(torch.bfloat16)
        qo = torch.empty_like(qb)
        pe = torch.full((1,), s.kv_len, dtype=torch.int32, device=dev)
        o = torch.randn(1, na, n_tok, D, generator=g, device=dev).to(torch.bfloat16)
        Ao = (0.02 * torch.randn(D, r, generator=g, device=dev)).to(torch.bfloat16)
        Bo = (0.02 * torch.randn(na, r, D, generator=g, device=dev)).to(torch.bfloat16)
        y = torch.randn(1, na, n_tok, D, generator=g, device=dev).to(torch.bfloat16)
        q_ms = _time_launches(lambda: la.lora_query_expand(qb, lrq, Bq, qo, pe, lora_scale=s.lora_scale,
                                                           rope_base=s.rope_base), flush)
        o_ms = _time_launches(lambda: la.lora_output_delta(o, Ao, Bo, y, lora_scale=s.lora_scale),
                              flush)
        if la.la_device_check() != 0:
            raise RuntimeError("qkvo device check failed")
        qbytes = (2 * na * n_tok * D + na * n_tok * r + na * r * D) * e
        obytes = (na * n_tok * D + D * r + na * r * D + 2 * na * n_tok * D) * e
        res[f"{n_tok}_tok"] = {
            "query_expand_us": q_ms * 1e3, "query_expand_GB/s": qbytes / (q_ms / 1e3) / 1e9,
            "query_expand_frac": qbytes / (q_ms / 1e3) / 1e9 / hbm, "query_expand_bytes": qbytes,
            "output_delta_us": o_ms * 1e3, "output_delta_GB/s": obytes / (o_ms / 1e3) / 1e9,
            "output_delta_frac": obytes / (o_ms / 1e3) / 1e9 / hbm, "output_delta_bytes": obytes}
    res["workload"] = f"{s.name}: {na} agents, n_q*d = {D}, r = {r}; one decode token and a 1024-token chunk per agent"
    res["timing"] = "median of 5 launches, CUDA events, L2 flushed before each"
    return res


def time_other_configs(dev):
    """The long-context batched decode sweep (16 requests x 5 agents, r = 32)
    and one layer of the 32-layer stack (4096-token chunk over a 32768-token
    prefix, 4 agents, r = 64: prefill, then decode over the 36864 keys)."""
    import torch
    from rank_attention_b200 import workloads as W
    res = []
    for ctx in W.SWEEP_CTX:
        res.append(time_decode_shape(dev, W.llama8b_sweep(ctx)))
        torch.cuda.empty_cache()
    pf = time_prefill(dev, s=W.llama8b_stack_prefill(0))
    pf["kind"] = "prefill"
    res.append(pf)
    torch.cuda.empty_cache()
    res.append(time_decode_shape(dev, W.llama8b_stack_decode(0)))
    torch.cuda.empty_cache()
    return res


STACK_STEPS = 16   # decode steps per layer after the chunk's prefill


class StackLayer:
    """One layer of the 32-layer stack workload (4 agents, r = 64, hidden 4096):
    the PreLRShared append of a 4096-token chunk, the prefill of that chunk
    over the 32768-token prefix, then STACK_STEPS decode steps, each appending
    its token's LR row and attending over prefix + chunk + the steps so far.
    Inputs are drawn on the device from the layer's own seed; the base K/V
    rows of the decode tokens are drawn like the cache (the base model's).
    Calls queue on the current stream; tensors live as long as the object."""

    def __init__(self, layer: int, dev, pf_out=None, dec_out=None):
        import torch
        from rank_attention_b200 import lora_attn as la
        from rank_attention_b200 import workloads as W
        s = W.llama8b_stack_prefill(layer)
        self.shape, self.layer = s, layer
        n_pre, n_chunk = s.kv_len - s.n_q_tokens, s.n_q_tokens
        L_max = s.kv_len + STACK_STEPS
        inp = W.direct_cache_inputs(s, device=dev, L_max=L_max)
        g = torch.Generator(device=dev)
        g.manual_seed(s.seed + 500)
        for k in ("k_base", "v_base"):
            inp[k][:, :, s.kv_len:] = (W.CACHE_STD * torch.randn(
                inp[k][:, :, s.kv_len:].shape, generator=g, device=dev)).to(s.dtype)
        ch = W.append_inputs(n_chunk, s.hidden, s.r, s.dtype, seed=s.seed + 600, device=dev)
        xs = W.append_inputs(STACK_STEPS, s.hidden, s.r, s.dtype, seed=s.seed + 700, device=dev)["X"]
        q_dec = (W.CACHE_STD * torch.randn((STACK_STEPS, 1, s.n_agents, 1, s.n_q_heads, s.head_dim),
                                           generator=g, device=dev)).to(s.dtype)
        self.pf_out = pf_out if pf_out is not None else torch.empty(inp["q"].shape, dtype=s.dtype,
                                                                    device=dev)
        self.dec_out = dec_out if dec_out is not None else torch.empty(
            (STACK_STEPS,) + tuple(q_dec.shape[1:]), dtype=torch.float32, device=dev)
        self.kv_lens = [torch.full((1,), s.kv_len + t + 1, dtype=torch.int32, device=dev)
                        for t in range(STACK_STEPS)]
        self.inp, self.chunk, self.xs, self.q_dec = inp, ch, xs, q_dec
        self.n_pre, self.n_chunk = n_pre, n_chunk
        self.pf_args = la.make_args(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"],
                                    inp["q"], self.pf_out, lora_scale=s.lora_scale,
                                    rope_base=s.rope_base, q_pos0=n_pre)
        self.dec_args = [la.make_args(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"],
                                      inp["B_v"], q_dec[t], self.dec_out[t],
                                      lora_scale=s.lora_scale, rope_base=s.rope_base,
                                      kv_len=self.kv_lens[t], max_kv_len=L_max)
                         for t in range(STACK_STEPS)]
        self.ws = la.decode_workspace(self.dec_args[0], dev)

    def append(self, stream=None):
        from rank_attention_b200 import lora_attn as la
        la.lr_cache_append(self.chunk["X"], self.chunk["A_kv"], self.inp["lr"], self.n_pre, stream)

    def prefill(self, stream=None):
        from rank_attention_b200 import lora_attn as la
        la.lora_attn_prefill(self.pf_args, stream)

    def decode_step(self, t: int, stream=None):
        from rank_attention_b200 import lora_attn as la
        la.lr_cache_append(self.xs[:, t:t + 1], self.chunk["A_kv"], self.inp["lr"],
                           self.shape.kv_len + t, stream)
        la.lora_attn_decode(self.dec_args[t], self.ws, stream)

    def run(self, stream=None):
        self.append(stream)
        self.prefill(stream)
        for t in range(STACK_STEPS):
            self.decode_step(t, stream)


def time_stack(dev, reps=3):
    """The full 32-layer stack (append, prefill, STACK_STEPS decode steps per
    layer) in one CUDA graph, and each phase alone over all 32 layers; per-step
    and per-token figures across the 32 layers.  The stack's inputs (about
    11 GB) exceed L2 many times over."""
    import torch
    from rank_attention_b200 import lora_attn as la
    from rank_attention_b200 import workloads as W
    pf_out = dec_out = None
    layers = []
    for l in range(W.STACK_LAYERS):
        layers.append(StackLayer(l, dev, pf_out, dec_out))
        pf_out, dec_out = layers[0].pf_out, layers[0].dec_out   # outputs shared, not read
    st = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()

    def graph(fn):
        with torch.cuda.stream(st):
            fn()   # warm-up, outside the capture
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=st):
            fn()
        return g

    def timed(g):
        ts = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(st):
                e0.record(st)
                g.replay()
                e1.record(st)
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    def all_layers(f):
        def fn():
            for L in layers:
                f(L)
        return fn

    g_all = graph(all_layers(lambda L: L.run(st)))
    g_app = graph(all_layers(lambda L: L.append(st)))
    g_pf = graph(all_layers(lambda L: L.prefill(st)))
    g_dec = graph(all_layers(lambda L: [L.decode_step(t, st) for t in range(STACK_STEPS)]))
    ms_all, ms_app, ms_pf, ms_dec = timed(g_all), timed(g_app), timed(g_pf), timed(g_dec)
    if la.la_device_check() != 0:
        raise RuntimeError("stack device check failed")
    del g_all, g_app, g_pf, g_dec
    s = layers[0].shape
    nl = len(layers)
    base, lora = prefill_flops(s)
    tc, tc_kind = tc_peak()
    hbm, _ = peaks()
    dec_step_ms = ms_dec / STACK_STEPS                        # one decode step, all layers
    kv_mid = s.kv_len + STACK_STEPS // 2
    dshape = s.replace(kv_len=kv_mid, n_q_tokens=1, mode="decode")
    dbytes = decode_bytes(dshape) + append_bytes(dshape, 1)
    abytes = append_bytes(s, s.n_q_tokens)
    res = {
        "workload": f"{nl}-layer stack: per layer append of a {s.n_q_tokens}-token chunk (r = {s.r}), "
                    f"its prefill over {s.kv_len - s.n_q_tokens} + {s.n_q_tokens} keys, "
                    f"{STACK_STEPS} decode steps of {s.n_agents} agents (append + decode)",
        "layers": nl, "decode_steps": STACK_STEPS,
        "stack_ms": ms_all, "append_ms": ms_app, "prefill_ms": ms_pf, "decode_ms": ms_dec,
        "append_per_layer_us": ms_app / nl * 1e3,
        "append_GB/s": abytes * nl / (ms_app / 1e3) / 1e9,
        "append_frac": abytes * nl / (ms_app / 1e3) / 1e9 / hbm,
        "prefill_per_layer_ms": ms_pf / nl,
        "prefill_TFLOP/s": base * nl / (ms_pf / 1e3) / 1e12,
        "prefill_frac": base * nl / (ms_pf / 1e3) / 1e12 / tc,
        "decode_step_all_layers_us": dec_step_ms * 1e3,
        "decode_step_per_layer_us": dec_step_ms / nl * 1e3,
        "decode_agent_tokens_per_s": s.n_agents / (dec_step_ms / 1e3),
        "decode_GB/s": dbytes * nl / (dec_step_ms / 1e3) / 1e9,
        "decode_frac": dbytes * nl / (dec_step_ms / 1e3) / 1e9 / hbm,
        "peaks": {"hbm_GB/s": hbm, "bf16_TFLOP/s": tc, "tc_kind": tc_kind},
        "timing": f"CUDA graphs over all {nl} layers, median of {reps} replays, CUDA events",
        "what": "decode_agent_tokens_per_s: agent tokens through all layers per second "
                "(n_agents / one decode step over the stack); decode bytes: base K, V and LR "
                "read once per layer and step plus the step's append"}
    del layers
    torch.cuda.empty_cache()
    return res


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]),
                "reasons": reasons, "samples": len(rows)}


# DRAM bytes per decode launch from an ncu capture of the workload, keyed by the
# sha256 prefix of the decode kernel's source: reported only while the kernel is
# unchanged since the counters were taken.
DECODE_TRAFFIC = {"e792fb7ef9ab6297": 34422272}


def decode_source_sha() -> str:
    """sha256 prefix of the decode source's code: comments, blank lines and
    trailing spaces removed, so that an edit of the comments keeps the key."""
    import hashlib
    import re
    path = os.path.join(ROOT, "rank_attention_b200", "csrc", "attn_decode_bf16.cu")
    with open(path) as f:
        src = f.read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    code = "\n".join(line.rstrip() for line in src.splitlines() if line.strip())
    return hashlib.sha256(code.encode()).hexdigest()[:16]


def step_kernels_per_call(s) -> int:
    """Kernels one decode step (lora_attn_decode_step) launches: the new LR
    row's append, then the decode's kernels."""
    return 1 + decode_kernels_per_call(s)


def torch_bf16():
    import torch
    return torch.bfloat16


def decode_kernels_per_call(s) -> int:
    """Kernels one lora_attn_decode call launches for this workload.  The
    tensor-core decode (d = 128, r in {16, 32, 64}, agents in groups of up to
    three a CTA) merges its key splits inside the same launch: one kernel.  The
    other bf16 shapes add a split-merge kernel when the keys are split over CTAs."""
    if s.head_dim == 128 and s.r in (16, 32, 64):
        return 1
    units = s.n_seqs * s.n_kv_heads
    splits = 1 if units >= 148 else min(32, 148 // units, (s.kv_len + 127) // 128)
    return 2 if splits > 1 else 1


def run_profile(kind: str = "decode"):
    """A short, deterministic run of one kernel alone, for profilers."""
    import torch
    from rank_attention_b200 import lora_attn as la
    from rank_attention_b200 import workloads as W
    dev = torch.device("cuda", 0)
    if kind == "append":   # one layer of the stack: a 4096-token chunk through r = 64 shared A
        s = W.llama8b_stack_prefill(0)
        inp = W.append_inputs(s.n_q_tokens, s.hidden, s.r, torch.bfloat16, seed=9, device=dev)
        lr = torch.zeros((1, s.kv_len, 2 * s.r), dtype=torch.bfloat16, device=dev)
        for _ in range(3):
            la.lr_cache_append(inp["X"], inp["A_kv"], lr, s.kv_len - s.n_q_tokens)
        torch.cuda.synchronize()
        return 0 if la.la_device_check() == 0 else 1
    if kind == "qkvo":     # query expand and output delta, 1024 tokens per agent
        timed = time_qkvo(dev)
        return 0 if timed else 1
    s = W.LLAMA8B_DECODE_8K if kind == "decode" else W.LLAMA8B_PREFILL_16K
    inp = {k: v.to(dev) for k, v in W.direct_cache_inputs(s, device=dev).items()}
    out = torch.empty(inp["q"].shape, dtype=torch.float32, device=dev)
    if kind == "decode":
        args = la.make_args(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"],
                            inp["q"], out, lora_scale=s.lora_scale, rope_base=s.rope_base,
                            kv_len=inp["kv_len"], max_kv_len=s.kv_len)
        ws = la.decode_workspace(args, dev)
        for _ in range(5):
            la.lora_attn_decode(args, ws)
    else:
        args = la.make_args(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"],
                            inp["q"], out, lora_scale=s.lora_scale, rope_base=s.rope_base,
                            q_pos0=s.q_pos0)
        for _ in range(3):
            la.lora_attn_prefill(args)
    torch.cuda.synchronize()
    return 0 if la.la_device_check() == 0 else 1


def max_over_ranks(x: float, world: int, device) -> float:
    """Maximum of a per-rank scalar over all ranks (every rank gets it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step: int, steps: int, world: int, ms_max: float) -> float:
    """Units processed by all ranks per second, timed by the slowest rank."""
    return units_per_rank_step * steps * world / (ms_max / 1e3)


def decode_bytes(s) -> int:
    """Algorithmic HBM bytes of one decode launch: base K and V read once, the
    LR cache read once (every agent's own with one cache per agent), every
    agent's B_k and B_v, the queries and the fp32 outputs."""
    e = 2  # bf16
    base = 2 * s.n_seqs * s.n_kv_heads * s.kv_len * s.head_dim * e
    lr = s.n_seqs * s.kv_len * 2 * s.r * e * (s.n_agents if s.lr_per_agent else 1)
    Bw = 2 * s.n_agents * s.r * s.n_kv_heads * s.head_dim * e
    q = s.n_seqs * s.n_agents * s.n_q_heads * s.head_dim * e
    out = s.n_seqs * s.n_agents * s.n_q_heads * s.head_dim * 4
    return base + lr + Bw + q + out


CACHE_SCHEMES = ("non_shared", "base_shared", "base_lr_shared")


def kv_cache_bytes(s, scheme: str) -> int:
    """Bytes of the KV caches of one layer that serve all n_agents agents of
    the shape's sequences, at its context length, under a cache-sharing scheme
    (LRAgent summary, §3 Methodology, BaseShared and BaseLRShared):
      non_shared      every agent its own K^a and V^a, each [n_kv][L][d] (the
                      buffers lora_materialize_agent_kv writes);
      base_shared     one base K and V [n_kv][L][d], and every agent its own LR
                      cache X A_a [L][2r] (lr_agent_stride > 0);
      base_lr_shared  one base K and V, and one LR cache X A [L][2r] that all
                      agents read (shared A).
    Counted from the layouts the library reads, per sequence, in bf16."""
    e = 2
    base = 2 * s.n_kv_heads * s.kv_len * s.head_dim * e
    lr = s.kv_len * 2 * s.r * e
    per_seq = {"non_shared": s.n_agents * base,
               "base_shared": base + s.n_agents * lr,
               "base_lr_shared": base + lr}[scheme]
    return s.n_seqs * per_seq


def kv_cache_report(s) -> dict:
    """kv_cache_bytes of every scheme for a shape, and each against non-shared."""
    b = {k: kv_cache_bytes(s, k) for k in CACHE_SCHEMES}
    return {"workload": s.name, "bytes": b,
            "vs_non_shared": {k: b[k] / b["non_shared"] for k in CACHE_SCHEMES}}


def append_bytes(s, n_tok: int) -> int:
    return s.n_seqs * (n_tok * s.hidden * 2 + n_tok * 2 * s.r * 2) + s.hidden * 2 * s.r * 2


def time_oracle_tiny(reps: int = 50) -> dict:
    """The oracle on the tiny fp32 case (one decode step from hidden states:
    base cache, LR rows, attention), on one host thread and on all of them."""
    from threadpoolctl import threadpool_limits
    from oracle import impl as oracle
    from rank_attention_b200 import workloads as W
    s = W.TINY_FP32
    w = W.hidden_layer_weights(s)

    def step():
        kb, vb = oracle.base_cache_from_hidden(w["X"], w["W_k"], w["W_v"], s.n_kv_heads, s.rope_base)
        lr = oracle.lr_cache_rows(w["X"], w["A_kv"])
        oracle.lora_attention(kb, vb, lr, w["B_k"], w["B_v"], w["q"], [s.kv_len],
                              lora_scale=s.lora_scale, softmax_scale=s.softmax_scale,
                              rope_base=s.rope_base, mode="decode")

    res = {"workload": s.name}
    for label, limit in (("one_thread", 1), ("all_threads", None)):
        with threadpool_limits(limits=limit):
            step()
            t0 = time.perf_counter()
            for _ in range(reps):
                step()
            per = (time.perf_counter() - t0) / reps
        res[label] = {"ms_per_step": per * 1e3,
                      "agent_tokens_per_s": s.n_seqs * s.n_agents / per}
    res["cores_all"] = blas_threads()
    return res


def oracle_step(inp, new, s):
    """One decode step on the fp64 oracle: append the new LR row, then attend."""
    from oracle import impl as oracle
    lr = oracle.lr_cache_append(inp["lr"], new["X"], new["A_kv"], s.kv_len - 1)
    return oracle.lora_attention(inp["k_base"], inp["v_base"], lr, inp["B_k"], inp["B_v"],
                                 inp["q"], inp["kv_len"], lora_scale=s.lora_scale,
                                 softmax_scale=s.softmax_scale, rope_base=s.rope_base,
                                 mode="decode")


def time_oracle_samples(budget_s: float = 10.0) -> dict:
    """The oracle on bounded samples of the prefill and the 32k sweep: one
    (agent, KV head) unit each, scaled by the units of a whole launch."""
    import numpy as np
    from oracle import impl as oracle
    from rank_attention_b200 import workloads as W
    res = {}
    # prefill, 16384 + 1024: the last 64 chunk tokens of one unit (its K^a and V^a
    # over all 17408 keys materialised, then their attention)
    s = W.LLAMA8B_PREFILL_16K
    inp = W.direct_cache_inputs(s)
    g = s.n_q_heads // s.n_kv_heads
    toks = list(range(s.n_q_tokens - 64, s.n_q_tokens))
    qpos = s.q_pos0 + np.arange(s.n_q_tokens)
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle.lora_attention_unit(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"],
                                   inp["q"], seq=0, agent=0, kv_head=0, kv_len=s.kv_len,
                                   q_positions=qpos, lora_scale=s.lora_scale,
                                   softmax_scale=s.softmax_scale, rope_base=s.rope_base,
                                   q_tokens=toks)
        n += 1
        if time.perf_counter() - t0 > budget_s / 2:
            break
    per = (time.perf_counter() - t0) / n
    pairs = g * sum(int(qpos[j]) + 1 for j in toks)
    res["prefill"] = {"workload": s.name, "TFLOP/s": 4 * s.head_dim * pairs / per / 1e12,
                      "sample": f"one (agent, KV head) unit, the last {len(toks)} chunk tokens x "
                                f"{g} heads over all {s.kv_len} keys, {n} runs"}
    # decode sweep at 32k: one (sequence, agent, KV head) unit of the 16 x 5 x 8
    s = W.llama8b_sweep(32768).replace(n_seqs=1)
    inp = W.direct_cache_inputs(s)
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle.lora_attention_unit(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"],
                                   inp["q"], seq=0, agent=0, kv_head=0, kv_len=s.kv_len,
                                   q_positions=[s.kv_len - 1], lora_scale=s.lora_scale,
                                   softmax_scale=s.softmax_scale, rope_base=s.rope_base)
        n += 1
        if time.perf_counter() - t0 > budget_s / 2:
            break
    per = (time.perf_counter() - t0) / n
    units = 16 * s.n_agents * s.n_kv_heads
    res["sweep_32k"] = {"workload": W.llama8b_sweep(32768).name,
                        "agent_tokens_per_s": 16 * s.n_agents / (per * units),
                        "sample": f"one (sequence, agent, KV head) unit of {units}, {n} runs, "
                                  "scaled by the units of a step"}
    return res


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def time_oracle(s, steps: int, budget_s: float):
    """Time the oracle's decode step; at most `steps` steps or `budget_s` seconds."""
    from rank_attention_b200 import workloads as W
    inp = W.direct_cache_inputs(s)
    new = W.append_inputs(1, s.hidden, s.r, s.dtype, seed=s.seed + 100, n_seqs=s.n_seqs)
    times = []
    t_all = time.perf_counter()
    for _ in range(max(1, steps)):
        t0 = time.perf_counter()
        oracle_step(inp, new, s)
        times.append(time.perf_counter() - t0)
        if time.perf_counter() - t_all > budget_s:
            break
    per = sum(times) / len(times)
    return s.n_seqs * s.n_agents / per, len(times), per


def step_config(s, world: int) -> dict:
    """The `config` of the JSON line, identical for both arms: the workload, the
    step, how the inputs exceed L2 and how the step is timed."""
    step_bytes = decode_bytes(s) + append_bytes(s, 1)
    n_sets = max(2, math.ceil(2 * L2_BYTES / step_bytes))
    return {"workload": s.name, "kv_len": s.kv_len, "agents": s.n_agents, "r": s.r,
            "step": "lora_attn_decode_step: the new token's LR row and the decode",
            "l2": f"inputs larger than L2: {n_sets} rotating cache sets of "
                  f"{step_bytes / 1e6:.1f} MB ({n_sets * step_bytes / 1e6:.0f} MB > 126 MB)",
            "timing": "CUDA graphs of the steps, CUDA events on the launch stream",
            "parallelism": f"replicas x{world}"}


def run_reference(args):
    """The reference arm: the fp64 oracle on the host cores (rank 0 only), each
    step one whole decode step of the workload (LR append of the new token,
    then every agent's materialised attention), as the GPU arm's step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from rank_attention_b200 import workloads as W
    s = W.LLAMA8B_DECODE_8K
    inp = W.direct_cache_inputs(s)
    new = W.append_inputs(1, s.hidden, s.r, s.dtype, seed=s.seed + 100, n_seqs=s.n_seqs)
    for _ in range(args.warmup):
        oracle_step(inp, new, s)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(inp, new, s)
    full_step = (time.perf_counter() - t0) / args.steps
    value = s.n_seqs * s.n_agents / full_step
    cores = blas_threads()
    sample = (f"{args.steps} whole decode steps of {s.name} on the host (append of the new "
              f"token's LR row, then all {s.n_agents * s.n_kv_heads} (agent, KV head) units' "
              f"materialised attention), after {args.warmup} untimed")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": full_step * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": step_config(s, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch
    import torch.distributed as dist

    from rank_attention_b200 import lora_attn as la
    from rank_attention_b200 import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    s = W.LLAMA8B_DECODE_8K
    step_bytes = decode_bytes(s) + append_bytes(s, 1)
    n_sets = max(2, math.ceil(2 * L2_BYTES / step_bytes))
    sets, steps_fn = [], []
    A_kv = W.append_inputs(1, s.hidden, s.r, s.dtype, seed=s.seed + 100)["A_kv"].to(dev)
    for i in range(n_sets):
        si = s.replace(seed=s.seed + 1000 * (rank + 1) + i)
        inp = {k: v.to(dev) for k, v in W.direct_cache_inputs(si, device=dev).items()}
        x0 = W.append_inputs(1, s.hidden, s.r, s.dtype, seed=si.seed + 7, device=dev)["X"]
        # the step's inputs back to back in one device buffer (one H2D copy a step)
        _, x_new, q, kv_len = la.packed_step_inputs(x0.shape, inp["q"].shape, s.n_seqs, s.dtype,
                                                    dev)
        x_new.copy_(x0)
        q.copy_(inp["q"])
        kv_len.copy_(inp["kv_len"])
        inp["q"], inp["kv_len"] = q, kv_len
        out = torch.empty(inp["q"].shape, dtype=torch.float32, device=dev)
        st = la.DecodeStep(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"],
                           inp["q"], out, inp["kv_len"], lora_scale=s.lora_scale,
                           rope_base=s.rope_base, max_kv_len=s.kv_len, A_kv=A_kv, x_new=x_new)
        sets.append((inp, x_new, out))
        steps_fn.append(st)

    stream = torch.cuda.Stream(device=dev)
    torch.cuda.synchronize()
    # warm-up (eager), then capture CUDA graphs of whole rotations over the sets
    with torch.cuda.stream(stream):
        for k in range(args.warmup):
            steps_fn[k % n_sets]()
    torch.cuda.synchronize()

    def capture(fns):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for f in fns:
                f()
        return g

    full, rem = divmod(args.steps, n_sets)
    g_rot = capture(steps_fn) if full else None
    g_rem = capture(steps_fn[:rem]) if rem else None
    # decode kernel alone, for the roofline of the dominant kernel
    reps = max(1, 64 // n_sets)
    dec_fns = [(lambda st=st: la.lora_attn_decode(st.args, st.workspace)) for st in steps_fn]
    g_dec = capture(dec_fns * reps)
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()


    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(full):
            g_rot.replay()
        if g_rem is not None:
            g_rem.replay()
        ev1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dev)
    # decode kernel alone: one untimed replay, then the median of five
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dec_times = []
    with torch.cuda.stream(stream):
        g_dec.replay()
        for _ in range(5):
            d0.record(stream)
            g_dec.replay()
            d1.record(stream)
            d1.synchronize()
            dec_times.append(d0.elapsed_time(d1))
    torch.cuda.synchronize()
    clk = clocks.stop()
    dec_ms = sorted(dec_times)[2] / (n_sets * reps)

    value = whole_job_rate(s.n_seqs * s.n_agents, args.steps, world, ms)

    # end to end through the public API with host buffers: lora_decode_step_host
    # copies the step's inputs in (new hidden row, queries, lengths), appends,
    # decodes and copies the outputs back
    h_x, h_q, h_len = [], [], []
    for (i, x, _) in sets:  # pinned, back to back as on the device
        _, hx, hq, hl = la.packed_step_inputs(x.shape, i["q"].shape, s.n_seqs, s.dtype, "cpu",
                                              pin=True)
        hx.copy_(x)
        hq.copy_(i["q"])
        hl.copy_(i["kv_len"])
        h_x.append(hx)
        h_q.append(hq)
        h_len.append(hl)
    h_out = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for (_, _, o) in sets]
    h2d = h_x[0].numel() * 2 + h_q[0].numel() * 2 + h_len[0].numel() * 4
    d2h = h_out[0].numel() * 4
    e_steps = min(args.steps, 100)

    def e2e_step(k):  # one library call: copies in, append, decode, copy out
        i = k % n_sets
        steps_fn[i].from_host(h_x[i], h_q[i], h_len[i], h_out[i], stream)

    with torch.cuda.stream(stream):
        for k in range(3):
            e2e_step(k)
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for k in range(e_steps):
            e2e_step(k)
        e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = whole_job_rate(s.n_seqs * s.n_agents, e_steps, world, e_ms)

    prefill = time_prefill(dev)
    non_shared = time_non_shared(dev, dec_ms * 1e3)
    base_shared = time_base_shared(dev)
    qkvo = time_qkvo(dev)
    value_ablation = time_value_ablation(dev, prefill)

    hbm, peak_kind = peaks()
    dbytes = decode_bytes(s)
    achieved = dbytes / (dec_ms / 1e3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": step_config(s, world),
        "roofline": {"kernel": "lora_attn_decode", "bound": "hbm", "achieved": achieved,
                     "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                     "peak_kind": f"{peak_kind} copy bandwidth",
                     "algorithmic_bytes_per_launch": dbytes, "launch_us": dec_ms * 1e3,
                     "traffic": DECODE_TRAFFIC.get(decode_source_sha()),
                     "frac_of_nominal": achieved / NOMINAL_HBM_GBS,
                     "nominal_peak": NOMINAL_HBM_GBS},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e_steps},
        "gpu_launches": step_kernels_per_call(s) * args.steps,
        "clocks": clk,
        "prefill": prefill,
        "non_shared_baseline": non_shared,
        "kv_cache_memory": kv_cache_report(s),
        "base_shared": base_shared,
        "qkvo": qkvo,
        "value_ablation": value_ablation,
    }
    line["other_configs"] = time_other_configs(dev)
    line["stack"] = time_stack(dev)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, n, per = time_oracle(s, 20, 15.0)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": blas_threads(),
                                "kind": "oracle",
                                "sample": f"{n} full decode steps of {s.name} on the host",
                                "tiny_fp32": time_oracle_tiny(),
                                "other_configs": time_oracle_samples()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        del g_rot, g_rem, g_dec
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.profile:
        return run_profile(args.profile)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
