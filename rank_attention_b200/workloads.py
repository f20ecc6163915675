"""Seeded synthetic workloads for Flash-LoRA-Attention.

This module only draws random tensors and describes shapes.  It holds none of
the method's arithmetic (no RoPE, no projections, no attention), so both the
CUDA path and the fp64 oracle can take their inputs from it.

The shapes follow the workloads the LRAgent and PReCache pages evaluate on:
LLaMA-3.1-8B-Instruct attention layers (hidden 4096, 32 query / 8 KV heads,
head_dim 128) with three role agents (plan / action / reflect) sharing one
trajectory, LoRA ranks 1..32, and context lengths from 0.25k up to 66.4k
tokens (LRAgent summary on paperlayer.ai, §4 Models and Datasets, App. C.6
Emulated Trace, App. D.4 Rank Ablations).  The pages measure on HotpotQA and
ScienceQA trajectories with trained adapters; seeded Gaussian tensors of the
same shapes stand in for them.

Value distributions:
* hidden states X: Gaussian rows scaled to unit RMS;
* W_k, W_v, A, B: N(0, 0.02) for the LLaMA-shaped cases, N(0,1)/sqrt(fan_in)
  for the tiny fp32 case;
* base K/V and the LR cache of the LLaMA-shaped cases are drawn directly with
  the standard deviation of X.W at unit-RMS X and N(0, 0.02) weights over
  hidden 4096, i.e. 0.02 * sqrt(4096) = 1.28 (the base keys are treated as
  already rotated);
* queries: N(0, 1) for the tiny case, N(0, 1.28^2) otherwise.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class AttnShape:
    """Shape of one Flash-LoRA-Attention problem (one layer)."""

    name: str
    n_seqs: int          # independent sequences (requests), each with its own caches
    n_agents: int        # agents (LoRA adapters with their own B) sharing each cache
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    hidden: int
    r: int               # LoRA rank
    alpha: float         # LoRA alpha; s = alpha / r
    rope_base: float
    kv_len: int          # cached tokens per sequence (decode) / prefix + chunk (prefill)
    n_q_tokens: int      # 1 for decode; chunk length for prefill
    dtype: torch.dtype   # storage dtype of caches, weights and queries
    seed: int
    mode: str            # "decode" or "prefill"
    lr_per_agent: bool = False   # one LR cache per agent (own A_a: BaseShared) instead of one shared

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def lora_scale(self) -> float:
        return self.alpha / self.r

    @property
    def softmax_scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def q_pos0(self) -> int:
        """Position of the first query token (decode: the last cached token)."""
        return self.kv_len - self.n_q_tokens

    def replace(self, **kw) -> "AttnShape":
        return dataclasses.replace(self, **kw)


# The workloads.  Names say what they are; sizes are in the fields.
TINY_FP32 = AttnShape(
    name="tiny_fp32_decode", n_seqs=1, n_agents=2, n_q_heads=4, n_kv_heads=2,
    head_dim=64, hidden=256, r=8, alpha=16.0, rope_base=10000.0, kv_len=256,
    n_q_tokens=1, dtype=torch.float32, seed=0, mode="decode")

LLAMA8B_DECODE_8K = AttnShape(
    name="llama8b_decode_ctx8192_3agents_r16", n_seqs=1, n_agents=3, n_q_heads=32,
    n_kv_heads=8, head_dim=128, hidden=4096, r=16, alpha=32.0, rope_base=500000.0,
    kv_len=8192, n_q_tokens=1, dtype=torch.bfloat16, seed=1, mode="decode")

LLAMA8B_PREFILL_16K = AttnShape(
    name="llama8b_prefill_prefix16384_chunk1024_3agents_r16", n_seqs=1, n_agents=3,
    n_q_heads=32, n_kv_heads=8, head_dim=128, hidden=4096, r=16, alpha=32.0,
    rope_base=500000.0, kv_len=16384 + 1024, n_q_tokens=1024, dtype=torch.bfloat16,
    seed=2, mode="prefill")


def llama8b_sweep(ctx: int) -> AttnShape:
    """Batched long-context decode: 16 requests x 5 agents, r=32."""
    return AttnShape(
        name=f"llama8b_decode_ctx{ctx}_16req_5agents_r32", n_seqs=16, n_agents=5,
        n_q_heads=32, n_kv_heads=8, head_dim=128, hidden=4096, r=32, alpha=64.0,
        rope_base=500000.0, kv_len=ctx, n_q_tokens=1, dtype=torch.bfloat16, seed=3,
        mode="decode")


SWEEP_CTX = (32768, 65536, 131072)

# 32-layer stack: append of a 4096-token chunk through r=64 shared A, then
# prefill of that chunk over a 32768-token prefix and decode, 4 agents.
STACK_LAYERS = 32


def llama8b_stack_prefill(layer: int) -> AttnShape:
    return AttnShape(
        name=f"llama8b_stack_layer{layer}_prefill_prefix32768_chunk4096_4agents_r64",
        n_seqs=1, n_agents=4, n_q_heads=32, n_kv_heads=8, head_dim=128, hidden=4096,
        r=64, alpha=128.0, rope_base=500000.0, kv_len=32768 + 4096, n_q_tokens=4096,
        dtype=torch.bfloat16, seed=4 + 1000 * layer, mode="prefill")


def llama8b_stack_decode(layer: int) -> AttnShape:
    return llama8b_stack_prefill(layer).replace(
        name=f"llama8b_stack_layer{layer}_decode_ctx36864_4agents_r64", n_q_tokens=1,
        mode="decode")


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, std, dtype, gen, device) -> torch.Tensor:
    t = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def unit_rms_rows(shape, dtype, gen, device) -> torch.Tensor:
    """Gaussian rows rescaled to unit root-mean-square (hidden states)."""
    t = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
    t.mul_(torch.rsqrt(t.pow(2).mean(dim=-1, keepdim=True)))
    return t.to(dtype)


def hidden_layer_weights(shape: AttnShape, device="cpu") -> Dict[str, torch.Tensor]:
    """X, W_k, W_v, A_kv = [A_k | A_v] and per-agent B_k, B_v for a hidden-state case.

    Used by the tiny case, where the base cache is derived from X.
    Layouts: X [n_seqs, kv_len, hidden]; W_k, W_v [hidden, n_kv*d];
    A_kv [hidden, 2r] (A_k columns first); B_k, B_v [n_agents, r, n_kv*d].
    """
    g = _gen(shape.seed, device)
    H, r, dkv = shape.hidden, shape.r, shape.n_kv_heads * shape.head_dim
    if shape.dtype == torch.float32:
        w_std, a_std, b_std = 1.0 / math.sqrt(H), 1.0 / math.sqrt(H), 1.0 / math.sqrt(r)
        X = _normal((shape.n_seqs, shape.kv_len, H), 1.0, shape.dtype, g, device)
    else:
        w_std = a_std = b_std = 0.02
        X = unit_rms_rows((shape.n_seqs, shape.kv_len, H), shape.dtype, g, device)
    W_k = _normal((H, dkv), w_std, shape.dtype, g, device)
    W_v = _normal((H, dkv), w_std, shape.dtype, g, device)
    A_kv = _normal((H, 2 * r), a_std, shape.dtype, g, device)
    B_k = _normal((shape.n_agents, r, dkv), b_std, shape.dtype, g, device)
    B_v = _normal((shape.n_agents, r, dkv), b_std, shape.dtype, g, device)
    q = _normal((shape.n_seqs, shape.n_agents, shape.n_q_tokens, shape.n_q_heads,
                 shape.head_dim), 1.0, shape.dtype, g, device)
    return dict(X=X, W_k=W_k, W_v=W_v, A_kv=A_kv, B_k=B_k, B_v=B_v, q=q)


CACHE_STD = 0.02 * math.sqrt(4096)   # std of X.W for unit-RMS X and N(0, 0.02) W


def direct_cache_inputs(shape: AttnShape, device="cpu", L_max: Optional[int] = None,
                        with_lora: bool = True) -> Dict[str, torch.Tensor]:
    """Base K/V, LR cache, B_k, B_v and queries drawn directly (LLaMA-shaped cases).

    Layouts: k_base, v_base [n_seqs, n_kv, L_max, d]; lr [n_seqs, L_max, 2r]
    (LR_k columns first), or [n_agents, n_seqs, L_max, 2r] with
    shape.lr_per_agent (agent a's cache drawn after agent a-1's);
    B_k, B_v [n_agents, r, n_kv*d];
    q [n_seqs, n_agents, n_q_tokens, n_q_heads, d]; kv_len int32 [n_seqs].
    Rows at or beyond kv_len are left at zero.
    """
    L_max = shape.kv_len if L_max is None else L_max
    g = _gen(shape.seed, device)
    d, r, n_kv = shape.head_dim, shape.r, shape.n_kv_heads
    dt = shape.dtype
    k_base = torch.zeros((shape.n_seqs, n_kv, L_max, d), dtype=dt, device=device)
    v_base = torch.zeros_like(k_base)
    n_lr = shape.n_agents if shape.lr_per_agent else 1
    lr = torch.zeros((n_lr, shape.n_seqs, L_max, 2 * r), dtype=dt, device=device)
    L = shape.kv_len
    k_base[:, :, :L] = _normal((shape.n_seqs, n_kv, L, d), CACHE_STD, dt, g, device)
    v_base[:, :, :L] = _normal((shape.n_seqs, n_kv, L, d), CACHE_STD, dt, g, device)
    for a in range(n_lr):
        lr[a, :, :L] = _normal((shape.n_seqs, L, 2 * r), CACHE_STD, dt, g, device)
    if not shape.lr_per_agent:
        lr = lr[0]
    b_std = 0.02 if with_lora else 0.0
    B_k = _normal((shape.n_agents, r, n_kv * d), b_std, dt, g, device)
    B_v = _normal((shape.n_agents, r, n_kv * d), b_std, dt, g, device)
    q = _normal((shape.n_seqs, shape.n_agents, shape.n_q_tokens, shape.n_q_heads, d),
                CACHE_STD, dt, g, device)
    kv_len = torch.full((shape.n_seqs,), L, dtype=torch.int32, device=device)
    return dict(k_base=k_base, v_base=v_base, lr=lr, B_k=B_k, B_v=B_v, q=q, kv_len=kv_len)


def append_inputs(n_tokens: int, hidden: int, r: int, dtype: torch.dtype, seed: int,
                  n_seqs: int = 1, device="cpu") -> Dict[str, torch.Tensor]:
    """Hidden-state chunk X [n_seqs, n_tokens, hidden] and shared A_kv [hidden, 2r]."""
    g = _gen(seed, device)
    X = unit_rms_rows((n_seqs, n_tokens, hidden), dtype, g, device)
    a_std = 0.02 if dtype != torch.float32 else 1.0 / math.sqrt(hidden)
    A_kv = _normal((hidden, 2 * r), a_std, dtype, g, device)
    return dict(X=X, A_kv=A_kv)
