"""Shared helpers of the parity tests: tolerances and oracle/CUDA runners."""
import math

import numpy as np
import torch

from oracle import impl as oracle

# Tolerances of the parity bar:
#   fp32 inputs:                max|err| <= 1e-4 * max|ref|
#   bf16 storage, fp32 accumulate: max|err| <= 1e-2 * max|ref|, mean|err| <= 1e-3 * max|ref|
FP32_MAX_REL = 1e-4
BF16_MAX_REL = 1e-2
BF16_MEAN_REL = 1e-3


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), "non-finite output"
    scale = np.abs(ref).max()
    err = np.abs(got - ref)
    return err.max() / scale, err.mean() / scale


def assert_parity(got, ref, dtype):
    mx, mean = errors(got, ref)
    if dtype == torch.float32:
        assert mx <= FP32_MAX_REL, f"max rel err {mx:.3e} > {FP32_MAX_REL}"
    else:
        assert mx <= BF16_MAX_REL, f"max rel err {mx:.3e} > {BF16_MAX_REL}"
        assert mean <= BF16_MEAN_REL, f"mean rel err {mean:.3e} > {BF16_MEAN_REL}"
    return mx, mean


def to_np(t):
    return t.detach().to("cpu", torch.float64).numpy()


def bf16_ulp(x):
    """Spacing of bf16 numbers at |x| (8 significant bits)."""
    ax = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    return np.where(ax > 0, 2.0 ** (e - 7), 2.0 ** -133)


def oracle_decode(inp, shape, lr=None):
    """Oracle outputs of a decode over the inputs' caches (fp64)."""
    return oracle.lora_attention(
        inp["k_base"], inp["v_base"], inp["lr"] if lr is None else lr, inp["B_k"], inp["B_v"],
        inp["q"], inp["kv_len"].cpu(), lora_scale=shape.lora_scale,
        softmax_scale=shape.softmax_scale, rope_base=shape.rope_base, mode="decode")


def to_device(inp, device="cuda"):
    return {k: v.to(device) for k, v in inp.items()}
