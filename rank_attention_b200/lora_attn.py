"""Python binding of liblora_attn.so (ctypes; argument marshalling only).

The names match the C ABI in include/lora_attn.h.  Tensors are torch CUDA
tensors; the binding passes their data pointers, sizes and strides, and the
current torch stream.  Every step of the computation runs in the library's
CUDA kernels.  If the compiled library is missing, importing this module
raises: there is no fallback.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "liblora_attn.so")

LA_OK, LA_ERR_INVALID_ARG, LA_ERR_UNSUPPORTED, LA_ERR_CAPACITY = 0, 1, 2, 3
LA_ERR_WORKSPACE, LA_ERR_CUDA, LA_ERR_DEVICE_CHECK, LA_ERR_SCRATCH_LIMIT = 4, 5, 6, 7
LA_STATIC_SCRATCH_BYTES = 4 << 20
LA_F32, LA_BF16 = 0, 1
LA_VALUE_REORDERED, LA_VALUE_REORDERED_GENERIC, LA_VALUE_PER_TILE, LA_VALUE_PER_TILE_GENERIC = 0, 1, 2, 3
LA_DEV_KV_LEN, LA_DEV_PIPE_WAIT, LA_DEV_MERGE_WAIT = 1, 2, 4

EXPORTED = ("la_status_string", "lr_cache_append", "lora_attn_prefill", "lora_attn_decode",
            "lora_attn_decode_workspace_bytes", "la_device_check",
            "lora_attn_decode_static_scratch", "lora_materialize_agent_kv",
            "lr_cache_append_agents", "lora_query_expand", "lora_output_delta",
            "la_device_check_word", "lora_decode_step_host", "lora_attn_decode_step",
            "lora_attn_decode_combine")


class LoraAttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


class AttnArgs(ctypes.Structure):
    """Mirror of la_attn_args."""

    _fields_ = [
        ("n_seqs", ctypes.c_int32), ("n_agents", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("r", ctypes.c_int32),
        ("lora_scale", ctypes.c_float), ("softmax_scale", ctypes.c_float),
        ("rope_base", ctypes.c_double),
        ("L_max", ctypes.c_int64),
        ("k_base", ctypes.c_void_p), ("v_base", ctypes.c_void_p),
        ("kv_seq_stride", ctypes.c_int64), ("kv_head_stride", ctypes.c_int64),
        ("kv_tok_stride", ctypes.c_int64),
        ("lr_cache", ctypes.c_void_p), ("lr_seq_stride", ctypes.c_int64),
        ("B_k", ctypes.c_void_p), ("B_v", ctypes.c_void_p),
        ("q", ctypes.c_void_p), ("out", ctypes.c_void_p),
        ("kv_len", ctypes.c_void_p),
        ("max_kv_len", ctypes.c_int64),
        ("q_pos0", ctypes.c_int64),
        ("n_q_tokens", ctypes.c_int32),
        ("io_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
        ("lr_agent_stride", ctypes.c_int64),
        ("value_path", ctypes.c_int32),
        ("key_pos0", ctypes.c_int64),
        ("row_stats", ctypes.c_void_p),
    ]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"liblora_attn.so is not built ({LIB_PATH}); run "
                          "python -m rank_attention_b200.build_lib")
    lib = ctypes.CDLL(LIB_PATH)
    lib.la_status_string.restype = ctypes.c_char_p
    lib.la_status_string.argtypes = [ctypes.c_int]
    lib.lr_cache_append.restype = ctypes.c_int
    lib.lr_cache_append.argtypes = [
        ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
        ctypes.c_int32, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
        ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p]
    lib.lr_cache_append_agents.restype = ctypes.c_int
    lib.lr_cache_append_agents.argtypes = [
        ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p,
        ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
        ctypes.c_int64, ctypes.c_int32, ctypes.c_int64, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p]
    lib.lora_query_expand.restype = ctypes.c_int
    lib.lora_query_expand.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
        ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
        ctypes.c_float, ctypes.c_double, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
    lib.lora_output_delta.restype = ctypes.c_int
    lib.lora_output_delta.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
        ctypes.c_int32, ctypes.c_float, ctypes.c_int, ctypes.c_void_p]
    lib.lora_attn_prefill.restype = ctypes.c_int
    lib.lora_attn_prefill.argtypes = [ctypes.POINTER(AttnArgs), ctypes.c_void_p]
    lib.lora_attn_decode.restype = ctypes.c_int
    lib.lora_attn_decode.argtypes = [ctypes.POINTER(AttnArgs), ctypes.c_void_p, ctypes.c_size_t,
                                     ctypes.c_void_p]
    lib.lora_attn_decode_workspace_bytes.restype = ctypes.c_size_t
    lib.lora_attn_decode_workspace_bytes.argtypes = [ctypes.POINTER(AttnArgs)]
    lib.la_device_check.restype = ctypes.c_int
    lib.la_device_check.argtypes = []
    lib.la_device_check_word.restype = ctypes.c_int
    lib.lora_decode_step_host.restype = ctypes.c_int
    lib.lora_decode_step_host.argtypes = [
        ctypes.POINTER(AttnArgs), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
        ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_void_p, ctypes.c_void_p]
    lib.la_device_check_word.argtypes = [ctypes.POINTER(ctypes.c_int32)]
    lib.lora_attn_decode_step.restype = ctypes.c_int
    lib.lora_attn_decode_step.argtypes = [ctypes.POINTER(AttnArgs), ctypes.c_void_p, ctypes.c_void_p,
                                          ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t,
                                          ctypes.c_void_p]
    lib.lora_attn_decode_static_scratch.restype = ctypes.c_int
    lib.lora_attn_decode_static_scratch.argtypes = [ctypes.POINTER(AttnArgs), ctypes.c_void_p]
    lib.lora_materialize_agent_kv.restype = ctypes.c_int
    lib.lora_materialize_agent_kv.argtypes = [ctypes.POINTER(AttnArgs), ctypes.c_void_p,
                                              ctypes.c_void_p, ctypes.c_void_p]
    lib.lora_attn_decode_combine.restype = ctypes.c_int
    lib.lora_attn_decode_combine.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int32,
                                             ctypes.c_int64, ctypes.c_int32, ctypes.c_int,
                                             ctypes.c_void_p, ctypes.c_void_p]
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.la_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != LA_OK:
        raise LoraAttnError(status, where)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return LA_F32
    if t.dtype == torch.bfloat16:
        return LA_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def lr_cache_append(X: torch.Tensor, A_kv: torch.Tensor, lr_cache: torch.Tensor, pos0: int,
                    stream=None) -> None:
    """lr_cache[:, pos0:pos0+n] = X @ A_kv.

    X [n_seqs, n, H] (last dim contiguous), A_kv [H, 2r] contiguous,
    lr_cache [n_seqs, L_max, 2r] (last two dims contiguous)."""
    n_seqs, n, H = X.shape
    r = A_kv.shape[1] // 2
    assert X.stride(2) == 1 and A_kv.is_contiguous()
    assert lr_cache.stride(2) == 1 and lr_cache.stride(1) == 2 * r
    st = lib.lr_cache_append(X.data_ptr(), X.stride(1), n, H, A_kv.data_ptr(), r,
                             lr_cache.data_ptr(), lr_cache.shape[1], pos0, n_seqs, X.stride(0),
                             lr_cache.stride(0), _dt(X), _stream(stream))
    _check(st, "lr_cache_append")


def lr_cache_append_agents(X: torch.Tensor, A_kv: torch.Tensor, lr_cache: torch.Tensor,
                           pos0: int, stream=None) -> None:
    """lr_cache[a, :, pos0:pos0+n] = X @ A_kv[a] for every agent a.

    X [n_seqs, n, H] (last dim contiguous), A_kv [n_agents, H, 2r] contiguous,
    lr_cache [n_agents, n_seqs, L_max, 2r] (last two dims contiguous)."""
    n_seqs, n, H = X.shape
    n_agents, r = A_kv.shape[0], A_kv.shape[2] // 2
    assert X.stride(2) == 1 and A_kv.is_contiguous()
    assert lr_cache.stride(3) == 1 and lr_cache.stride(2) == 2 * r
    st = lib.lr_cache_append_agents(X.data_ptr(), X.stride(1), n, H, A_kv.data_ptr(), n_agents, r,
                                    lr_cache.data_ptr(), lr_cache.stride(0), lr_cache.shape[2],
                                    pos0, n_seqs, X.stride(0), lr_cache.stride(1), _dt(X),
                                    _stream(stream))
    _check(st, "lr_cache_append_agents")


def lora_query_expand(q_base: torch.Tensor, lr_q: torch.Tensor, B_q: torch.Tensor,
                      q_out: torch.Tensor, pos_end: torch.Tensor, *, lora_scale: float,
                      rope_base: float, stream=None) -> None:
    """q_out = RoPE(q_base + s lr_q B_q^a) per agent and head.

    q_base, q_out [n_seqs, n_agents, n_tok, n_q, d] contiguous (may be the same
    tensor); lr_q [n_seqs, n_agents, n_tok, r]; B_q [n_agents, r, n_q*d];
    pos_end int32 [n_seqs]: token j sits at pos_end - n_tok + j."""
    n_seqs, n_agents, n_tok, n_q, d = q_base.shape
    r = lr_q.shape[-1]
    assert q_base.is_contiguous() and q_out.is_contiguous() and lr_q.is_contiguous()
    assert B_q.is_contiguous() and pos_end.dtype == torch.int32
    st = lib.lora_query_expand(q_base.data_ptr(), lr_q.data_ptr(), B_q.data_ptr(),
                               q_out.data_ptr(), n_seqs, n_agents, n_tok, n_q, d, r, lora_scale,
                               rope_base, pos_end.data_ptr(), _dt(q_base), _stream(stream))
    _check(st, "lora_query_expand")


def lora_output_delta(o: torch.Tensor, A_o: torch.Tensor, B_o: torch.Tensor, y: torch.Tensor, *,
                      lora_scale: float, stream=None) -> None:
    """y += s (o A_o) B_o^a per agent.

    o [n_seqs, n_agents, n_tok, d_in]; A_o [d_in, r] shared, or [n_agents, d_in, r];
    B_o [n_agents, r, d_out]; y [n_seqs, n_agents, n_tok, d_out]; all contiguous."""
    n_seqs, n_agents, n_tok, d_in = o.shape
    r, d_out = B_o.shape[1], B_o.shape[2]
    a_stride = A_o.stride(0) if A_o.dim() == 3 else 0
    assert o.is_contiguous() and A_o.is_contiguous() and B_o.is_contiguous() and y.is_contiguous()
    st = lib.lora_output_delta(o.data_ptr(), A_o.data_ptr(), a_stride, B_o.data_ptr(), y.data_ptr(),
                               n_seqs, n_agents, n_tok, d_in, d_out, r, lora_scale, _dt(o),
                               _stream(stream))
    _check(st, "lora_output_delta")


def make_args(k_base, v_base, lr, B_k, B_v, q, out, *, lora_scale: float, rope_base: float,
              softmax_scale: Optional[float] = None, kv_len: Optional[torch.Tensor] = None,
              max_kv_len: int = 0, q_pos0: int = 0, value_path: int = LA_VALUE_REORDERED,
              key_pos0: int = 0, row_stats: Optional[torch.Tensor] = None) -> AttnArgs:
    """Fill la_attn_args from tensors.

    k_base, v_base [n_seqs, n_kv, L_max, d] (any strides with a unit last
    stride); lr [n_seqs, L_max, 2r], one LR cache shared by every agent, or
    [n_agents, n_seqs, L_max, 2r], one per agent; B_k, B_v [n_agents, r, n_kv*d];
    q, out [n_seqs, n_agents, n_tok, n_q, d] contiguous; kv_len int32 [n_seqs].
    Sequence-sharded decode: key_pos0 is the position of the caches' key row 0;
    row_stats a float32 [n_seqs, n_agents, n_q, 2] tensor the decode fills
    with each row's (M, L) for lora_attn_decode_combine."""
    n_seqs, n_kv, L_max, d = k_base.shape
    n_agents, n_tok, n_q = q.shape[1], q.shape[2], q.shape[3]
    per_agent = lr.dim() == 4
    lr_agent_stride = lr.stride(0) if per_agent else 0
    if per_agent:
        assert lr.shape[0] == n_agents
        lr = lr[0]
    r = lr.shape[2] // 2
    assert k_base.stride() == v_base.stride() and k_base.stride(3) == 1
    assert lr.stride(2) == 1 and lr.stride(1) == 2 * r
    assert B_k.is_contiguous() and B_v.is_contiguous() and q.is_contiguous() and out.is_contiguous()
    a = AttnArgs()
    a.n_seqs, a.n_agents, a.n_q_heads, a.n_kv_heads = n_seqs, n_agents, n_q, n_kv
    a.head_dim, a.r = d, r
    a.lora_scale = lora_scale
    a.softmax_scale = softmax_scale if softmax_scale is not None else 1.0 / math.sqrt(d)
    a.rope_base = rope_base
    a.L_max = L_max
    a.k_base, a.v_base = k_base.data_ptr(), v_base.data_ptr()
    a.kv_seq_stride, a.kv_head_stride, a.kv_tok_stride = (k_base.stride(0), k_base.stride(1),
                                                          k_base.stride(2))
    a.lr_cache, a.lr_seq_stride = lr.data_ptr(), lr.stride(0)
    a.B_k, a.B_v = B_k.data_ptr(), B_v.data_ptr()
    a.q, a.out = q.data_ptr(), out.data_ptr()
    a.kv_len = kv_len.data_ptr() if kv_len is not None else None
    a.max_kv_len = max_kv_len
    a.q_pos0 = q_pos0
    a.n_q_tokens = n_tok
    a.io_dtype, a.out_dtype = _dt(k_base), _dt(out)
    a.lr_agent_stride = lr_agent_stride
    a.value_path = value_path
    a.key_pos0 = key_pos0
    if row_stats is not None:
        assert row_stats.dtype == torch.float32 and row_stats.is_contiguous()
        assert row_stats.numel() == 2 * n_seqs * n_agents * n_q
    a.row_stats = row_stats.data_ptr() if row_stats is not None else None
    return a


def lora_attn_decode_workspace_bytes(args: AttnArgs) -> int:
    return int(lib.lora_attn_decode_workspace_bytes(ctypes.byref(args)))


def decode_workspace(args: AttnArgs, device) -> torch.Tensor:
    """A zero-filled workspace large enough for these decode arguments."""
    n = lora_attn_decode_workspace_bytes(args)
    if n == 0:
        raise LoraAttnError(LA_ERR_INVALID_ARG, "lora_attn_decode_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def lora_attn_decode(args: AttnArgs, workspace: torch.Tensor, stream=None) -> None:
    st = lib.lora_attn_decode(ctypes.byref(args), workspace.data_ptr(), workspace.numel(),
                              _stream(stream))
    _check(st, "lora_attn_decode")


def lora_attn_decode_combine(outs: torch.Tensor, stats: torch.Tensor, out: torch.Tensor,
                             stream=None) -> None:
    """Merge the decodes of n_parts key slices of the same queries: outs
    [n_parts, *rows, d] (fp32 or bf16), stats float32 [n_parts, *rows, 2] as
    row_stats holds them, out [*rows, d] of outs' dtype; all contiguous."""
    assert outs.is_contiguous() and stats.is_contiguous() and out.is_contiguous()
    assert stats.dtype == torch.float32 and out.dtype == outs.dtype
    n_parts, d = outs.shape[0], outs.shape[-1]
    rows = out.numel() // d
    assert outs.numel() == n_parts * rows * d and stats.numel() == 2 * n_parts * rows
    st = lib.lora_attn_decode_combine(outs.data_ptr(), stats.data_ptr(), n_parts, rows, d, _dt(out),
                                      out.data_ptr(), _stream(stream))
    _check(st, "lora_attn_decode_combine")


def lora_attn_decode_step(args: AttnArgs, A_kv: torch.Tensor, x_new: torch.Tensor,
                          workspace: torch.Tensor, stream=None) -> None:
    """A decode step on device buffers: the new token's LR row x_new[q] A_kv at
    kv_len[q] - 1 of the LR cache(s), then the decode.  x_new [n_seqs, hidden] contiguous;
    A_kv [hidden, 2r], or [n_agents, hidden, 2r] with per-agent caches."""
    assert x_new.is_contiguous() and A_kv.is_contiguous()
    st = lib.lora_attn_decode_step(ctypes.byref(args), A_kv.data_ptr(), x_new.data_ptr(),
                                   x_new.shape[-1], workspace.data_ptr(), workspace.numel(),
                                   _stream(stream))
    _check(st, "lora_attn_decode_step")


def lora_decode_step_host(args: AttnArgs, workspace: torch.Tensor, A_kv: torch.Tensor,
                          x_dev: torch.Tensor, x_host: torch.Tensor, q_host: torch.Tensor,
                          kv_len_host: torch.Tensor, out_host: torch.Tensor, stream=None) -> None:
    """One decode step from host buffers (copies in, LR append, decode, copy
    out), queued on the stream by one library call.  x_dev is the device
    staging [n_seqs, hidden]; the host tensors are CPU tensors, pinned for
    asynchronous copies."""
    for t in (x_host, q_host, kv_len_host, out_host):
        assert t.device.type == "cpu" and t.is_contiguous()
    assert x_dev.is_contiguous() and kv_len_host.dtype == torch.int32
    st = lib.lora_decode_step_host(ctypes.byref(args), workspace.data_ptr(), workspace.numel(),
                                   A_kv.data_ptr(), x_dev.shape[-1], x_dev.data_ptr(),
                                   x_host.data_ptr(), q_host.data_ptr(), kv_len_host.data_ptr(),
                                   out_host.data_ptr(), _stream(stream))
    _check(st, "lora_decode_step_host")


def packed_step_inputs(x_shape, q_shape, n_seqs: int, dtype: torch.dtype, device,
                       pin: bool = False):
    """x [x_shape], q [q_shape] (dtype) and kv_len int32 [n_seqs] as back-to-back
    views of one buffer: laid out so on both sides, lora_decode_step_host moves
    a step's inputs in one copy.  Returns (buffer, x, q, kv_len)."""
    es = torch.empty(0, dtype=dtype).element_size()
    nx, nq = math.prod(x_shape) * es, math.prod(q_shape) * es
    buf = torch.empty(nx + nq + 4 * n_seqs, dtype=torch.uint8, device=device,
                      pin_memory=pin)
    return (buf, buf[:nx].view(dtype).view(x_shape), buf[nx:nx + nq].view(dtype).view(q_shape),
            buf[nx + nq:].view(torch.int32))


def lora_attn_decode_static_scratch(args: AttnArgs, stream=None) -> None:
    """Decode without a workspace: the split scratch is the library's own device
    array (for callers that cannot allocate device memory; see the header)."""
    st = lib.lora_attn_decode_static_scratch(ctypes.byref(args), _stream(stream))
    _check(st, "lora_attn_decode_static_scratch")


def lora_materialize_agent_kv(args: AttnArgs, k_out: torch.Tensor, v_out: torch.Tensor,
                              stream=None) -> None:
    """Every agent's full K^a, V^a ([n_seqs, n_agents, n_kv, L_max, d] each): the
    non-shared baseline's caches (see the header)."""
    assert k_out.is_contiguous() and v_out.is_contiguous()
    st = lib.lora_materialize_agent_kv(ctypes.byref(args), k_out.data_ptr(), v_out.data_ptr(),
                                       _stream(stream))
    _check(st, "lora_materialize_agent_kv")


def lora_attn_prefill(args: AttnArgs, stream=None) -> None:
    st = lib.lora_attn_prefill(ctypes.byref(args), _stream(stream))
    _check(st, "lora_attn_prefill")


def la_device_check() -> int:
    return int(lib.la_device_check())


def la_device_check_word() -> tuple:
    """(status, bits of the device error word that fired); reads and clears it."""
    w = ctypes.c_int32(0)
    st = int(lib.la_device_check_word(ctypes.byref(w)))
    return st, int(w.value)


class DecodeStep:
    """One decode step of the hot path: the new token's LR row at kv_len - 1,
    then every agent's query over the shared caches (lora_attn_decode_step:
    one library call: the row append, then the decode).

    Holds the argument struct and the zero-filled split-K workspace.  Tensors
    must stay alive while it is used.  Without x_new / A_kv it is the decode
    alone."""

    def __init__(self, k_base, v_base, lr, B_k, B_v, q, out, kv_len, *, lora_scale, rope_base,
                 max_kv_len, A_kv=None, x_new=None):
        self.args = make_args(k_base, v_base, lr, B_k, B_v, q, out, lora_scale=lora_scale,
                              rope_base=rope_base, kv_len=kv_len, max_kv_len=max_kv_len)
        self.workspace = decode_workspace(self.args, q.device)
        self.lr, self.A_kv = lr, A_kv
        self.x_new = None if x_new is None else x_new.reshape(x_new.shape[0], -1)
        self._keep = (k_base, v_base, lr, B_k, B_v, q, out, kv_len, x_new)

    def __call__(self, stream=None) -> None:
        if self.x_new is not None:
            lora_attn_decode_step(self.args, self.A_kv, self.x_new, self.workspace, stream)
        else:
            lora_attn_decode(self.args, self.workspace, stream)

    def from_host(self, x_host, q_host, kv_len_host, out_host, stream=None) -> None:
        """The same step with its inputs and outputs in host memory: one call
        that copies them in and out around the append and the decode; the new
        rows land at kv_len_host - 1."""
        lora_decode_step_host(self.args, self.workspace, self.A_kv, self.x_new, x_host, q_host,
                              kv_len_host, out_host, stream)
