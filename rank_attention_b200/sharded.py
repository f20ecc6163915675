"""Sequence-sharded decode over several GPUs (one process per GPU).

Every sequence's base and LR caches are cut along the keys: rank p holds the
rows [lo_p, hi_p) of each cache (tile-aligned slices of L_max) in its own HBM.
A decode step on rank p runs lora_attn_decode over its slice alone, with
key_pos0 = lo_p (its keys are RoPE'd at their global positions) and row_stats
(each output row's largest scaled score M and softmax sum L over the slice).
The ranks then all-gather the outputs and the stats -- (d + 2) fp32 values per
query row, over NCCL on NVLink -- and every rank merges them with
lora_attn_decode_combine (the split-K combine, across devices).  No rank reads
another rank's cache: the only traffic is the gather.

The decode and the merge are the library's kernels; this module only slices
the shapes, moves the per-row results with torch.distributed and orders them
by rank.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import torch
import torch.distributed as dist

from . import lora_attn as la

KEY_TILE = 128   # slices start on whole key tiles of the decode


def shard_bounds(L_max: int, world: int, rank: int, tile: int = KEY_TILE) -> Tuple[int, int]:
    """Rows [lo, hi) of every cache held by `rank`: the L_max rows cut into
    `world` contiguous slices of whole tiles, as equal as whole tiles allow
    (the last slices may be a tile shorter, or empty when L_max is short)."""
    assert world >= 1 and 0 <= rank < world and L_max >= 0
    tiles = (L_max + tile - 1) // tile
    t0 = rank * tiles // world
    t1 = (rank + 1) * tiles // world
    return min(t0 * tile, L_max), min(t1 * tile, L_max)


def local_kv_len(kv_len: Sequence[int], lo: int, hi: int) -> List[int]:
    """Keys of each sequence inside the slice [lo, hi): sequence q sees keys
    [0, kv_len[q]), so the slice holds min(max(kv_len[q] - lo, 0), hi - lo)."""
    return [min(max(int(k) - lo, 0), hi - lo) for k in kv_len]


def gather_rows(local: torch.Tensor, group=None) -> torch.Tensor:
    """[world, *local.shape]: every rank's tensor, in rank order (one
    all-gather into a flat buffer)."""
    world = dist.get_world_size(group)
    flat = torch.empty(world * local.numel(), dtype=local.dtype, device=local.device)
    dist.all_gather_into_tensor(flat, local.contiguous().view(-1), group=group)
    return flat.view((world,) + tuple(local.shape))


class ShardedDecode:
    """One rank's part of a sequence-sharded decode step.

    k_base, v_base [n_seqs, n_kv, hi - lo, d] and lr [n_seqs, hi - lo, 2r]
    (or [n_agents, n_seqs, hi - lo, 2r]) are this rank's slices of the
    caches; B_k, B_v, q are the full (replicated) tensors; kv_len the global
    lengths (host ints).  Calling it writes the decode over all the ranks'
    keys into `out` on every rank."""

    def __init__(self, k_base, v_base, lr, B_k, B_v, q, out, kv_len: Sequence[int], lo: int, hi: int,
                 *, lora_scale: float, rope_base: float, group=None):
        self.group = group
        dev = q.device
        self.out = out
        self.out_local = torch.empty_like(out)
        self.stats = torch.empty((q.shape[0], q.shape[1], q.shape[3], 2), dtype=torch.float32, device=dev)
        self.args = None
        if hi > lo:
            self.kv_local = torch.tensor(local_kv_len(kv_len, lo, hi), dtype=torch.int32, device=dev)
            self.args = la.make_args(k_base, v_base, lr, B_k, B_v, q, self.out_local, lora_scale=lora_scale,
                                     rope_base=rope_base, kv_len=self.kv_local, max_kv_len=hi - lo,
                                     key_pos0=lo, row_stats=self.stats)
            self.workspace = la.decode_workspace(self.args, dev)
        else:   # a rank holding no rows: the merge's identity element (no keys, weight 0)
            self.out_local.zero_()
            self.stats[..., 0] = float("-inf")
            self.stats[..., 1] = 0.0

    def __call__(self) -> None:
        """On the current stream: the local decode, the all-gathers, the merge."""
        if self.args is not None:
            la.lora_attn_decode(self.args, self.workspace)
        outs = gather_rows(self.out_local, self.group)
        stats = gather_rows(self.stats, self.group)
        la.lora_attn_decode_combine(outs, stats, self.out)
