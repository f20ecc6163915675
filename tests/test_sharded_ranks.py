"""Host logic of the sequence-sharded decode (rank_attention_b200.sharded) on
CPU: the slices every rank holds, each sequence's keys inside a slice, and the
rank-ordered all-gather, run on two and three gloo ranks.  Each rank's slice
result comes from the oracle here (the kernels need a GPU; the one-GPU test of
the same arithmetic on the kernels is tests/test_sharded_gpu.py); the merge of
the gathered slices must reproduce the oracle's decode over all keys."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.mark.parametrize("L,world", [(8192, 4), (8192, 3), (300, 4), (128, 2), (1000, 8), (0, 2)])
def test_slices_cover_the_cache_in_whole_tiles(L, world):
    sys.path.insert(0, ROOT)
    from rank_attention_b200.sharded import KEY_TILE, shard_bounds
    b = [shard_bounds(L, world, p) for p in range(world)]
    assert b[0][0] == 0 and b[-1][1] == L
    for (lo, hi), (lo2, _) in zip(b[:-1], b[1:]):
        assert hi == lo2 and lo <= hi
    for lo, hi in b:
        assert lo % KEY_TILE == 0 and (hi % KEY_TILE == 0 or hi == L)
    sizes = [hi - lo for lo, hi in b if hi < L]
    assert not sizes or max(sizes) - min(sizes) <= KEY_TILE


def test_local_kv_len():
    sys.path.insert(0, ROOT)
    from rank_attention_b200.sharded import local_kv_len
    assert local_kv_len([8192, 100, 2048, 2049], 2048, 4096) == [2048, 0, 0, 1]
    assert local_kv_len([5], 0, 128) == [5]


def _inputs():
    gen = torch.Generator().manual_seed(11)
    rn = lambda *shape, sc=1.0: torch.randn(*shape, generator=gen, dtype=torch.float64) * sc
    n_seqs, n_agents, n_kv, g, d, r, L = 2, 2, 2, 2, 16, 4, 700
    return dict(k_base=rn(n_seqs, n_kv, L, d), v_base=rn(n_seqs, n_kv, L, d), lr=rn(n_seqs, L, 2 * r),
                B_k=rn(n_agents, r, n_kv * d, sc=0.3), B_v=rn(n_agents, r, n_kv * d, sc=0.3),
                q=rn(n_seqs, n_agents, 1, n_kv * g, d)), [700, 300]


KW = dict(lora_scale=2.0, softmax_scale=0.25, rope_base=10000.0)


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from oracle import impl as O
    from rank_attention_b200.sharded import gather_rows, local_kv_len, shard_bounds
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    inp, kv_len = _inputs()
    n_seqs, n_kv, L, d = inp["k_base"].shape
    n_agents, n_q = inp["q"].shape[1], inp["q"].shape[3]
    g = n_q // n_kv
    lo, hi = shard_bounds(L, world, rank)
    kl = local_kv_len(kv_len, lo, hi)
    out = torch.zeros(n_seqs, n_agents, n_q, d, dtype=torch.float64)
    stats = torch.zeros(n_seqs, n_agents, n_q, 2, dtype=torch.float64)
    for s in range(n_seqs):
        for a in range(n_agents):
            for j in range(n_kv):
                o, M, Lsum = O.decode_slice(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"],
                                            inp["q"], seq=s, agent=a, kv_head=j, lo=lo, hi=lo + kl[s], **KW)
                out[s, a, j * g:(j + 1) * g] = torch.from_numpy(o)
                stats[s, a, j * g:(j + 1) * g, 0] = torch.from_numpy(M)
                stats[s, a, j * g:(j + 1) * g, 1] = torch.from_numpy(Lsum)
    outs = gather_rows(out)
    st = gather_rows(stats)
    merged = O.combine_slices(outs.numpy(), st[..., 0].numpy(), st[..., 1].numpy())
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, merged))


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_gather_in_rank_order_and_merge_to_the_whole_decode(world):
    ctx = mp.get_context("spawn")
    qu = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, qu)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted((qu.get(timeout=180) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    sys.path.insert(0, ROOT)
    from oracle import impl as O
    inp, kv_len = _inputs()
    ref = O.lora_attention(inp["k_base"], inp["v_base"], inp["lr"], inp["B_k"], inp["B_v"], inp["q"],
                           torch.tensor(kv_len), mode="decode", **KW)[:, :, 0]
    for _, merged in res:
        np.testing.assert_allclose(merged, ref, rtol=1e-11, atol=1e-11)
