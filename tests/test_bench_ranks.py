"""The multi-rank aggregation of bench.py on two gloo ranks (CPU): the job time is
the slowest rank's, and the rate counts every rank's units."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    ms = 10.0 + 5.0 * rank            # rank 1 is the slow one
    m = bench.max_over_ranks(ms, world, "cpu")
    rate = bench.whole_job_rate(3, 100, world, m)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, m, rate))


def test_two_gloo_ranks_take_the_slowest_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, m, rate in res:
        assert m == 15.0
        assert rate == pytest.approx(3 * 100 * 2 / 0.015)


def test_single_rank_rate():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(7.0, 1, "cpu") == 7.0
    assert bench.whole_job_rate(3, 200, 1, 50.0) == pytest.approx(12000.0)
