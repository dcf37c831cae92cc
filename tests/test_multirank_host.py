"""The benchmark's multi-rank host logic on CPU with gloo, world size 2 (no
GPU): every rank gets its own seed, the job time is the max over ranks, and the
whole-job throughput counts all ranks' pairs over that time."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import datetime
    import sys
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mine = 10.0 + 5.0 * rank                       # rank 1 is the slow one
        job = bench.max_over_ranks(mine, world, "cpu")
        v = bench.job_throughput(world, 196608, 20, job)
        q.put((rank, bench.rank_seed(7, rank), job, v))
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [7, 1007]            # distinct seeds: independent layers
    assert all(r[2] == 15.0 for r in res)               # max over ranks on every rank
    assert all(r[3] == pytest.approx(2 * 196608 * 20 / 0.015) for r in res)
