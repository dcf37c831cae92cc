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


def _agree_worker(rank, world, port, fail_rank, q):
    import datetime
    import sys
    import torch.distributed as dist
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        q.put((rank, bench.all_ranks_ok(rank != fail_rank, world, "cpu")))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("fail_rank", [None, 0, 1])
def test_optional_pass_is_all_or_none(fail_rank):
    """The end-to-end pass's pinned buffers: when one rank cannot allocate
    them, every rank skips the pass (none waits at a barrier for it)."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_agree_worker, args=(r, 2, port, fail_rank, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [ok for _, ok in res] == [fail_rank is None] * 2


def _gather_worker(rank, world, port, q):
    """One rank of the rank-local form's exchange: its own expert counts, the
    all-gather into [R, E] (gather_counts, gloo), and the list offsets a rank
    derives from the gathered matrix."""
    import datetime
    import sys
    import numpy as np
    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import oracle as O
        from gpu_path import case_inputs
        from token_dispatch_histogram_b200.ranks import gather_counts
        S, K, E = 300, 4, 8 * world
        topk, _, _ = case_inputs(world, S, K, E, 0, seed=17, bias_scale=1.5)
        own = topk[rank * S:(rank + 1) * S]
        row = torch.from_numpy(np.bincount(own.reshape(-1), minlength=E).astype(np.int32))
        counts = torch.full((world, E), -1, dtype=torch.int32)
        gather_counts(row, counts)
        C = counts.numpy()
        # every pair of this rank: (pairs of its expert on lower source ranks)
        # + (its stable rank among this rank's pairs of that expert) must be its
        # rank among ALL pairs of that expert in global pair order
        base = C[:rank].sum(axis=0)
        flat_all = topk.reshape(-1)
        ok = True
        seen = np.zeros(E, dtype=np.int64)
        for i, e in enumerate(own.reshape(-1)):
            p = rank * S * K + i
            g_rank = int(np.count_nonzero(flat_all[:p] == e))
            ok &= int(base[e] + seen[e]) == g_rank
            seen[e] += 1
        loads, _, _ = O.route_stats(topk, E)
        q.put((rank, C.tolist(), bool(ok), C.sum(axis=0).tolist() == loads.tolist()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_rank_local_count_exchange_gloo(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_gather_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert all(r[1] == res[0][1] for r in res)          # the same matrix on every rank
    assert all(r[2] for r in res)                        # source prefix + local rank = global rank
    assert all(r[3] for r in res)                        # column sums = the oracle's loads


def _exchange_worker(rank, world, port, R, q):
    """One process of the rank-local job's handle exchange, with stand-ins for
    the IPC export and open (no GPU): every process ends with the same R
    addresses, its own ranks' buffers by their own address and every other
    rank's through the opener, given that rank's own handle and offset."""
    import datetime
    import sys
    import torch
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from token_dispatch_histogram_b200.ranks import EP_IPC_HANDLE_BYTES, exchange_addresses
        n = R // world
        local = {rank * n + i: torch.zeros(16) for i in range(n)}

        def exporter(t):
            r = next(k for k, v in local.items() if v is t)
            h = bytes([r % 251]) * EP_IPC_HANDLE_BYTES
            return h, 16 * r

        opened_args = []

        def opener(h, off):
            opened_args.append((h[0], off))
            return 1000 + off, 0x7000_0000 + off

        addrs, opened = exchange_addresses(local, R, exporter=exporter, opener=opener)
        ok_local = all(addrs[r] == t.data_ptr() for r, t in local.items())
        ok_remote = all(addrs[r] == 0x7000_0000 + 16 * r for r in range(R) if r not in local)
        ok_args = sorted(opened_args) == sorted((r % 251, 16 * r) for r in range(R) if r not in local)
        q.put((rank, bool(ok_local), bool(ok_remote), bool(ok_args), len(opened)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,R", [(2, 2), (2, 8), (3, 6)])
def test_rank_local_handle_exchange_gloo(world, R):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_exchange_worker, args=(r, world, port, R, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert all(r[1] and r[2] and r[3] for r in res)
    assert all(r[4] == R - R // world for r in res)       # every other process's ranks opened once


def test_export_record_round_trip():
    from token_dispatch_histogram_b200.ranks import RECORD_BYTES, pack_export, unpack_export
    h = bytes(range(64))
    rec = pack_export(37, h, 123456789012, 4242)
    assert rec.size == RECORD_BYTES
    assert unpack_export(rec) == (37, 123456789012, 4242, h)
