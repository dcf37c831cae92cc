"""The rank-local form across processes (-m gpu): RankLocalJob with the peer
tables built from CUDA IPC handles exchanged over torch.distributed.

Two processes share the one GPU of the test box (IPC between processes works
on one device as it does across devices); each holds R/2 of the R ranks.  The
processes exchange their buffers' IPC handles and the count rows over gloo,
and order the ranks' kernels with host fences (stream synchronisation and a
barrier): no kernel waits on another process's kernel.  Every rank's layout,
receive rows, combined rows and home-expert gradients must equal its slice of
the CPU oracle's one-buffer outputs, bit for bit.  A one-process job (no
process group, every rank local) is checked the same way.
"""
import os
import socket
import sys

import numpy as np
import pytest

import oracle as O
import workload as W
from gpu_path import case_inputs, expected_plan_tables

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)

CASES = [
    # R, S, K, E, H, grad_n, processes
    (4, 64, 2, 16, 128, 1000, 2),    # two ranks per process
    (2, 700, 6, 32, 256, 4096, 2),   # one rank per process, ragged tiles
    (8, 96, 4, 64, 64, 0, 2),
    (4, 64, 2, 16, 128, 1000, 1),    # one process holds every rank
]


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _inputs(case):
    R, S, K, E, H, n, _ = case
    topk, w, x = case_inputs(R, S, K, E, H, seed=R * 13 + S, bias_scale=1.5)
    g_home = W.grad_rows(3, W.STREAM_GHOME, n, E) if n else None
    g_rep = W.grad_rows(4, W.STREAM_GREP, n, E + R - 1) if n else None
    return topk, w, x, g_home, g_rep


def _run_job(case, group_world):
    """Run the job's ranks held by this process; returns {rank: outputs}."""
    import torch
    from token_dispatch_histogram_b200.ranks import RankLocalJob
    R, S, K, E, H, n, _ = case
    topk, w, x, g_home, g_rep = _inputs(case)
    loads, _, _ = O.route_stats(topk, E)
    pl = O.plan(loads, R, S, K, E)
    lo = O.layout(topk, pl, R, S, E)
    exp = expected_plan_tables(pl, lo, R, S, K, E)
    dev = torch.device("cuda", 0)
    job = RankLocalJob(R, S, K, E, H, device=dev, grad_n=n)
    ER = E // R
    for rk in job.ranks:
        r = rk.rank
        rk.topk_local.copy_(torch.from_numpy(topk[r * S:(r + 1) * S]))
        rk.w_local.copy_(torch.from_numpy(w[r * S:(r + 1) * S]))
        rk.x_local.copy_(torch.from_numpy(x[r * S:(r + 1) * S].view(np.int16)).view(torch.bfloat16))
        rk.buf.fill_(-1.0)
        if n:
            rk.g_home.copy_(torch.from_numpy(g_home[r * ER:(r + 1) * ER]))
            f, c = exp["rank_rep_first"][r], exp["rank_nrep"][r]
            assert c <= rk.rep_rows
            rk.g_rep.zero_()
            if c:
                rk.g_rep[:c].copy_(torch.from_numpy(g_rep[f:f + c]))
    job.open_peers()
    job.route()
    job.dispatch()
    job.fence()
    bufs = {rk.rank: rk.buf.view(torch.int16).cpu().numpy().view(np.uint16) for rk in job.ranks}
    job.fence()  # every process has read its rows before any combine runs
    job.combine()
    if n:
        job.fence()
        job.grad_reduce()
    job.fence()
    out = {}
    for rk in job.ranks:
        out[rk.rank] = {"status": rk.status(), "pos": rk.pos_local.cpu().numpy(), "buf": bufs[rk.rank],
                        "out": rk.out_local.view(torch.int16).cpu().numpy().view(np.uint16),
                        "g_home": rk.g_home.cpu().numpy() if n else None,
                        "loads": rk.loads.cpu().numpy()}
    job.close()
    return out


def _worker(rank, world, port, case, q):
    import datetime
    sys.path.insert(0, ROOT)
    sys.path.insert(0, HERE)
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        q.put((rank, _run_job(case, world)))
    except BaseException as exc:  # report, then let the process group time out the peer
        q.put((rank, repr(exc)))
        raise
    finally:
        dist.destroy_process_group()


def _check(case, results):
    R, S, K, E, H, n, _ = case
    topk, w, x, g_home, g_rep = _inputs(case)
    SK, T, ER = S * K, R * S, E // R
    loads, _, _ = O.route_stats(topk, E)
    pl = O.plan(loads, R, S, K, E)
    lo = O.layout(topk, pl, R, S, E)
    buf = O.dispatch(x, lo["pos"], K, T * K)
    want = O.combine(buf, w, lo["pos"], K)
    gh = O.grad_reduce(g_home, g_rep, pl["rep_expert"])[0] if n else None
    assert sorted(results) == list(range(R))
    for r, got in results.items():
        assert got["status"] == 0
        np.testing.assert_array_equal(got["loads"], loads)
        np.testing.assert_array_equal(got["pos"], lo["pos"][r * SK:(r + 1) * SK])
        np.testing.assert_array_equal(got["buf"], buf[r * SK:(r + 1) * SK])
        np.testing.assert_array_equal(got["out"], want[r * S:(r + 1) * S])
        if n:
            np.testing.assert_array_equal(got["g_home"], gh[r * ER:(r + 1) * ER])


@pytest.mark.parametrize("case", CASES, ids=lambda c: "R{}_S{}_K{}_E{}_H{}_n{}_procs{}".format(*c))
def test_rank_local_job_across_processes(case):
    procs_n = case[-1]
    if procs_n == 1:
        _check(case, _run_job(case, 1))
        return
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, procs_n, port, case, q)) for r in range(procs_n)]
    for p in procs:
        p.start()
    results, errors = {}, []
    try:
        for _ in range(procs_n):
            rank, res = q.get(timeout=240)
            if isinstance(res, str):
                errors.append((rank, res))
            else:
                results.update(res)
    finally:
        for p in procs:
            p.join(60)
            if p.is_alive():
                p.kill()
                p.join(10)
    assert not errors, errors
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    _check(case, results)
