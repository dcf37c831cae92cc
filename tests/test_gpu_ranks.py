"""Rank-local form of the path (one rank of R per process) against the oracle.

The R ranks are emulated on one GPU: R sets of per-rank buffers (separate
allocations, reached through the peer table exactly as peers' buffers would
be), each rank's kernels launched in turn, and the all-gather of the counts
replaced by a copy of the R rows.  No kernel waits on another rank's kernel.
Every rank's output must equal its slice of the oracle's one-buffer outputs,
bit for bit: counts row = histogram of its own pairs, plan identical on every
rank, pos_local = pos[r*S*K : (r+1)*S*K], the R receive buffers = the
dispatch buffer's R partitions, combine and replica gradient reduction equal.
"""
import numpy as np
import pytest

import oracle as O
import workload as W
from gpu_path import case_inputs, expected_plan_tables

pytestmark = pytest.mark.gpu

CASES = [
    # R, S, K, E, H, kind
    (4, 64, 2, 16, 128, "skew"),
    (8, 700, 6, 64, 2048, "skew"),     # S*K = 4200: ragged histogram tiles per rank
    (2, 5000, 8, 32, 256, "single"),   # a dominant expert
    (16, 300, 4, 64, 64, "uniform"),   # no replica
    (1, 500, 3, 8, 72, "skew"),        # one rank
    (32, 128, 8, 256, 512, "skew"),
    (64, 40, 8, 384, 16, "skew"),      # many ranks, few tokens each
]


def _t(torch, a, dev):
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def _u16(t):
    return t.view(__import__("torch").int16).cpu().numpy().view(np.uint16)


def _ranks(R, S, K, E, H, topk, w, x, grad_n=0, grad_dtype=None):
    import torch
    import token_dispatch_histogram_b200 as tdh
    from token_dispatch_histogram_b200.ranks import EpRank
    dev = torch.device("cuda")
    ranks = []
    for r in range(R):
        rk = EpRank(r, R, S, K, E, H, device=dev, grad_n=grad_n,
                    grad_dtype=grad_dtype if grad_dtype is not None else torch.float32)
        rk.topk_local.copy_(_t(torch, topk[r * S:(r + 1) * S], dev))
        rk.w_local.copy_(_t(torch, w[r * S:(r + 1) * S], dev))
        rk.x_local.copy_(_t(torch, x[r * S:(r + 1) * S], dev))
        rk.buf.fill_(-1.0)
        rk.pos_local.fill_(-7)
        ranks.append(rk)
    for rk in ranks:
        rk.count()
    counts = torch.stack([rk.counts_row for rk in ranks])  # the all-gather
    for rk in ranks:
        rk.counts.copy_(counts)
        rk.plan_and_layout()
    peers = tdh.peer_table([rk.buf for rk in ranks])
    for rk in ranks:
        rk.set_peers(peers)
        rk.dispatch()
    torch.cuda.synchronize()  # every rank's rows have landed before any combine
    return ranks, peers


@pytest.mark.parametrize("case", CASES, ids=lambda c: "R{}_S{}_K{}_E{}_H{}_{}".format(*c))
def test_rank_local_path(case):
    import torch
    import token_dispatch_histogram_b200 as tdh
    R, S, K, E, H, kind = case
    topk, w, x = case_inputs(R, S, K, E, H, seed=R * 31 + S, kind=kind, bias_scale=1.5)
    T, SK = R * S, S * K
    ranks, peers = _ranks(R, S, K, E, H, topk, w, x)

    # oracle, one buffer
    loads, _, _ = O.route_stats(topk, E)
    pl = O.plan(loads, R, S, K, E)
    lo = O.layout(topk, pl, R, S, E)
    buf = O.dispatch(x, lo["pos"], K, T * K)
    exp = expected_plan_tables(pl, lo, R, S, K, E)
    n = pl["n_rep"]
    L = ranks[0].plan_layout

    def field(plan, name, cnt):
        return plan[L[name]:L[name] + cnt]

    for r, rk in enumerate(ranks):
        assert rk.status() == 0
        own, _, _ = O.route_stats(topk[r * S:(r + 1) * S], E)
        np.testing.assert_array_equal(rk.counts_row.cpu().numpy(), own)
        np.testing.assert_array_equal(rk.loads.cpu().numpy(), loads)
        plan = rk.plan.cpu().numpy()
        assert field(plan, "n_rep", 1)[0] == n
        np.testing.assert_array_equal(field(plan, "rep_expert", n), pl["rep_expert"])
        np.testing.assert_array_equal(field(plan, "rep_rank", n), pl["rep_rank"])
        np.testing.assert_array_equal(field(plan, "rep_count", n), pl["rep_count"])
        np.testing.assert_array_equal(field(plan, "home_count", E), pl["home_count"])
        np.testing.assert_array_equal(field(plan, "cu_seqlens", E + n + 1), lo["cu_seqlens"])
        np.testing.assert_array_equal(field(plan, "rank_rep_first", R), exp["rank_rep_first"])
        np.testing.assert_array_equal(rk.pos_local.cpu().numpy(), lo["pos"][r * SK:(r + 1) * SK])
        np.testing.assert_array_equal(_u16(rk.buf), buf[r * SK:(r + 1) * SK])

    # stand-in expert on every receiving rank (rows -> pairs from the oracle's
    # src; only the test's expert needs it), then combine from the peers
    scale = W.expert_scale(E)
    t_scale = _t(torch, scale.astype(np.float32), "cuda")
    t_topk = _t(torch, topk, "cuda")
    for d, rk in enumerate(ranks):
        src_d = _t(torch, lo["src"][d * SK:(d + 1) * SK].astype(np.int32), "cuda")
        tdh.ep_expert_scale(rk.buf, src_d, t_topk, t_scale, rk.buf, rk.dev_status)
    torch.cuda.synchronize()
    y = O.expert_standin(buf, lo["src"], topk, scale)
    want = O.combine(y, w, lo["pos"], K)
    for r, rk in enumerate(ranks):
        rk.out_local.fill_(-1.0)
        rk.combine()
    torch.cuda.synchronize()
    for r, rk in enumerate(ranks):
        assert rk.status() == 0
        np.testing.assert_array_equal(_u16(rk.out_local), want[r * S:(r + 1) * S])
    # backward of dispatch through the peers: unit weights
    want_dx = O.dispatch_backward(y, lo["pos"], T, K)
    for r, rk in enumerate(ranks):
        dx = torch.full((S, H), -1.0, dtype=torch.bfloat16, device="cuda")
        tdh.ep_combine_peer(peers, SK, R * SK, None, rk.pos_local, dx, K=K, dev_status=rk.dev_status)
        np.testing.assert_array_equal(_u16(dx), want_dx[r * S:(r + 1) * S])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("clear", [False, True])
def test_rank_local_grad_reduce(dtype, clear):
    import torch
    import token_dispatch_histogram_b200 as tdh
    R, S, K, E, H = 8, 512, 6, 64, 16
    topk, w, x = case_inputs(R, S, K, E, H, seed=91, bias_scale=1.5)
    loads, _, _ = O.route_stats(topk, E)
    pl = O.plan(loads, R, S, K, E)
    lo = O.layout(topk, pl, R, S, E)
    exp = expected_plan_tables(pl, lo, R, S, K, E)
    assert pl["n_rep"] > 0
    ER, cap = E // R, E + R - 1
    for n in (1000, 4096, 3 * 128 * 64 + 8):  # n % 8 != 0 takes the scalar path
        g_home = W.grad_rows(3, W.STREAM_GHOME, n, E)
        g_rep = W.grad_rows(4, W.STREAM_GREP, n, cap, dtype)
        gt = torch.bfloat16 if dtype == "bf16" else torch.float32
        ranks, _ = _ranks(R, S, K, E, H, topk, w, x, grad_n=n, grad_dtype=gt)
        for r, rk in enumerate(ranks):
            rk.g_home.copy_(_t(torch, g_home[r * ER:(r + 1) * ER], "cuda"))
            f, c = exp["rank_rep_first"][r], exp["rank_nrep"][r]
            assert c <= rk.rep_rows
            rk.g_rep.zero_()
            if c:
                rk.g_rep[:c].copy_(_t(torch, g_rep[f:f + c], "cuda"))
        gpeers = tdh.peer_table([rk.g_rep for rk in ranks])
        for rk in ranks:
            rk.set_grad_peers(gpeers)
            rk.grad_reduce(clear)
        torch.cuda.synchronize()
        gh, gr = O.grad_reduce(g_home, g_rep, pl["rep_expert"], clear)
        for r, rk in enumerate(ranks):
            assert rk.status() == 0
            got = rk.g_home.cpu().numpy()
            ref = gh[r * ER:(r + 1) * ER]
            assert (np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)).max() <= 1e-6
            np.testing.assert_array_equal(got, ref)  # same adds, same order
            f, c = exp["rank_rep_first"][r], exp["rank_nrep"][r]
            rows = rk.g_rep[:c]
            rows = _u16(rows) if dtype == "bf16" else rows.cpu().numpy()
            np.testing.assert_array_equal(rows, gr[f:f + c])  # cleared (if asked) or untouched


def test_rank_local_missing_peer_is_flagged():
    """A zero entry in the peer table is never dereferenced: the rows it would
    serve are skipped and EP_DEV_BAD_ROW is raised; every other row lands."""
    import torch
    import token_dispatch_histogram_b200 as tdh
    R, S, K, E, H = 4, 256, 4, 16, 64
    topk, w, x = case_inputs(R, S, K, E, H, seed=5, bias_scale=1.0)
    ranks, peers = _ranks(R, S, K, E, H, topk, w, x)
    for rk in ranks:
        rk.buf.fill_(-1.0)
        rk.dev_status.zero_()
    holed = peers.clone()
    holed[2] = 0
    for rk in ranks:
        rk.set_peers(holed)
        rk.dispatch()
    torch.cuda.synchronize()
    loads, _, _ = O.route_stats(topk, E)
    pl = O.plan(loads, R, S, K, E)
    lo = O.layout(topk, pl, R, S, E)
    buf = O.dispatch(x, lo["pos"], K, R * S * K)
    SK = S * K
    flagged = [rk.status() for rk in ranks]
    assert all(f in (0, tdh.EP_DEV_BAD_ROW) for f in flagged) and any(flagged)
    for d, rk in enumerate(ranks):
        got = _u16(rk.buf)
        if d == 2:
            assert (got == _u16(torch.full((1,), -1.0, dtype=torch.bfloat16))[0]).all()  # untouched
        else:
            np.testing.assert_array_equal(got, buf[d * SK:(d + 1) * SK])


# ---- the quota-driven planner in rank-local form

QUOTA_CASES = [
    # R, S, K, E, H, B, kind
    (4, 64, 2, 16, 128, 1, "skew"),
    (8, 700, 6, 64, 256, 2, "skew"),
    (8, 512, 8, 64, 64, 8, "single"),
    (16, 300, 4, 64, 64, 1, "uniform"),
    (1, 500, 3, 8, 72, 2, "skew"),
    (32, 96, 8, 256, 32, 3, "skew"),
    (8, 512, 2, 8, 32, 0, "skew"),      # B = 0: no replica, the unplanned loads
]


def _quota_ranks(R, S, K, E, H, B, topk, w, x, buf_rows, grad_n=0):
    import torch
    import token_dispatch_histogram_b200 as tdh
    from token_dispatch_histogram_b200.ranks import EpRank
    dev = torch.device("cuda")
    ranks = []
    for r in range(R):
        rk = EpRank(r, R, S, K, E, H, device=dev, grad_n=grad_n, planner="quota", B=B, buf_rows=buf_rows)
        rk.topk_local.copy_(_t(torch, topk[r * S:(r + 1) * S], dev))
        rk.w_local.copy_(_t(torch, w[r * S:(r + 1) * S], dev))
        rk.x_local.copy_(_t(torch, x[r * S:(r + 1) * S], dev))
        rk.buf.fill_(-1.0)
        rk.pos_local.fill_(-7)
        ranks.append(rk)
    for rk in ranks:
        rk.count()
    counts = torch.stack([rk.counts_row for rk in ranks])  # the all-gather
    for rk in ranks:
        rk.counts.copy_(counts)
        rk.plan_and_layout()
    peers = tdh.peer_table([rk.buf for rk in ranks])
    for rk in ranks:
        rk.set_peers(peers)
        rk.dispatch()
    torch.cuda.synchronize()
    return ranks, peers


@pytest.mark.parametrize("case", QUOTA_CASES, ids=lambda c: "R{}_S{}_K{}_E{}_H{}_B{}_{}".format(*c))
def test_rank_local_quota_path(case):
    import torch
    R, S, K, E, H, B, kind = case
    topk, w, x = case_inputs(R, S, K, E, H, seed=R * 17 + S + B, kind=kind, bias_scale=1.5)
    T, SK = R * S, S * K
    loads, _, _ = O.route_stats(topk, E)
    qp = O.quota_plan(loads, R, S, K, E, B)
    lo = O.quota_layout(topk, qp, R, S, K, E)
    n = qp["n_rep"]
    buf_rows = max(int(lo["rank_load"].max()), 1)  # tau*: every rank's rows fit
    ranks, peers = _quota_ranks(R, S, K, E, H, B, topk, w, x, buf_rows)
    buf = O.dispatch(x, lo["pos"], K, T * K)
    off = np.concatenate([[0], np.cumsum(lo["rank_load"])[:-1]]).astype(np.int64)
    L = ranks[0].plan_layout

    def field(plan, name, cnt):
        return plan[L[name]:L[name] + cnt]

    for r, rk in enumerate(ranks):
        assert rk.status() == 0
        plan = rk.plan.cpu().numpy()
        assert int(field(plan, "tau", 1)[0]) == qp["tau"]
        assert int(field(plan, "n_rep", 1)[0]) == n
        assert int(field(plan, "n_local", 1)[0]) == lo["n_local"]
        np.testing.assert_array_equal(field(plan, "rep_expert", n), qp["rep_expert"])
        np.testing.assert_array_equal(field(plan, "rep_rank", n), qp["rep_rank"])
        np.testing.assert_array_equal(field(plan, "rep_count", n), qp["rep_count"])
        np.testing.assert_array_equal(field(plan, "home_quota", E), qp["home_quota"])
        np.testing.assert_array_equal(field(plan, "rank_load", R), lo["rank_load"])
        np.testing.assert_array_equal(field(plan, "rank_off", R), off)
        np.testing.assert_array_equal(field(plan, "cu_seqlens", E + n + 1), lo["cu_seqlens"])
        np.testing.assert_array_equal(rk.pos_local.cpu().numpy(), lo["pos"][r * SK:(r + 1) * SK])
    for d, rk in enumerate(ranks):  # rank d's rows [off_d, off_d + load_d) of the one buffer
        ld = int(lo["rank_load"][d])
        got = _u16(rk.buf)
        np.testing.assert_array_equal(got[:ld], buf[off[d]:off[d] + ld])
    # combine through the peers (rows = the dispatched rows, no expert in between)
    want = O.combine(buf, w, lo["pos"], K)
    for rk in ranks:
        rk.out_local.fill_(-1.0)
        rk.combine()
    torch.cuda.synchronize()
    for r, rk in enumerate(ranks):
        assert rk.status() == 0
        np.testing.assert_array_equal(_u16(rk.out_local), want[r * S:(r + 1) * S])


def test_rank_local_quota_grad_reduce():
    import torch
    import token_dispatch_histogram_b200 as tdh
    R, S, K, E, H, B = 8, 512, 6, 64, 16, 2
    topk, w, x = case_inputs(R, S, K, E, H, seed=93, bias_scale=1.5)
    loads, _, _ = O.route_stats(topk, E)
    qp = O.quota_plan(loads, R, S, K, E, B)
    lo = O.quota_layout(topk, qp, R, S, K, E)
    n_rep = qp["n_rep"]
    assert n_rep > 0
    ER, cap = E // R, E + R - 1
    nrep_r = np.bincount(qp["rep_rank"], minlength=R)
    first = np.concatenate([[0], np.cumsum(nrep_r)[:-1]])
    n = 4096 + 8
    g_home = W.grad_rows(3, W.STREAM_GHOME, n, E)
    g_rep = W.grad_rows(4, W.STREAM_GREP, n, cap)
    ranks, _ = _quota_ranks(R, S, K, E, H, B, topk, w, x, max(int(lo["rank_load"].max()), 1), grad_n=n)
    for r, rk in enumerate(ranks):
        rk.g_home.copy_(_t(torch, g_home[r * ER:(r + 1) * ER], "cuda"))
        rk.g_rep.zero_()
        c = int(nrep_r[r])
        if c:
            rk.g_rep[:c].copy_(_t(torch, g_rep[first[r]:first[r] + c], "cuda"))
    gpeers = tdh.peer_table([rk.g_rep for rk in ranks])
    for rk in ranks:
        rk.set_grad_peers(gpeers)
        rk.grad_reduce(True)
    torch.cuda.synchronize()
    gh, gr = O.grad_reduce(g_home, g_rep, qp["rep_expert"], True)
    for r, rk in enumerate(ranks):
        assert rk.status() == 0
        np.testing.assert_array_equal(rk.g_home.cpu().numpy(), gh[r * ER:(r + 1) * ER])
        c = int(nrep_r[r])
        np.testing.assert_array_equal(rk.g_rep[:c].cpu().numpy(), gr[first[r]:first[r] + c])


def _nccl_one_rank(port, q):
    """Child process: EpRank.route() through a real NCCL process group of one
    rank (the all-gather of the counts is a genuine NCCL call), then dispatch
    and combine through the peer table; results back through the queue."""
    import datetime
    import os
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    sys.path.insert(0, os.path.join(root, "tests"))
    import numpy as np
    import torch
    import torch.distributed as dist
    from gpu_path import case_inputs
    import token_dispatch_histogram_b200 as tdh
    from token_dispatch_histogram_b200.ranks import EpRank
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        S, K, E, H = 1000, 4, 16, 256
        topk, w, x = case_inputs(1, S, K, E, H, seed=8, bias_scale=1.5)
        rk = EpRank(0, 1, S, K, E, H, device="cuda")
        rk.topk_local.copy_(torch.from_numpy(topk))
        rk.w_local.copy_(torch.from_numpy(w))
        rk.x_local.copy_(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16))
        rk.route()
        rk.set_peers(tdh.peer_table([rk.buf]))
        rk.dispatch()
        rk.combine()
        torch.cuda.synchronize()
        # the handle records are host bytes: through NCCL they are staged on the GPU and come back to the host
        from token_dispatch_histogram_b200.ranks import all_gather_rows
        recs = torch.arange(2 * 88, dtype=torch.int32).to(torch.uint8).view(2, 88)
        back = all_gather_rows(recs)
        q.put(dict(status=rk.status(), counts=rk.counts.cpu().numpy(), pos=rk.pos_local.cpu().numpy(),
                   out=rk.out_local.view(torch.int16).cpu().numpy().view(np.uint16),
                   recs_ok=bool(back.device.type == "cpu" and torch.equal(back, recs))))
    finally:
        dist.destroy_process_group()


def test_rank_local_route_through_nccl():
    import socket
    import torch.multiprocessing as mp
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_nccl_one_rank, args=(port, q))
    p.start()
    res = q.get(timeout=240)
    p.join(60)
    assert p.exitcode == 0
    S, K, E, H = 1000, 4, 16, 256
    topk, w, x = case_inputs(1, S, K, E, H, seed=8, bias_scale=1.5)
    loads, _, _ = O.route_stats(topk, E)
    pl = O.plan(loads, 1, S, K, E)
    lo = O.layout(topk, pl, 1, S, E)
    assert res["status"] == 0
    assert res["recs_ok"]
    np.testing.assert_array_equal(res["counts"][0], loads)
    np.testing.assert_array_equal(res["pos"], lo["pos"])
    buf = O.dispatch(x, lo["pos"], K, S * K)
    np.testing.assert_array_equal(res["out"], O.combine(buf, w, lo["pos"], K))


def test_rank_local_fuzz():
    """Random shapes through the rank-local form, both planners: every rank's
    rows, receive buffer and combine equal its slice of the oracle's."""
    import torch
    rng = np.random.default_rng(4242)
    for it in range(20):
        R = int(rng.choice([1, 2, 3, 4, 6, 8, 16, 24]))
        E = R * int(rng.integers(1, 7))
        K = int(rng.integers(1, min(8, E) + 1))
        S = int(rng.integers(1, 400))
        H = 8 * int(rng.integers(1, 40))
        planner = "quota" if it % 2 else "exact"
        B = int(rng.integers(0, 4))
        topk, w, x = case_inputs(R, S, K, E, H, seed=1000 + it, bias_scale=float(rng.uniform(0.5, 3.0)))
        T, SK = R * S, S * K
        loads, _, _ = O.route_stats(topk, E)
        if planner == "exact":
            pl = O.plan(loads, R, S, K, E)
            lo = O.layout(topk, pl, R, S, E)
            off = np.arange(R, dtype=np.int64) * SK
            rl = np.full(R, SK)
            ranks, _ = _ranks(R, S, K, E, H, topk, w, x)
        else:
            qp = O.quota_plan(loads, R, S, K, E, B)
            lo = O.quota_layout(topk, qp, R, S, K, E)
            rl = lo["rank_load"]
            off = np.concatenate([[0], np.cumsum(rl)[:-1]]).astype(np.int64)
            ranks, _ = _quota_ranks(R, S, K, E, H, B, topk, w, x, max(int(rl.max()), 1))
        buf = O.dispatch(x, lo["pos"], K, T * K)
        want = O.combine(buf, w, lo["pos"], K)
        for rk in ranks:
            rk.out_local.fill_(-1.0)
            rk.combine()
        torch.cuda.synchronize()
        for r, rk in enumerate(ranks):
            msg = f"it {it} {planner} R={R} S={S} K={K} E={E} H={H} B={B} rank {r}"
            assert rk.status() == 0, msg
            np.testing.assert_array_equal(rk.pos_local.cpu().numpy(), lo["pos"][r * SK:(r + 1) * SK], err_msg=msg)
            ld = int(rl[r])
            np.testing.assert_array_equal(_u16(rk.buf)[:ld], buf[off[r]:off[r] + ld], err_msg=msg)
            np.testing.assert_array_equal(_u16(rk.out_local), want[r * S:(r + 1) * S], err_msg=msg)
