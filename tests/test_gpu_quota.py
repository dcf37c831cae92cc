"""Quota-driven planner on the GPU vs the CPU oracle (-m gpu).

Everything is integer work, so every output is compared bit for bit: loads,
the threshold tau*, the replicas, home quotas, rank loads and offsets, slot
order, cu_seqlens, the locality count and per-instance tables, pos and src.
Cases: the hand-derived 4-rank example, fuzzed shapes with ragged tiles (S*K
not a multiple of 512), the degenerate cases (one rank, B = 0, uniform
routing, all top-1 on one expert, T = 0, many experts), and the routings of
four workloads at full size.  Dispatch -> stand-in expert -> combine through
the quota layout must give the layout-free combine of the oracle bit for bit.
"""
import json
import os

import numpy as np
import pytest

import oracle as O
import oracle_pins as PINS
import workload as W

pytestmark = pytest.mark.gpu

QUOTA_GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "quota_hand_example_4rank.json")


def run_quota(topk, R, S, E, B):
    import torch
    import token_dispatch_histogram_b200 as tdh
    T, K = topk.shape
    P = T * K
    dev = torch.device("cuda")
    t_topk = torch.from_numpy(np.ascontiguousarray(topk, dtype=np.int32)).to(dev)
    loads = torch.full((E,), -7, dtype=torch.int32, device=dev)
    lay = tdh.ep_quota_plan_layout(E, R)
    plan = torch.full((lay["words"],), -7, dtype=torch.int32, device=dev)
    pos = torch.full((max(P, 1),), -7, dtype=torch.int32, device=dev)
    src = torch.full((max(P, 1),), -7, dtype=torch.int32, device=dev)
    ws = torch.full((tdh.ep_quota_workspace_size(T, K, E, R),), 0xAB, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    tdh.ep_quota_route(t_topk, E, R, S, B, loads, plan, pos, src, ws, status)
    pl = plan.cpu().numpy()

    def f(name, n):
        return pl[lay[name]:lay[name] + n]

    return dict(loads=loads.cpu().numpy(), plan=pl, f=f, lay=lay, pos=pos.cpu().numpy()[:P], src=src.cpu().numpy()[:P],
                status=tdh.ep_status_read(status), t_topk=t_topk, t_pos=pos, t_src=src)


def check_quota(topk, R, S, E, B):
    T, K = topk.shape
    P, SK, ER = T * K, S * K, E // R
    cu = run_quota(topk, R, S, E, B)
    assert cu["status"] == 0
    loads = np.bincount(topk.ravel(), minlength=E).astype(np.int32) if P else np.zeros(E, np.int32)
    np.testing.assert_array_equal(cu["loads"], loads)
    qp = O.quota_plan(loads, R, S, K, E, B)
    lo = O.quota_layout(topk, qp, R, S, K, E)
    f = cu["f"]
    n = qp["n_rep"]
    assert int(f("tau", 1)[0]) == qp["tau"]
    assert int(f("n_rep", 1)[0]) == n
    assert int(f("n_local", 1)[0]) == lo["n_local"]
    np.testing.assert_array_equal(f("rep_expert", n), qp["rep_expert"])
    np.testing.assert_array_equal(f("rep_rank", n), qp["rep_rank"])
    np.testing.assert_array_equal(f("rep_count", n), qp["rep_count"])
    np.testing.assert_array_equal(f("home_quota", E), qp["home_quota"])
    rep_experts = [int(e) for e in dict.fromkeys(qp["rep_expert"].tolist())]  # replicated experts, match order
    assert int(f("n_chunks", 1)[0]) == len(rep_experts)
    assert f("rep_experts", E)[:len(rep_experts)].tolist() == rep_experts
    np.testing.assert_array_equal(f("rank_load", R), lo["rank_load"])
    off = np.concatenate([[0], np.cumsum(lo["rank_load"])[:-1]])
    np.testing.assert_array_equal(f("rank_off", R), off)
    nrep_r = np.bincount(qp["rep_rank"], minlength=R) if n else np.zeros(R, np.int64)
    np.testing.assert_array_equal(f("rank_nrep", R), nrep_r)
    np.testing.assert_array_equal(f("rank_rep_first", R), np.concatenate([[0], np.cumsum(nrep_r)[:-1]]))
    np.testing.assert_array_equal(f("slot_order", E + n), lo["slot_order"])
    np.testing.assert_array_equal(f("cu_seqlens", E + n + 1), lo["cu_seqlens"])
    cap = E + R - 1
    assert np.all(f("slot_order", E + cap)[E + n:] == -1)
    assert np.all(f("cu_seqlens", E + cap + 1)[E + n + 1:] == P)
    np.testing.assert_array_equal(cu["pos"], lo["pos"])
    np.testing.assert_array_equal(cu["src"], lo["src"])
    # per-instance tables against their definitions
    Lm = O.load_matrix(topk, R, S, K, E) if P else np.zeros((R, E), np.int32)
    for i in range(E + n):
        e = i if i < E else int(qp["rep_expert"][i - E])
        r = e // ER if i < E else int(qp["rep_rank"][i - E])
        q = int(qp["home_quota"][e]) if i < E else int(qp["rep_count"][i - E])
        assert f("inst_local", E + n)[i] == min(q, int(Lm[r, e]))
        assert f("inst_lpre", E + n)[i] == int(Lm[:r, e].sum())
    return cu, qp, lo


def test_quota_hand_example():
    g = PINS.golden()
    with open(QUOTA_GOLDEN) as fh:
        q = json.load(fh)
    topk = np.array(g["topk_ids"], dtype=np.int32)
    for key, B in (("B1", 1), ("B2", 2), ("B0", 0)):
        cu, qp, lo = check_quota(topk, g["R"], g["S"], g["E"], B)
        assert int(cu["f"]("tau", 1)[0]) == q[key]["tau"]
        if "pos" in q[key]:
            assert cu["pos"].tolist() == q[key]["pos"]


CASES = [
    # R, S, K, E, B, bias sigma
    (4, 64, 2, 16, 1, 1.0),
    (8, 200, 6, 64, 2, 1.5),  # S*K = 1200: ragged rank-aligned tiles
    (16, 301, 4, 64, 3, 2.0),
    (2, 1000, 8, 32, 1, 2.5),
    (32, 96, 8, 256, 8, 1.0),
    (64, 40, 8, 384, 4, 2.0),
    (1, 700, 3, 8, 2, 1.0),  # one rank
    (8, 512, 2, 8, 0, 2.0),  # B = 0
    (1024, 2, 2, 1024, 1, 1.0),  # many ranks and experts
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "R%d_S%d_K%d_E%d_B%d" % c[:5])
def test_quota_shapes(case):
    R, S, K, E, B, sig = case
    rng = np.random.default_rng(R * 1000 + S)
    bias = rng.normal(0.0, sig, E).astype(np.float32)
    topk, _ = W.routing_from(R * S, E, K, seed=7, bias_e=bias)
    check_quota(topk, R, S, E, B)


def test_quota_fuzz():
    rng = np.random.default_rng(2024)
    for it in range(60):
        R = int(rng.choice([1, 2, 3, 4, 8, 16, 32]))
        ER = int(rng.integers(1, 9))
        E = R * ER
        K = int(rng.integers(1, min(E, 8) + 1))
        S = int(rng.integers(0, 400))
        B = int(rng.integers(0, 6))
        bias = rng.normal(0.0, rng.uniform(0.0, 3.0), E).astype(np.float32)
        topk, _ = W.routing_from(R * S, E, K, seed=900 + it, bias_e=bias)
        check_quota(topk.reshape(R * S, K), R, S, E, B)


def test_quota_degenerate():
    E, K, R, S = 64, 4, 8, 300
    T = R * S
    uni, _ = W.routing_from(T, E, K, seed=3, uniform=True)
    check_quota(uni, R, S, E, 2)
    one, _ = W.routing_from(T, E, K, seed=3, force_expert0=True)
    check_quota(one, R, S, E, 1)
    check_quota(one, R, S, E, 7)
    check_quota(np.zeros((0, K), dtype=np.int32), R, 0, E, 2)


def test_quota_bad_expert_id():
    import token_dispatch_histogram_b200 as tdh
    topk, _ = W.routing_from(8 * 100, 32, 4, seed=5)
    topk = topk.copy()
    topk[17, 2] = 32
    cu = run_quota(topk, 8, 100, 32, 2)
    assert cu["status"] & tdh.EP_DEV_BAD_EXPERT_ID
    assert int(cu["f"]("tau", 1)[0]) == -1
    assert np.all(cu["pos"] == -1)


@pytest.mark.parametrize("cfg,variant", [(1, "default"), (2, "default"), (3, "default"), (5, "default"),
                                         (5, "single_expert"), (4, "default")])
def test_quota_fullsize(cfg, variant):
    c = W.shape(cfg)
    topk, _ = W.routing(cfg, 0, 0, variant)
    R, S, E = c["R"], c["S"], c["E"]
    for B in sorted({1, 3, E // R}):
        check_quota(topk, R, S, E, B)


def test_quota_rows_through_dispatch_and_combine():
    """The row kernels need only pos: dispatch, the stand-in expert and combine
    over the quota layout reproduce the layout-free combine bit for bit."""
    import torch
    import token_dispatch_histogram_b200 as tdh
    R, S, K, E, H = 8, 256, 6, 64, 256
    T, P = R * S, R * S * K
    bias = np.random.default_rng(1).normal(0.0, 2.0, E).astype(np.float32)
    topk, w = W.routing_from(T, E, K, seed=11, bias_e=bias)
    x = W.hidden(T, H, seed=12)
    scale = W.expert_scale(E)
    cu = run_quota(topk, R, S, E, 2)
    assert cu["status"] == 0
    dev = torch.device("cuda")
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    t_x = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    buf = torch.full((P, H), -1, dtype=torch.int16, device=dev).view(torch.bfloat16)
    tdh.ep_dispatch(t_x, K, cu["t_pos"], buf, status)
    tdh.ep_expert_scale(buf, cu["t_src"], cu["t_topk"], torch.from_numpy(scale).to(dev), buf, status)
    out = torch.full((T, H), -1, dtype=torch.int16, device=dev).view(torch.bfloat16)
    tdh.ep_combine(buf, torch.from_numpy(w).to(dev), cu["t_pos"], out, status)
    assert tdh.ep_status_read(status) == 0
    want = O.combine_closed(x, w, topk, scale)
    np.testing.assert_array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), want)


@pytest.mark.parametrize("gdt", ["f32", "bf16"])
def test_quota_grad_reduce(gdt):
    """Replica gradients into their home expert, in match order, read from the
    quota plan: bit-exact against the oracle's fp32 adds in the same order."""
    import torch
    import token_dispatch_histogram_b200 as tdh
    for (R, S, K, E, B, n) in [(8, 300, 6, 64, 1, 1000), (16, 200, 8, 64, 3, 4096 + 520)]:
        bias = np.random.default_rng(R).normal(0.0, 2.0, E).astype(np.float32)
        topk, _ = W.routing_from(R * S, E, K, seed=21, bias_e=bias)
        cu = run_quota(topk, R, S, E, B)
        assert cu["status"] == 0
        loads = np.bincount(topk.ravel(), minlength=E).astype(np.int32)
        qp = O.quota_plan(loads, R, S, K, E, B)
        cap = E + R - 1
        gh = W.grad_rows(3, W.STREAM_GHOME, n, E, "f32")
        gr = W.grad_rows(3, W.STREAM_GREP, n, cap, gdt)
        dev = torch.device("cuda")
        t_gh = torch.from_numpy(gh.copy()).to(dev)
        t_gr = (torch.from_numpy(gr.view(np.int16).copy()).to(dev).view(torch.bfloat16) if gdt == "bf16"
                else torch.from_numpy(gr.copy()).to(dev))
        lay = tdh.ep_quota_plan_layout(E, R)
        plan = torch.from_numpy(cu["plan"]).to(dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        tdh.ep_quota_replica_grad_reduce(t_gh, t_gr, E, R, plan, False, status)
        assert tdh.ep_status_read(status) == 0
        want_h, _ = O.grad_reduce(gh, gr, qp["rep_expert"])
        np.testing.assert_array_equal(t_gh.cpu().numpy(), want_h)
        assert lay["words"] == plan.numel()
