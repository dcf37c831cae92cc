"""Run the CUDA path (through the Python binding of libep.so) on given inputs
and fetch its outputs as numpy arrays, and compute the oracle's outputs for
the same inputs.  Used by the -m gpu parity tests."""
import numpy as np

import oracle as O
import workload as W


def _torch():
    import torch
    return torch


def run_cuda(topk, w, x, R, S, E, block_m, scale=None, g_home=None, g_rep=None, clear=False, with_y=True,
             fused=False):
    """All outputs of one pass: stats, plan, layout, align-sort, dispatch,
    stand-in expert, combine, grad-reduce.  x: uint16 [T,H] (or None).
    fused: False (the separate route calls), True (ep_route_fused) or
    "dispatch" (ep_route_dispatch_fused: route and dispatch in one launch)."""
    torch = _torch()
    import token_dispatch_histogram_b200 as tdh
    T, K = topk.shape
    P = T * K
    dev = torch.device("cuda")
    out = {}
    t_topk = torch.from_numpy(np.ascontiguousarray(topk, dtype=np.int32)).to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    loads = torch.full((E,), -7, dtype=torch.int32, device=dev)
    mv = torch.full((1,), -7.0, dtype=torch.float64, device=dev)
    ws = torch.full((tdh.ep_workspace_size(T, K, E),), 0xAB, dtype=torch.uint8, device=dev)
    lay = tdh.ep_plan_layout(E, R)
    plan = torch.full((lay["words"],), -7, dtype=torch.int32, device=dev)
    pos = torch.full((P,), -7, dtype=torch.int32, device=dev)
    src = torch.full((P,), -7, dtype=torch.int32, device=dev)
    slot = torch.full((P,), -7, dtype=torch.int32, device=dev)
    cap, capb = tdh.align_sort_capacity(P, E, block_m)
    sids = torch.full((cap,), -7, dtype=torch.int32, device=dev)
    eids = torch.full((capb,), -7, dtype=torch.int32, device=dev)
    ntpp = torch.full((1,), -7, dtype=torch.int32, device=dev)
    if fused == "dispatch":  # route and dispatch in one launch
        H = x.shape[1]
        t_x = torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16).to(dev)
        buf = torch.full((P, H), -1, dtype=torch.int16, device=dev).view(torch.bfloat16)
        tdh.ep_route_dispatch_fused(t_topk, E, R, S, loads, mv, plan, pos, src, ws, t_x, buf, slot, block_m, sids,
                                    eids, ntpp, status)
    elif fused:
        tdh.ep_route_fused(t_topk, E, R, S, loads, mv, plan, pos, src, ws, slot, block_m, sids, eids, ntpp, status)
    else:
        tdh.ep_route_stats(t_topk, E, loads, mv, ws, status)
        tdh.ep_plan(loads, R, S, K, E, plan, status)
        tdh.ep_layout(t_topk, E, R, S, plan, ws, pos, src, slot, status)
        tdh.ep_align_sort(t_topk, E, block_m, sids, eids, ntpp, ws, status)
    out.update(loads=loads.cpu().numpy(), max_vio=float(mv.cpu().numpy()[0]), plan=plan.cpu().numpy(), layout=lay,
               pos=pos.cpu().numpy(), src=src.cpu().numpy(), pair_slot=slot.cpu().numpy(),
               sorted_ids=sids.cpu().numpy(), expert_ids=eids.cpu().numpy(), ntpp=int(ntpp.cpu().numpy()[0]))
    if x is not None:
        H = x.shape[1]
        if fused != "dispatch":
            t_x = torch.from_numpy(np.ascontiguousarray(x)).view(torch.bfloat16).to(dev)
            buf = torch.full((P, H), -1, dtype=torch.int16, device=dev).view(torch.bfloat16)
            tdh.ep_dispatch(t_x, K, pos, buf, status)
        out["buf"] = buf.view(torch.int16).cpu().numpy().view(np.uint16)
        if with_y:
            t_scale = torch.from_numpy(np.ascontiguousarray(scale, dtype=np.float32)).to(dev)
            tdh.ep_expert_scale(buf, src, t_topk, t_scale, buf, status)
            out["y"] = buf.view(torch.int16).cpu().numpy().view(np.uint16)
        t_w = torch.from_numpy(np.ascontiguousarray(w, dtype=np.float32)).to(dev)
        o = torch.full((T, H), -1, dtype=torch.int16, device=dev).view(torch.bfloat16)
        tdh.ep_combine(buf, t_w, pos, o, status)
        out["out"] = o.view(torch.int16).cpu().numpy().view(np.uint16)
    if g_home is not None:
        t_gh = torch.from_numpy(np.ascontiguousarray(g_home)).to(dev)
        if g_rep.dtype == np.uint16:
            t_gr = torch.from_numpy(g_rep.view(np.int16)).to(dev).view(torch.bfloat16)
        else:
            t_gr = torch.from_numpy(np.ascontiguousarray(g_rep)).to(dev)
        tdh.ep_replica_grad_reduce(t_gh, t_gr, E, R, plan, clear, status)
        out["g_home"] = t_gh.cpu().numpy()
        gr = t_gr.cpu()
        out["g_rep"] = gr.view(torch.int16).numpy().view(np.uint16) if g_rep.dtype == np.uint16 else gr.numpy()
    out["status"] = tdh.ep_status_read(status)
    return out


def run_oracle(topk, w, x, R, S, E, block_m, scale=None, g_home=None, g_rep=None, clear=False):
    T, K = topk.shape
    loads, mv, bad = O.route_stats(topk, E)
    pl = O.plan(loads, R, S, K, E)
    lo = O.layout(topk, pl, R, S, E)
    ids, eids, n = O.align_sort(topk, E, block_m)
    res = dict(loads=loads, max_vio=mv, plan=pl, layout=lo, sorted_ids=ids, expert_ids=eids, ntpp=n)
    if x is not None:
        buf = O.dispatch(x, lo["pos"], K, T * K)
        res["buf"] = buf
        y = O.expert_standin(buf, lo["src"], topk, scale)
        res["y"] = y
        res["out"] = O.combine(y, w, lo["pos"], K)
    if g_home is not None:
        gh, gr = O.grad_reduce(g_home, g_rep, pl["rep_expert"], clear)
        res["g_home"], res["g_rep"] = gh, gr
    return res


def plan_field(out, name, count):
    off = out["layout"][name]
    return out["plan"][off:off + count]


def expected_plan_tables(pl, lo, R, S, K, E):
    """Derived plan tables from the oracle's plan and layout, for checking the
    CUDA plan buffer: home_base, copy_first/cnt, rep_begin/base, rank tables."""
    n = pl["n_rep"]
    order, cu = lo["slot_order"], lo["cu_seqlens"]
    first_row = {int(s): int(cu[i]) for i, s in enumerate(order)}
    home_base = np.array([first_row[e] for e in range(E)], dtype=np.int32)
    rep_base = np.array([first_row[E + m] for m in range(n)], dtype=np.int32)
    copy_first = np.zeros(E, dtype=np.int32)
    copy_cnt = np.zeros(E, dtype=np.int32)
    rep_begin = np.zeros(n, dtype=np.int32)
    nxt = pl["home_count"].astype(np.int64).copy()
    for m in range(n):
        e = int(pl["rep_expert"][m])
        if copy_cnt[e] == 0:
            copy_first[e] = m
        copy_cnt[e] += 1
        rep_begin[m] = nxt[e]
        nxt[e] += pl["rep_count"][m]
    rank_nrep = np.bincount(pl["rep_rank"], minlength=R).astype(np.int32) if n else np.zeros(R, np.int32)
    rank_rep_first = np.concatenate([[0], np.cumsum(rank_nrep)[:-1]]).astype(np.int32)
    return dict(home_base=home_base, rep_base=rep_base, copy_first=copy_first, copy_cnt=copy_cnt,
                rep_begin=rep_begin, rank_nrep=rank_nrep, rank_rep_first=rank_rep_first)


def bf16_ulp_diff(a_u16, b_u16):
    """|difference| in bf16 units in the last place (monotone integer mapping)."""
    def key(u):
        u = u.astype(np.int32)
        return np.where(u & 0x8000, 0x8000 - (u & 0x7FFF), 0x8000 + (u & 0x7FFF))
    return np.abs(key(a_u16) - key(b_u16))


def case_inputs(R, S, K, E, H, seed, kind="skew", bias_scale=1.0):
    T = R * S
    if kind == "uniform":
        topk, w = W.routing_from(T, E, K, seed=seed, uniform=True)
    elif kind == "single":
        topk, w = W.routing_from(T, E, K, seed=seed, force_expert0=True)
    else:
        rng = np.random.default_rng(seed)
        topk, w = W.routing_from(T, E, K, seed=seed, bias_e=rng.normal(0, bias_scale, E))
    x = W.hidden(T, H, seed=seed + 1000) if H else None
    return topk, w, x


def assert_route_parity(cu, orc, R, S, K, E):
    """Every route output of run_cuda equals the oracle's, bit for bit."""
    assert cu["status"] == 0
    np.testing.assert_array_equal(cu["loads"], orc["loads"])
    assert cu["max_vio"] == orc["max_vio"]  # fp64, same expression on both sides
    pl = orc["plan"]
    n = pl["n_rep"]
    assert plan_field(cu, "n_rep", 1)[0] == n
    np.testing.assert_array_equal(plan_field(cu, "rep_expert", n), pl["rep_expert"])
    np.testing.assert_array_equal(plan_field(cu, "rep_rank", n), pl["rep_rank"])
    np.testing.assert_array_equal(plan_field(cu, "rep_count", n), pl["rep_count"])
    np.testing.assert_array_equal(plan_field(cu, "home_count", E), pl["home_count"])
    lo = orc["layout"]
    np.testing.assert_array_equal(plan_field(cu, "slot_order", E + n), lo["slot_order"])
    np.testing.assert_array_equal(plan_field(cu, "cu_seqlens", E + n + 1), lo["cu_seqlens"])
    exp = expected_plan_tables(pl, lo, R, S, K, E)
    for name in ("home_base", "copy_cnt", "rank_nrep", "rank_rep_first"):
        np.testing.assert_array_equal(plan_field(cu, name, len(exp[name])), exp[name], err_msg=name)
    for name in ("rep_base", "rep_begin"):
        np.testing.assert_array_equal(plan_field(cu, name, n), exp[name], err_msg=name)
    has = exp["copy_cnt"] > 0
    np.testing.assert_array_equal(plan_field(cu, "copy_first", E)[has], exp["copy_first"][has])
    np.testing.assert_array_equal(cu["pos"], lo["pos"])
    np.testing.assert_array_equal(cu["src"], lo["src"])
    np.testing.assert_array_equal(cu["pair_slot"], lo["pair_slot"])
    np.testing.assert_array_equal(cu["sorted_ids"], orc["sorted_ids"])
    np.testing.assert_array_equal(cu["expert_ids"], orc["expert_ids"])
    assert cu["ntpp"] == orc["ntpp"]
