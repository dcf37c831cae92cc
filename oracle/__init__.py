"""CPU oracle for the expert-parallel dispatch path -- TEST INFRASTRUCTURE.

Only tests/, the package smoke check and the benchmark's CPU-baseline leg may
import this module.  The product path (token_dispatch_histogram_b200) never
does, and shares no code with it.

Thin numpy marshalling over liboracle.so (oracle.c), a plain single-threaded C
restatement of the definitions on the source pages; the C file cites the
passage each function follows.  Every function here takes and returns numpy
arrays; bf16 data travel as uint16 bit patterns.
"""
import ctypes

import numpy as np

from . import build as _build

_lib = None
_c = ctypes


def lib(path=None):
    """Load the oracle library (the default build unless `path` is given)."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(_build.build()))
    return _lib


def _bind(L):
    P = _c.c_void_p
    L.oracle_route_stats.restype = _c.c_int64
    L.oracle_route_stats.argtypes = [P, _c.c_int64, _c.c_int, _c.c_int, P, P]
    L.oracle_plan.restype = _c.c_int
    L.oracle_plan.argtypes = [P, _c.c_int, _c.c_int64, _c.c_int, _c.c_int, P, P, P, P]
    L.oracle_layout.restype = _c.c_int
    L.oracle_layout.argtypes = [P, _c.c_int64, _c.c_int, _c.c_int, _c.c_int, _c.c_int64, _c.c_int, P, P, P, P, P, P,
                                P, P, P]
    L.oracle_align_sort.restype = _c.c_int64
    L.oracle_align_sort.argtypes = [P, _c.c_int64, _c.c_int, _c.c_int, _c.c_int, P, _c.c_int64, P, _c.c_int64]
    L.oracle_dispatch.restype = None
    L.oracle_dispatch.argtypes = [P, _c.c_int64, _c.c_int, _c.c_int64, P, P]
    L.oracle_expert_standin.restype = None
    L.oracle_expert_standin.argtypes = [P, _c.c_int64, _c.c_int64, P, P, P, P]
    L.oracle_combine.restype = None
    L.oracle_combine.argtypes = [P, P, P, _c.c_int64, _c.c_int, _c.c_int64, P]
    L.oracle_combine_closed.restype = None
    L.oracle_combine_closed.argtypes = [P, P, P, _c.c_int64, _c.c_int, _c.c_int64, P, P]
    L.oracle_dispatch_backward.restype = None
    L.oracle_dispatch_backward.argtypes = [P, P, _c.c_int64, _c.c_int, _c.c_int64, P]
    L.oracle_combine_backward.restype = None
    L.oracle_combine_backward.argtypes = [P, P, P, P, _c.c_int64, _c.c_int, _c.c_int64, P, P]
    L.oracle_prefetch_slots.restype = None
    L.oracle_prefetch_slots.argtypes = [_c.c_int, P, P, P, _c.c_int, _c.c_int, _c.c_int64, _c.c_int, P, P, P]
    L.oracle_load_matrix.restype = None
    L.oracle_load_matrix.argtypes = [P, _c.c_int, _c.c_int64, _c.c_int, P]
    L.oracle_quota_plan_at.restype = _c.c_int
    L.oracle_quota_plan_at.argtypes = [P, _c.c_int, _c.c_int, _c.c_int64, _c.c_int, P, P, P, P]
    L.oracle_quota_threshold.restype = _c.c_int64
    L.oracle_quota_threshold.argtypes = [P, _c.c_int, _c.c_int, _c.c_int64, _c.c_int]
    L.oracle_quota_layout.restype = _c.c_int
    L.oracle_quota_layout.argtypes = [P, _c.c_int, _c.c_int64, _c.c_int, _c.c_int, P, P, P, P, P, P, P, P, P, P]
    L.oracle_grad_reduce.restype = None
    L.oracle_grad_reduce.argtypes = [P, P, _c.c_int, _c.c_int64, _c.c_int, P, _c.c_int]
    return L


def _p(a):
    assert a.flags["C_CONTIGUOUS"]
    return _c.c_void_p(a.ctypes.data)


def _i32(a):
    return np.ascontiguousarray(a, dtype=np.int32)


def route_stats(topk, E, L=None):
    """(loads int32 [E], max_vio float, n_bad_ids)."""
    L = L or lib()
    topk = _i32(topk)
    T, K = topk.shape
    loads = np.zeros(E, dtype=np.int32)
    mv = np.zeros(1, dtype=np.float64)
    bad = L.oracle_route_stats(_p(topk), T, K, E, _p(loads), _p(mv))
    return loads, float(mv[0]), int(bad)


def plan(loads, R, S, K, E, L=None):
    """Replica plan: dict(n_rep, rep_expert, rep_rank, rep_count, home_count)."""
    L = L or lib()
    loads = _i32(loads)
    cap = E + R - 1
    re = np.full(cap, -1, dtype=np.int32)
    rr = np.full(cap, -1, dtype=np.int32)
    rc = np.zeros(cap, dtype=np.int32)
    hc = np.zeros(E, dtype=np.int32)
    n = L.oracle_plan(_p(loads), R, S, K, E, _p(re), _p(rr), _p(rc), _p(hc))
    if n < 0:
        raise ValueError("loads do not sum to R*S*K")
    return dict(n_rep=n, rep_expert=re[:n].copy(), rep_rank=rr[:n].copy(), rep_count=rc[:n].copy(), home_count=hc)


def layout(topk, pl, R, S, E, L=None):
    """dict(pos [P], src [P], pair_slot [P], slot_order [E+n_rep], cu_seqlens [E+n_rep+1])."""
    L = L or lib()
    topk = _i32(topk)
    T, K = topk.shape
    P = T * K
    n = pl["n_rep"]
    pos = np.empty(P, dtype=np.int32)
    src = np.full(P, -1, dtype=np.int32)
    slot = np.empty(P, dtype=np.int32)
    order = np.empty(E + n, dtype=np.int32)
    cu = np.empty(E + n + 1, dtype=np.int32)
    re, rr, rc = (_i32(pl[k]) if n else np.zeros(1, np.int32) for k in ("rep_expert", "rep_rank", "rep_count"))
    hc = _i32(pl["home_count"])
    rcode = L.oracle_layout(_p(topk), T, K, E, R, S, n, _p(re), _p(rr), _p(rc), _p(hc), _p(pos), _p(src), _p(slot),
                            _p(order), _p(cu))
    if rcode != 0:
        raise ValueError("a rank's rows do not come out to S*K")
    return dict(pos=pos, src=src, pair_slot=slot, slot_order=order, cu_seqlens=cu)


def align_sort_capacity(P, E, block_m):
    cap = P + E * (block_m - 1)
    return cap, (cap + block_m - 1) // block_m


def align_sort(topk, E, block_m, L=None):
    """(sorted_token_ids [cap], expert_ids [cap_blocks], num_tokens_post_pad)."""
    L = L or lib()
    topk = _i32(topk)
    T, K = topk.shape
    cap, capb = align_sort_capacity(T * K, E, block_m)
    ids = np.empty(cap, dtype=np.int32)
    eids = np.empty(capb, dtype=np.int32)
    n = L.oracle_align_sort(_p(topk), T, K, E, block_m, _p(ids), cap, _p(eids), capb)
    if n < 0:
        raise ValueError("capacity")
    return ids, eids, int(n)


def dispatch(x, pos, K, nrows, L=None):
    """buf [nrows, H] uint16 with buf[pos[p]] = x[p // K]; unwritten rows 0."""
    L = L or lib()
    x = np.ascontiguousarray(x, dtype=np.uint16)
    T, H = x.shape
    buf = np.zeros((nrows, H), dtype=np.uint16)
    L.oracle_dispatch(_p(x), T, K, H, _p(_i32(pos)), _p(buf))
    return buf


def expert_standin(buf, src, topk, scale, L=None):
    L = L or lib()
    buf = np.ascontiguousarray(buf, dtype=np.uint16)
    nrows, H = buf.shape
    y = np.empty_like(buf)
    L.oracle_expert_standin(_p(buf), nrows, H, _p(_i32(src)), _p(_i32(topk).reshape(-1)),
                            _p(np.ascontiguousarray(scale, dtype=np.float32)), _p(y))
    return y


def combine(y, w, pos, K, L=None):
    L = L or lib()
    y = np.ascontiguousarray(y, dtype=np.uint16)
    w = np.ascontiguousarray(w, dtype=np.float32)
    T = w.shape[0]
    H = y.shape[1]
    out = np.empty((T, H), dtype=np.uint16)
    L.oracle_combine(_p(y), _p(w), _p(_i32(pos)), T, K, H, _p(out))
    return out


def combine_closed(x_rows, w_rows, topk_rows, scale, L=None):
    L = L or lib()
    x_rows = np.ascontiguousarray(x_rows, dtype=np.uint16)
    w_rows = np.ascontiguousarray(w_rows, dtype=np.float32)
    topk_rows = _i32(topk_rows)
    nt, H = x_rows.shape
    K = w_rows.shape[1]
    out = np.empty((nt, H), dtype=np.uint16)
    L.oracle_combine_closed(_p(x_rows), _p(w_rows), _p(topk_rows), nt, K, H,
                            _p(np.ascontiguousarray(scale, dtype=np.float32)), _p(out))
    return out


def grad_reduce(g_home, g_rep, rep_expert, clear=False, L=None):
    """In place on copies: returns (g_home', g_rep')."""
    L = L or lib()
    gh = np.array(g_home, dtype=np.float32, copy=True, order="C")
    gr = np.array(g_rep, copy=True, order="C")
    dt = 0 if gr.dtype == np.float32 else 1
    if dt == 1:
        assert gr.dtype == np.uint16
    n = gh.shape[1]
    re = _i32(rep_expert) if len(rep_expert) else np.zeros(1, np.int32)
    L.oracle_grad_reduce(_p(gh), _p(gr), dt, n, len(rep_expert), _p(re), int(clear))
    return gh, gr


def dispatch_backward(dbuf, pos, T, K, L=None):
    """dx [T, H]: the unpermute gradient of dispatch."""
    L = L or lib()
    dbuf = np.ascontiguousarray(dbuf, dtype=np.uint16)
    H = dbuf.shape[1]
    dx = np.empty((T, H), dtype=np.uint16)
    L.oracle_dispatch_backward(_p(dbuf), _p(_i32(pos)), T, K, H, _p(dx))
    return dx


def combine_backward(dout, w, y, pos, dy_init=None, L=None):
    """(dy [rows, H] uint16, dw [T, K] float64): the gradient of combine."""
    L = L or lib()
    dout = np.ascontiguousarray(dout, dtype=np.uint16)
    w = np.ascontiguousarray(w, dtype=np.float32)
    y = np.ascontiguousarray(y, dtype=np.uint16)
    T, H = dout.shape
    K = w.shape[1]
    dy = np.zeros_like(y) if dy_init is None else np.array(dy_init, dtype=np.uint16, copy=True)
    dw = np.empty((T, K), dtype=np.float64)
    L.oracle_combine_backward(_p(dout), _p(w), _p(y), _p(_i32(pos)), T, K, H, _p(dy), _p(dw))
    return dy, dw


def prefetch_slots(pl, E, R, B, SK=0, L=None):
    """(slot [n_rep] int32: E + j or -1, n_remote [R] int32, load_capped [R]
    int64: rank loads when slotless replicas' pairs stay home; needs SK = S*K)."""
    L = L or lib()
    n = pl["n_rep"]
    re, rr, rc = (_i32(pl[k]) if n else np.zeros(1, np.int32) for k in ("rep_expert", "rep_rank", "rep_count"))
    slot = np.empty(max(n, 1), dtype=np.int32)
    nrem = np.empty(R, dtype=np.int32)
    capped = np.empty(R, dtype=np.int64)
    L.oracle_prefetch_slots(n, _p(re), _p(rr), _p(rc), E, R, SK, B, _p(slot), _p(nrem), _p(capped))
    return slot[:n].copy(), nrem, capped


def load_matrix(topk, R, S, K, E, L=None):
    """int32 [R, E]: pairs of each source rank per expert."""
    L = L or lib()
    topk = _i32(topk)
    Lm = np.empty((R, E), dtype=np.int32)
    L.oracle_load_matrix(_p(topk), R, S * K, E, _p(Lm))
    return Lm


def quota_plan_at(loads, E, R, tau, B, L=None):
    """The quota plan at threshold tau (dict), or None when tau is infeasible."""
    L = L or lib()
    loads = _i32(loads)
    cap = E + R - 1
    re = np.full(cap, -1, dtype=np.int32)
    rr = np.full(cap, -1, dtype=np.int32)
    rc = np.zeros(cap, dtype=np.int32)
    hq = np.zeros(E, dtype=np.int32)
    n = L.oracle_quota_plan_at(_p(loads), E, R, int(tau), int(B), _p(re), _p(rr), _p(rc), _p(hq))
    if n < 0:
        return None
    return dict(tau=int(tau), n_rep=n, rep_expert=re[:n].copy(), rep_rank=rr[:n].copy(), rep_count=rc[:n].copy(),
                home_quota=hq)


def quota_threshold(loads, E, R, P, B, L=None):
    L = L or lib()
    return int(L.oracle_quota_threshold(_p(_i32(loads)), E, R, int(P), int(B)))


def quota_plan(loads, R, S, K, E, B, L=None):
    """Threshold search then the plan at tau*."""
    tau = quota_threshold(loads, E, R, R * S * K, B, L=L)
    return quota_plan_at(loads, E, R, tau, B, L=L)


def quota_layout(topk, qp, R, S, K, E, L=None):
    """dict(pos [P], src [P], slot_order, cu_seqlens, rank_load [R], n_local)."""
    L = L or lib()
    topk = _i32(topk)
    P = R * S * K
    n = qp["n_rep"]
    pos = np.full(P, -1, dtype=np.int32)
    src = np.full(P, -1, dtype=np.int32)
    order = np.empty(E + n, dtype=np.int32)
    cu = np.empty(E + n + 1, dtype=np.int32)
    rl = np.empty(R, dtype=np.int32)
    nl = np.zeros(1, dtype=np.int64)
    re, rr, rc = (_i32(qp[k]) if n else np.zeros(1, np.int32) for k in ("rep_expert", "rep_rank", "rep_count"))
    code = L.oracle_quota_layout(_p(topk), R, S * K, E, n, _p(re), _p(rr), _p(rc), _p(_i32(qp["home_quota"])),
                                 _p(pos), _p(src), _p(order), _p(cu), _p(rl), _p(nl))
    if code != 0:
        raise ValueError(f"quota layout failed ({code})")
    return dict(pos=pos, src=src, slot_order=order, cu_seqlens=cu, rank_load=rl, n_local=int(nl[0]))


def bf16_to_f32(u16):
    return (np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
