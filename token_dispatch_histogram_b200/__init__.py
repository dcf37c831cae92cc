"""B200 expert-parallel dispatch path: Python binding of libep.so (include/ep.h).

Argument marshalling only: each function below checks tensor dtypes and
devices, passes data pointers, sizes and the CUDA stream to the C entry point
of the same name, and turns a negative return code into an exception.  Every
step of the path runs in the library's sm_100a kernels; there is no fallback.
If libep.so is missing the import fails.

Device memory and streams come from PyTorch; nothing here computes.
"""
import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libep.so")

EP_OK, EP_ERR_ARG, EP_ERR_CAPACITY, EP_ERR_CUDA = 0, -1, -2, -3
EP_DEV_BAD_EXPERT_ID = 0x1
EP_DEV_LOOKBACK_TIMEOUT = 0x2
EP_DEV_BAD_LOADS = 0x4
EP_DEV_BAD_ROW = 0x8
EP_DEV_COPY_TIMEOUT = 0x10
EP_MAX_EXPERTS = 1024
EP_MAX_RANKS = 1024
EP_DTYPE_F32, EP_DTYPE_BF16 = 0, 1
EP_IPC_HANDLE_BYTES = 64


class EpError(RuntimeError):
    def __init__(self, name, code):
        what = {EP_ERR_ARG: "invalid argument", EP_ERR_CAPACITY: "capacity too small",
                EP_ERR_CUDA: "CUDA launch failed"}.get(code, "error")
        super().__init__(f"{name}: {what} ({code})")
        self.code = code


class EpPlanLayout(ctypes.Structure):
    _fields_ = [("words", ctypes.c_int64), ("cap", ctypes.c_int32)] + [
        (n, ctypes.c_int32) for n in ("n_rep", "n_chunks", "rank_load", "rank_nrep", "rank_rep_first", "home_count",
                                      "home_base", "copy_first", "copy_cnt", "rep_expert", "rep_rank", "rep_count",
                                      "rep_begin", "rep_base", "rep_experts", "slot_order", "cu_seqlens")]


class EpQuotaLayout(ctypes.Structure):
    _fields_ = [("words", ctypes.c_int64), ("cap", ctypes.c_int32)] + [
        (n, ctypes.c_int32) for n in ("tau", "n_rep", "n_local", "n_chunks", "rank_load", "rank_off", "rank_nrep",
                                      "rank_rep_first", "home_quota", "rep_first", "rep_cnt", "rep_experts",
                                      "rep_expert", "rep_rank",
                                      "rep_count", "inst_local", "inst_cum", "inst_base", "inst_lpre", "rep_local_incl",
                                      "slot_order",
                                      "cu_seqlens")]


_lib = None
_V, _I, _I64, _SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t

_SIGS = {
    "ep_version": (ctypes.c_char_p, []),
    "ep_launch_count": (ctypes.c_uint64, []),
    "ep_workspace_size": (_I, [_I64, _I, _I, _V]),
    "ep_plan_layout": (_I, [_I, _I, _V]),
    "ep_route_stats": (_I, [_V, _I64, _I, _I, _V, _V, _V, _SZ, _V, _V]),
    "ep_route_stats_noalloc": (_I, [_V, _I64, _I, _I, _V, _V, _V, _V]),
    "ep_plan": (_I, [_V, _I, _I64, _I, _I, _V, _SZ, _V, _V]),
    "ep_quota_workspace_size": (_I, [_I64, _I, _I, _I, _V]),
    "ep_quota_plan_layout": (_I, [_I, _I, _V]),
    "ep_quota_replica_grad_reduce": (_I, [_V, _V, _I, _I64, _I, _I, _V, _SZ, _I, _V, _V]),
    "ep_quota_route": (_I, [_V, _I64, _I, _I, _I, _I64, _I, _V, _V, _SZ, _V, _V, _V, _SZ, _V, _V]),
    "ep_prefetch_slots": (_I, [_V, _SZ, _I, _I, _I64, _I, _V, _V, _V, _V]),
    "ep_layout": (_I, [_V, _I64, _I, _I, _I, _I64, _V, _SZ, _V, _SZ, _V, _V, _V, _V, _V]),
    "ep_align_sort": (_I, [_V, _I64, _I, _I, _I, _V, _I64, _V, _I64, _V, _V, _SZ, _V, _V]),
    "ep_route_fused": (_I, [_V, _I64, _I, _I, _I, _I64, _V, _V, _V, _SZ, _V, _V, _V, _I, _V, _I64, _V, _I64, _V,
                            _V, _SZ, _V, _V]),
    "ep_route_dispatch_fused": (_I, [_V, _I64, _I, _I, _I, _I64, _V, _V, _V, _SZ, _V, _V, _V, _I, _V, _I64, _V,
                                     _I64, _V, _V, _I64, _V, _I64, _V, _SZ, _V, _V]),
    "ep_dispatch": (_I, [_V, _I64, _I, _I64, _V, _V, _I64, _V, _V]),
    "ep_expert_scale": (_I, [_V, _I64, _I64, _V, _V, _I64, _V, _I, _V, _V, _V]),
    "ep_dispatch_backward": (_I, [_V, _I64, _V, _I64, _I, _I64, _V, _V, _V]),
    "ep_combine_backward": (_I, [_V, _V, _V, _I64, _V, _I64, _I, _I64, _V, _V, _V, _V]),
    "ep_combine": (_I, [_V, _I64, _V, _V, _I64, _I, _I64, _V, _V, _V]),
    "ep_replica_grad_reduce": (_I, [_V, _V, _I, _I64, _I, _I, _V, _SZ, _I, _V, _V]),
    "ep_plan_from_counts": (_I, [_V, _I, _I64, _I, _I, _V, _V, _SZ, _V, _V]),
    "ep_layout_rank": (_I, [_V, _I64, _I, _I, _I, _I, _V, _V, _SZ, _V, _SZ, _V, _V, _V, _V]),
    "ep_dispatch_peer": (_I, [_V, _I64, _I, _I64, _V, _V, _V, _I, _I64, _I64, _V, _V]),
    "ep_combine_peer": (_I, [_V, _V, _I, _I64, _I64, _V, _V, _I64, _I, _I64, _V, _V, _V]),
    "ep_quota_counts_workspace_size": (_I, [_I, _I, _V]),
    "ep_quota_plan_from_counts": (_I, [_V, _I, _I64, _I, _I, _I, _V, _V, _SZ, _V, _SZ, _V, _V]),
    "ep_quota_layout_rank": (_I, [_V, _I64, _I, _I, _I, _I, _V, _V, _SZ, _V, _SZ, _V, _V, _V]),
    "ep_quota_replica_grad_reduce_peer": (_I, [_V, _V, _I64, _I, _I64, _I, _I, _I, _V, _SZ, _I, _V, _V]),
    "ep_replica_grad_reduce_peer": (_I, [_V, _V, _I64, _I, _I64, _I, _I, _I, _V, _SZ, _I, _V, _V]),
    "ep_ipc_export": (_I, [_V, _V, _V]),
    "ep_ipc_open": (_I, [_V, ctypes.c_uint64, _V, _V]),
    "ep_ipc_close": (_I, [_V]),
    "ep_status_read": (_I, [_V, _V, _V]),
    "ep_selftest_lookback_timeout": (_I, [_V, _I64, _I, _I, _V, _V, _V, _SZ, _V, _V]),
}


def lib():
    """The loaded libep.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} not built: run token_dispatch_histogram_b200/build.py "
                              "(or __graft_entry__.build())")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


lib()  # fail at import time when the library is missing


def _check(name, code):
    if code != EP_OK:
        raise EpError(name, code)


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _s(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype(t, *dts):
    if t.dtype not in dts:
        raise TypeError(f"dtype {t.dtype}, expected one of {dts}")


def version():
    return lib().ep_version().decode()


def ep_launch_count():
    return int(lib().ep_launch_count())


def ep_workspace_size(T, K, E):
    n = ctypes.c_size_t(0)
    _check("ep_workspace_size", lib().ep_workspace_size(T, K, E, ctypes.byref(n)))
    return int(n.value)


def ep_plan_layout(E, R):
    L = EpPlanLayout()
    _check("ep_plan_layout", lib().ep_plan_layout(E, R, ctypes.byref(L)))
    return {name: getattr(L, name) for name, _ in EpPlanLayout._fields_}


def ep_route_stats(topk_ids, E, loads, max_vio, ws, dev_status=None, stream=None):
    _dtype(topk_ids, torch.int32)
    _dtype(loads, torch.int32)
    _dtype(max_vio, torch.float64)
    T, K = topk_ids.shape
    _check("ep_route_stats", lib().ep_route_stats(_p(topk_ids), T, K, E, _p(loads), _p(max_vio), _p(ws),
                                                  ws.numel() * ws.element_size(), _p(dev_status), _s(stream)))


def ep_route_stats_noalloc(topk_ids, E, loads, max_vio, dev_status=None, stream=None):
    """ep_route_stats with the library's fixed internal scratch instead of a
    caller workspace (for callers that cannot allocate one)."""
    _dtype(topk_ids, torch.int32)
    _dtype(loads, torch.int32)
    _dtype(max_vio, torch.float64)
    T, K = topk_ids.shape
    _check("ep_route_stats_noalloc", lib().ep_route_stats_noalloc(_p(topk_ids), T, K, E, _p(loads), _p(max_vio),
                                                                  _p(dev_status), _s(stream)))


def ep_plan(loads, R, S, K, E, plan, dev_status=None, stream=None):
    _dtype(loads, torch.int32)
    _dtype(plan, torch.int32)
    _check("ep_plan", lib().ep_plan(_p(loads), R, S, K, E, _p(plan), plan.numel(), _p(dev_status), _s(stream)))


def ep_quota_workspace_size(T, K, E, R):
    n = ctypes.c_size_t(0)
    _check("ep_quota_workspace_size", lib().ep_quota_workspace_size(T, K, E, R, ctypes.byref(n)))
    return int(n.value)


def ep_quota_plan_layout(E, R):
    L = EpQuotaLayout()
    _check("ep_quota_plan_layout", lib().ep_quota_plan_layout(E, R, ctypes.byref(L)))
    return {name: getattr(L, name) for name, _ in EpQuotaLayout._fields_}


def ep_quota_route(topk_ids, E, R, S, B, loads, plan, pos, src, ws, dev_status=None, stream=None):
    """Quota-driven replica plan under a per-rank replica budget B, and the
    local-first per-pair layout (see ep.h)."""
    for t in (topk_ids, loads, plan, pos, src):
        _dtype(t, torch.int32)
    T, K = topk_ids.shape
    _check("ep_quota_route", lib().ep_quota_route(_p(topk_ids), T, K, E, R, S, B, _p(loads), _p(plan), plan.numel(),
                                                  _p(pos), _p(src), _p(ws), ws.numel() * ws.element_size(),
                                                  _p(dev_status), _s(stream)))


def ep_prefetch_slots(plan, E, R, SK, B, slot, n_remote, load_capped=None, stream=None):
    """Weight row (E + j or -1) of every replica under a per-rank slot budget B,
    replicas each rank reads from home, and optionally the rank loads when
    slotless replicas' pairs stay home."""
    for t in (plan, slot, n_remote):
        _dtype(t, torch.int32)
    if load_capped is not None:
        _dtype(load_capped, torch.int64)
    _check("ep_prefetch_slots", lib().ep_prefetch_slots(_p(plan), plan.numel(), E, R, SK, B, _p(slot), _p(n_remote),
                                                        _p(load_capped), _s(stream)))


def ep_layout(topk_ids, E, R, S, plan, ws, pos, src, pair_slot=None, dev_status=None, stream=None):
    for t in (topk_ids, plan, pos, src) + ((pair_slot,) if pair_slot is not None else ()):
        _dtype(t, torch.int32)
    T, K = topk_ids.shape
    _check("ep_layout", lib().ep_layout(_p(topk_ids), T, K, E, R, S, _p(plan), plan.numel(), _p(ws),
                                        ws.numel() * ws.element_size(), _p(pos), _p(src), _p(pair_slot),
                                        _p(dev_status), _s(stream)))


def ep_align_sort(topk_ids, E, block_m, sorted_token_ids, expert_ids, num_tokens_post_pad, ws, dev_status=None,
                  stream=None):
    for t in (topk_ids, sorted_token_ids, expert_ids, num_tokens_post_pad):
        _dtype(t, torch.int32)
    T, K = topk_ids.shape
    _check("ep_align_sort", lib().ep_align_sort(_p(topk_ids), T, K, E, block_m, _p(sorted_token_ids),
                                                sorted_token_ids.numel(), _p(expert_ids), expert_ids.numel(),
                                                _p(num_tokens_post_pad), _p(ws), ws.numel() * ws.element_size(),
                                                _p(dev_status), _s(stream)))


def ep_route_fused(topk_ids, E, R, S, loads, max_vio, plan, pos, src, ws, pair_slot=None, block_m=0,
                   sorted_token_ids=None, expert_ids=None, num_tokens_post_pad=None, dev_status=None, stream=None):
    """ep_route_stats + ep_plan + ep_layout (+ ep_align_sort when
    sorted_token_ids is given) in one cooperative launch."""
    for t in (topk_ids, loads, plan, pos, src):
        _dtype(t, torch.int32)
    _dtype(max_vio, torch.float64)
    T, K = topk_ids.shape
    align = sorted_token_ids is not None
    _check("ep_route_fused", lib().ep_route_fused(
        _p(topk_ids), T, K, E, R, S, _p(loads), _p(max_vio), _p(plan), plan.numel(), _p(pos), _p(src),
        _p(pair_slot), block_m, _p(sorted_token_ids), sorted_token_ids.numel() if align else 0,
        _p(expert_ids), expert_ids.numel() if align else 0, _p(num_tokens_post_pad), _p(ws),
        ws.numel() * ws.element_size(), _p(dev_status), _s(stream)))


def ep_route_dispatch_fused(topk_ids, E, R, S, loads, max_vio, plan, pos, src, ws, x, buf, pair_slot=None,
                            block_m=0, sorted_token_ids=None, expert_ids=None, num_tokens_post_pad=None,
                            dev_status=None, stream=None):
    """ep_route_fused followed by ep_dispatch(x, K, pos, buf), in one
    cooperative launch (the rows are copied as each tile is placed)."""
    for t in (topk_ids, loads, plan, pos, src):
        _dtype(t, torch.int32)
    _dtype(max_vio, torch.float64)
    _dtype(x, torch.bfloat16, torch.int16, torch.uint16)
    _dtype(buf, torch.bfloat16, torch.int16, torch.uint16)
    T, K = topk_ids.shape
    H = x.shape[1]
    if x.shape[0] != T or buf.shape[1] != H:
        raise EpError("ep_route_dispatch_fused", EP_ERR_ARG)
    align = sorted_token_ids is not None
    _check("ep_route_dispatch_fused", lib().ep_route_dispatch_fused(
        _p(topk_ids), T, K, E, R, S, _p(loads), _p(max_vio), _p(plan), plan.numel(), _p(pos), _p(src),
        _p(pair_slot), block_m, _p(sorted_token_ids), sorted_token_ids.numel() if align else 0,
        _p(expert_ids), expert_ids.numel() if align else 0, _p(num_tokens_post_pad), _p(x), H, _p(buf),
        buf.shape[0], _p(ws), ws.numel() * ws.element_size(), _p(dev_status), _s(stream)))


def align_sort_capacity(P, E, block_m):
    cap = P + E * (block_m - 1)
    return cap, (cap + block_m - 1) // block_m


def ep_dispatch(x, K, pos, buf, dev_status=None, stream=None):
    _dtype(x, torch.bfloat16, torch.int16, torch.uint16)
    _dtype(buf, torch.bfloat16, torch.int16, torch.uint16)
    _dtype(pos, torch.int32)
    T, H = x.shape
    _check("ep_dispatch", lib().ep_dispatch(_p(x), T, K, H, _p(pos), _p(buf), buf.shape[0], _p(dev_status),
                                            _s(stream)))


def ep_expert_scale(buf, src, topk_ids, scale, y, dev_status=None, stream=None):
    _dtype(scale, torch.float32)
    rows, H = buf.shape
    _check("ep_expert_scale", lib().ep_expert_scale(_p(buf), rows, H, _p(src), _p(topk_ids), topk_ids.numel(),
                                                    _p(scale), scale.numel(), _p(y), _p(dev_status), _s(stream)))


def ep_combine(y, w, pos, out, dev_status=None, stream=None):
    _dtype(w, torch.float32)
    _dtype(pos, torch.int32)
    T, K = w.shape
    H = y.shape[1]
    _check("ep_combine", lib().ep_combine(_p(y), y.shape[0], _p(w), _p(pos), T, K, H, _p(out), _p(dev_status),
                                          _s(stream)))


def ep_dispatch_backward(dbuf, pos, T, K, dx, dev_status=None, stream=None):
    """dx[t] = sum_k dbuf[pos[t*K+k]] (the unpermute gradient of dispatch)."""
    _dtype(pos, torch.int32)
    H = dbuf.shape[1]
    _check("ep_dispatch_backward", lib().ep_dispatch_backward(_p(dbuf), dbuf.shape[0], _p(pos), T, K, H, _p(dx),
                                                              _p(dev_status), _s(stream)))


def ep_combine_backward(dout, w, y, pos, dy, dw, dev_status=None, stream=None):
    """dy[pos[t,k]] = w[t,k] * dout[t]; dw[t,k] = <dout[t], y[pos[t,k]]>."""
    _dtype(w, torch.float32)
    _dtype(dw, torch.float32)
    _dtype(pos, torch.int32)
    T, K = w.shape
    H = dout.shape[1]
    _check("ep_combine_backward", lib().ep_combine_backward(_p(dout), _p(w), _p(y), y.shape[0], _p(pos), T, K, H,
                                                            _p(dy), _p(dw), _p(dev_status), _s(stream)))


def _grad_dtype(g_home, g_rep, plan):
    _dtype(g_home, torch.float32)
    _dtype(plan, torch.int32)
    if g_rep.dtype == torch.float32:
        return EP_DTYPE_F32
    if g_rep.dtype in (torch.bfloat16, torch.int16, torch.uint16):
        return EP_DTYPE_BF16
    raise TypeError(g_rep.dtype)


def ep_replica_grad_reduce(g_home, g_rep, E, R, plan, clear_replicas=False, dev_status=None, stream=None):
    dt = _grad_dtype(g_home, g_rep, plan)
    n = g_home.shape[1]
    _check("ep_replica_grad_reduce", lib().ep_replica_grad_reduce(_p(g_home), _p(g_rep), dt, n, E, R, _p(plan),
                                                                  plan.numel(), int(bool(clear_replicas)),
                                                                  _p(dev_status), _s(stream)))


def ep_quota_replica_grad_reduce(g_home, g_rep, E, R, plan, clear_replicas=False, dev_status=None, stream=None):
    """ep_replica_grad_reduce for a plan written by ep_quota_route."""
    dt = _grad_dtype(g_home, g_rep, plan)
    n = g_home.shape[1]
    _check("ep_quota_replica_grad_reduce",
           lib().ep_quota_replica_grad_reduce(_p(g_home), _p(g_rep), dt, n, E, R, _p(plan), plan.numel(),
                                              int(bool(clear_replicas)), _p(dev_status), _s(stream)))


# ---- rank-local form: one rank of R (one process per GPU), rows moved
# through a device table of the R ranks' buffer addresses (see ep.h)

def peer_table(tensors, device=None):
    """Device int64 table of the base addresses of R buffers (this rank's own
    and the peers' buffers mapped into this process).  The addresses are read
    on the host from the tensors given; nothing is copied but the table."""
    addrs = [int(t.data_ptr()) for t in tensors]
    dev = device if device is not None else tensors[0].device
    return torch.tensor(addrs, dtype=torch.int64, device=dev)


def ep_ipc_export(tensor):
    """(handle bytes, byte offset) naming `tensor`'s device memory for another
    process (ep_ipc_open there)."""
    h = (ctypes.c_uint8 * EP_IPC_HANDLE_BYTES)()
    off = ctypes.c_uint64(0)
    _check("ep_ipc_export", lib().ep_ipc_export(_p(tensor), ctypes.byref(h), ctypes.byref(off)))
    return bytes(h), int(off.value)


def ep_ipc_open(handle, offset):
    """Map another process's exported buffer here: (base, device address);
    base is what ep_ipc_close takes."""
    if len(handle) != EP_IPC_HANDLE_BYTES:
        raise ValueError("IPC handle must be EP_IPC_HANDLE_BYTES bytes")
    h = (ctypes.c_uint8 * EP_IPC_HANDLE_BYTES).from_buffer_copy(handle)
    base, ptr = ctypes.c_void_p(0), ctypes.c_void_p(0)
    _check("ep_ipc_open", lib().ep_ipc_open(ctypes.byref(h), int(offset), ctypes.byref(base), ctypes.byref(ptr)))
    return int(base.value), int(ptr.value)


def ep_ipc_close(base):
    _check("ep_ipc_close", lib().ep_ipc_close(ctypes.c_void_p(int(base))))


def ep_plan_from_counts(counts, S, K, plan, loads=None, dev_status=None, stream=None):
    """The plan from the gathered [R, E] load matrix (the same on every rank)."""
    _dtype(counts, torch.int32)
    _dtype(plan, torch.int32)
    if loads is not None:
        _dtype(loads, torch.int32)
    R, E = counts.shape
    _check("ep_plan_from_counts", lib().ep_plan_from_counts(_p(counts), R, S, K, E, _p(loads), _p(plan), plan.numel(),
                                                            _p(dev_status), _s(stream)))


def ep_layout_rank(topk_local, rank, counts, plan, ws, pos_local, pair_slot=None, dev_status=None, stream=None):
    """Global rows of rank `rank`'s pairs; ws is the scratch ep_route_stats
    filled for topk_local."""
    for t in (topk_local, counts, plan, pos_local) + ((pair_slot,) if pair_slot is not None else ()):
        _dtype(t, torch.int32)
    S, K = topk_local.shape
    R, E = counts.shape
    _check("ep_layout_rank", lib().ep_layout_rank(_p(topk_local), S, K, E, R, rank, _p(counts), _p(plan), plan.numel(),
                                                  _p(ws), ws.numel() * ws.element_size(), _p(pos_local),
                                                  _p(pair_slot), _p(dev_status), _s(stream)))


def ep_dispatch_peer(x_local, K, pos_local, peers, rows_per_rank, total_rows, rank_first_row=None, dev_status=None,
                     stream=None):
    """Rows of x_local [S, H] to their global rows in the R rank buffers (rank
    of a row: row // rows_per_rank, or by rank_first_row when given)."""
    _dtype(x_local, torch.bfloat16, torch.int16, torch.uint16)
    _dtype(pos_local, torch.int32)
    _dtype(peers, torch.int64)
    if rank_first_row is not None:
        _dtype(rank_first_row, torch.int32)
    S, H = x_local.shape
    _check("ep_dispatch_peer", lib().ep_dispatch_peer(_p(x_local), S, K, H, _p(pos_local), _p(peers), _p(rank_first_row),
                                                      peers.numel(), rows_per_rank, total_rows, _p(dev_status),
                                                      _s(stream)))


def ep_combine_peer(peers, rows_per_rank, total_rows, w_local, pos_local, out_local, K=None, rank_first_row=None,
                    dev_status=None, stream=None):
    """out_local[t] = sum_k w_local[t,k] * row pos_local[t*K+k] of the rank
    buffers (w_local None: unit weights, the backward of dispatch; K given)."""
    _dtype(pos_local, torch.int32)
    _dtype(peers, torch.int64)
    if rank_first_row is not None:
        _dtype(rank_first_row, torch.int32)
    S, H = out_local.shape
    if w_local is not None:
        _dtype(w_local, torch.float32)
        K = w_local.shape[1]
    _check("ep_combine_peer", lib().ep_combine_peer(_p(peers), _p(rank_first_row), peers.numel(), rows_per_rank,
                                                    total_rows, _p(w_local), _p(pos_local), S, K, H, _p(out_local),
                                                    _p(dev_status), _s(stream)))


def ep_quota_counts_workspace_size(E, R):
    n = ctypes.c_size_t(0)
    _check("ep_quota_counts_workspace_size", lib().ep_quota_counts_workspace_size(E, R, ctypes.byref(n)))
    return int(n.value)


def ep_quota_plan_from_counts(counts, S, K, B, loads, plan, ws, dev_status=None, stream=None):
    """The quota-driven plan (budget B replicas per rank) from the gathered
    [R, E] load matrix; the same on every rank."""
    for t in (counts, loads, plan):
        _dtype(t, torch.int32)
    R, E = counts.shape
    _check("ep_quota_plan_from_counts",
           lib().ep_quota_plan_from_counts(_p(counts), R, S, K, E, B, _p(loads), _p(plan), plan.numel(), _p(ws),
                                           ws.numel() * ws.element_size(), _p(dev_status), _s(stream)))


def ep_quota_layout_rank(topk_local, rank, counts, plan, ws, pos_local, dev_status=None, stream=None):
    """Global rows of rank `rank`'s pairs under a quota plan; ws is the scratch
    ep_route_stats filled for topk_local."""
    for t in (topk_local, counts, plan, pos_local):
        _dtype(t, torch.int32)
    S, K = topk_local.shape
    R, E = counts.shape
    _check("ep_quota_layout_rank",
           lib().ep_quota_layout_rank(_p(topk_local), S, K, E, R, rank, _p(counts), _p(plan), plan.numel(), _p(ws),
                                      ws.numel() * ws.element_size(), _p(pos_local), _p(dev_status), _s(stream)))


def ep_replica_grad_reduce_peer(g_home_local, peers, rep_rows, rep_dtype, E, rank, plan, clear_replicas=False,
                                dev_status=None, stream=None):
    """Home rank `rank` adds its experts' replica gradients, read through the
    peer table of the R ranks' [rep_rows, n] reduce buffers, into
    g_home_local [E/R, n]."""
    _dtype(g_home_local, torch.float32)
    _dtype(plan, torch.int32)
    _dtype(peers, torch.int64)
    dt = {torch.float32: EP_DTYPE_F32, torch.bfloat16: EP_DTYPE_BF16}[rep_dtype]
    n = g_home_local.shape[1]
    _check("ep_replica_grad_reduce_peer",
           lib().ep_replica_grad_reduce_peer(_p(g_home_local), _p(peers), rep_rows, dt, n, E, peers.numel(), rank,
                                             _p(plan), plan.numel(), int(bool(clear_replicas)), _p(dev_status),
                                             _s(stream)))


def ep_quota_replica_grad_reduce_peer(g_home_local, peers, rep_rows, rep_dtype, E, rank, plan, clear_replicas=False,
                                      dev_status=None, stream=None):
    """ep_replica_grad_reduce_peer for a plan from ep_quota_plan_from_counts."""
    _dtype(g_home_local, torch.float32)
    _dtype(plan, torch.int32)
    _dtype(peers, torch.int64)
    dt = {torch.float32: EP_DTYPE_F32, torch.bfloat16: EP_DTYPE_BF16}[rep_dtype]
    n = g_home_local.shape[1]
    _check("ep_quota_replica_grad_reduce_peer",
           lib().ep_quota_replica_grad_reduce_peer(_p(g_home_local), _p(peers), rep_rows, dt, n, E, peers.numel(), rank,
                                                   _p(plan), plan.numel(), int(bool(clear_replicas)), _p(dev_status),
                                                   _s(stream)))


def ep_selftest_lookback_timeout(topk_ids, E, loads, max_vio, ws, dev_status, stream=None):
    """Failure-detection self-test: a look-back wait that runs out (see ep.h)."""
    T, K = topk_ids.shape
    _check("ep_selftest_lookback_timeout",
           lib().ep_selftest_lookback_timeout(_p(topk_ids), T, K, E, _p(loads), _p(max_vio), _p(ws),
                                              ws.numel() * ws.element_size(), _p(dev_status), _s(stream)))


def ep_status_read(dev_status, stream=None):
    h = ctypes.c_int32(0)
    _check("ep_status_read", lib().ep_status_read(_p(dev_status), ctypes.byref(h), _s(stream)))
    return int(h.value)


from .layer import EpLayer  # noqa: E402  (needs the binding above)
