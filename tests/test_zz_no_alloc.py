"""ep_route_stats_noalloc: the route-statistics call for callers that cannot
allocate device scratch (hosts that hand a kernel only its inputs and outputs
at enqueue time, runtimes whose memory is planned in advance).  It keeps its
scratch in a fixed array inside libep.so instead of a caller workspace.

Checked through the C ABI against ep_route_stats (which takes a workspace)
and against the CPU oracle: loads and max_vio must agree exactly (integer
counts, and max_vio is the same fp64 expression), on several calls in a row
that reuse the shared array; after the first call no further call changes the
device's free memory; and a problem larger than the array must be refused
before anything is enqueued.  This file is collected last on purpose, and
each test also runs on its own.
"""
import ctypes

import numpy as np
import pytest

import oracle as O
import workload as W

pytestmark = pytest.mark.gpu


def _call_both(topk_np, E):
    import torch
    import token_dispatch_histogram_b200 as tdh
    L = tdh.lib()
    dev = torch.device("cuda")
    topk = torch.from_numpy(np.ascontiguousarray(topk_np, dtype=np.int32)).to(dev)
    T, K = topk.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    loads_a = torch.full((E,), -1, dtype=torch.int32, device=dev)
    mv_a = torch.full((1,), -1.0, dtype=torch.float64, device=dev)
    rc = L.ep_route_stats_noalloc(ctypes.c_void_p(topk.data_ptr()), T, K, E, ctypes.c_void_p(loads_a.data_ptr()),
                                  ctypes.c_void_p(mv_a.data_ptr()), ctypes.c_void_p(status.data_ptr()), stream)
    assert rc == 0
    ws = torch.zeros(tdh.ep_workspace_size(T, K, E), dtype=torch.uint8, device=dev)
    loads_b = torch.full((E,), -2, dtype=torch.int32, device=dev)
    mv_b = torch.full((1,), -2.0, dtype=torch.float64, device=dev)
    rc = L.ep_route_stats(ctypes.c_void_p(topk.data_ptr()), T, K, E, ctypes.c_void_p(loads_b.data_ptr()),
                          ctypes.c_void_p(mv_b.data_ptr()), ctypes.c_void_p(ws.data_ptr()), ws.numel(),
                          ctypes.c_void_p(status.data_ptr()), stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return (loads_a.cpu().numpy(), float(mv_a.item())), (loads_b.cpu().numpy(), float(mv_b.item()))


def test_noalloc_matches_route_stats_on_consecutive_calls():
    cases = [(2, 0), (5, 0), (1, 3), (2, 1)]  # moderate, adversarial prefill (1.5 MB of scratch), tiny, moderate
    for cfg, seed in cases:
        c = W.shape(cfg)
        topk, _ = W.routing(cfg, seed)
        (la, ma), (lb, mb) = _call_both(topk, c["E"])
        np.testing.assert_array_equal(la, lb)
        assert ma == mb
        lo, mo, bad = O.route_stats(topk, c["E"])
        assert bad == 0
        np.testing.assert_array_equal(la, lo)
        assert ma == mo


def test_noalloc_calls_leave_free_memory_unchanged():
    """Once the first call has run, further calls allocate nothing: the
    device's free memory (cudaMemGetInfo) is the same after twenty calls."""
    import torch
    import token_dispatch_histogram_b200 as tdh
    L = tdh.lib()
    c = W.shape(5)
    topk_np, _ = W.routing(5, 0)
    dev = torch.device("cuda")
    topk = torch.from_numpy(topk_np).to(dev)
    loads = torch.zeros(c["E"], dtype=torch.int32, device=dev)
    mv = torch.zeros(1, dtype=torch.float64, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    args = (ctypes.c_void_p(topk.data_ptr()), c["T"], c["K"], c["E"], ctypes.c_void_p(loads.data_ptr()),
            ctypes.c_void_p(mv.data_ptr()), ctypes.c_void_p(status.data_ptr()), stream)
    assert L.ep_route_stats_noalloc(*args) == 0
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(20):
        assert L.ep_route_stats_noalloc(*args) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert int(status.item()) == 0
    lo, mo, _ = O.route_stats(topk_np, c["E"])
    np.testing.assert_array_equal(loads.cpu().numpy(), lo)
    assert float(mv.item()) == mo


def test_noalloc_refuses_problems_larger_than_its_array():
    import torch
    import token_dispatch_histogram_b200 as tdh
    L = tdh.lib()
    fake = ctypes.c_void_p(0x1000)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # E = 1024 with 2^26 pairs needs 12 * 8192 tiles * 1024 ~ 100 MB of scratch
    rc = L.ep_route_stats_noalloc(fake, 1 << 23, 8, 1024, fake, fake, None, stream)
    assert rc == tdh.EP_ERR_CAPACITY
