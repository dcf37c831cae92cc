"""The C ABI library loads and exports every entry point include/ep.h declares,
and its host-side logic (sizes, plan layout, argument checks) works without a
GPU.  No compute call is made here."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ep.h")


def declared():
    text = open(HEADER).read()
    return re.findall(r"EP_API\s+[\w\s\*]+?\b(ep_\w+)\s*\(", text)


def test_header_declares_the_path():
    names = set(declared())
    for n in ("ep_route_stats", "ep_plan", "ep_layout", "ep_align_sort", "ep_dispatch", "ep_combine",
              "ep_replica_grad_reduce", "ep_workspace_size", "ep_plan_layout", "ep_status_read"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import token_dispatch_histogram_b200 as tdh
    L = ctypes.CDLL(tdh.LIB_PATH)
    for name in declared():
        assert hasattr(L, name), name


def test_binding_has_same_names():
    import token_dispatch_histogram_b200 as tdh
    for name in declared():
        if name in ("ep_version",):
            continue
        assert hasattr(tdh, name), name


def test_host_only_calls():
    import token_dispatch_histogram_b200 as tdh
    assert "sm_100a" in tdh.version()
    lay = tdh.ep_plan_layout(64, 8)
    assert lay["cap"] == 64 + 8 - 1
    offs = sorted(v for k, v in lay.items() if k not in ("words", "cap"))
    assert len(set(offs)) == len(offs) and offs[-1] < lay["words"]
    assert all(v % 8 == 0 for k, v in lay.items() if k not in ("words", "cap"))
    # workspace grows with the tile count and E
    a = tdh.ep_workspace_size(32768, 6, 64)
    b = tdh.ep_workspace_size(524288, 8, 384)
    assert 0 < a < b
    assert tdh.ep_workspace_size(0, 2, 16) > 0


def test_argument_errors_return_before_any_launch():
    import token_dispatch_histogram_b200 as tdh
    L = tdh.lib()
    n = ctypes.c_size_t()
    assert L.ep_workspace_size(10, 0, 8, ctypes.byref(n)) == tdh.EP_ERR_ARG      # K < 1
    assert L.ep_workspace_size(10, 9, 8, ctypes.byref(n)) == tdh.EP_ERR_ARG      # K > E
    assert L.ep_workspace_size(10, 2, 2000, ctypes.byref(n)) == tdh.EP_ERR_ARG   # E > max
    assert L.ep_workspace_size(1 << 30, 4, 8, ctypes.byref(n)) == tdh.EP_ERR_ARG  # P >= 2^31
    lay = tdh.EpPlanLayout()
    assert L.ep_plan_layout(10, 4, ctypes.byref(lay)) == tdh.EP_ERR_ARG          # E % R
    fake = ctypes.c_void_p(0x1000)
    # ep_plan: E % R != 0
    assert L.ep_plan(fake, 3, 4, 2, 8, fake, 1 << 20, None, None) == tdh.EP_ERR_ARG
    # ep_plan: plan buffer too small
    assert L.ep_plan(fake, 4, 4, 2, 8, fake, 3, None, None) == tdh.EP_ERR_CAPACITY
    # ep_route_stats: workspace too small
    assert L.ep_route_stats(fake, 16, 2, 8, fake, fake, fake, 8, None, None) == tdh.EP_ERR_CAPACITY
    # ep_layout: R*S != T
    assert L.ep_layout(fake, 16, 2, 8, 4, 5, fake, 1 << 20, fake, 1 << 20, fake, fake, None, None,
                       None) == tdh.EP_ERR_ARG
    # ep_align_sort: sorted capacity too small
    assert L.ep_align_sort(fake, 16, 2, 8, 4, fake, 10, fake, 100, fake, fake, 1 << 20, None,
                           None) == tdh.EP_ERR_CAPACITY
    # ep_dispatch / ep_combine: H not a multiple of 8, misaligned pointers
    assert L.ep_dispatch(fake, 16, 2, 12, fake, fake, 32, None, None) == tdh.EP_ERR_ARG
    assert L.ep_dispatch(ctypes.c_void_p(0x1008), 16, 2, 16, fake, fake, 32, None, None) == tdh.EP_ERR_ARG
    assert L.ep_combine(fake, 32, fake, fake, 16, 2, 12, fake, None, None) == tdh.EP_ERR_ARG
    assert L.ep_combine(fake, 32, fake, fake, 16, 33, 16, fake, None, None) == tdh.EP_ERR_ARG  # K > 32
    # grad reduce: bad dtype, plan too small
    assert L.ep_replica_grad_reduce(fake, fake, 7, 8, 8, 4, fake, 1 << 20, 0, None, None) == tdh.EP_ERR_ARG
    assert L.ep_replica_grad_reduce(fake, fake, 0, 8, 8, 4, fake, 3, 0, None, None) == tdh.EP_ERR_CAPACITY
    # a row wider than two shared-memory stages (about 100 KB) is refused
    assert L.ep_dispatch(fake, 16, 2, 51200, fake, fake, 32, None, None) == tdh.EP_ERR_ARG
    # fused layout + dispatch: the route's checks, then the dispatch's (before anything is enqueued)
    def rdf(x, H, R=4, S=4):
        return L.ep_route_dispatch_fused(fake, R * S, 2, 8, R, S, fake, fake, fake, 1 << 20, fake, fake, None, 4,
                                         None, 0, None, 0, None, x, H, fake, 32, fake, 1 << 20, None, None)
    assert rdf(None, 16) == tdh.EP_ERR_ARG                       # no x
    assert rdf(fake, 12) == tdh.EP_ERR_ARG                       # H % 8
    assert rdf(fake, 51200) == tdh.EP_ERR_ARG                    # rows the dispatch kernel refuses
    assert rdf(ctypes.c_void_p(0x1008), 16) == tdh.EP_ERR_ARG    # misaligned x
    assert rdf(fake, 16, R=3) == tdh.EP_ERR_ARG                  # E % R
    # zero-size work is a no-op that succeeds without touching the device
    assert L.ep_dispatch(None, 0, 2, 16, None, None, 0, None, None) == tdh.EP_OK
    assert L.ep_combine(None, 0, None, None, 0, 2, 16, None, None, None) == tdh.EP_OK


def test_binding_rejects_cpu_tensors():
    import torch
    import token_dispatch_histogram_b200 as tdh
    t = torch.zeros((4, 2), dtype=torch.int32)
    with pytest.raises(ValueError):
        tdh.ep_route_stats(t, 8, torch.zeros(8, dtype=torch.int32), torch.zeros(1, dtype=torch.float64),
                           torch.zeros(64, dtype=torch.uint8))


def test_rank_local_and_quota_argument_errors():
    """The rank-local and quota entry points refuse bad shapes and short
    buffers on the host, before anything is enqueued (no GPU needed)."""
    import token_dispatch_histogram_b200 as tdh
    L = tdh.lib()
    fake = ctypes.c_void_p(0x1000)
    n = ctypes.c_size_t()
    # plan from the gathered matrix: E % R, plan buffer too small
    assert L.ep_plan_from_counts(fake, 3, 4, 2, 8, None, fake, 1 << 20, None, None) == tdh.EP_ERR_ARG
    assert L.ep_plan_from_counts(fake, 4, 4, 2, 8, None, fake, 3, None, None) == tdh.EP_ERR_CAPACITY
    # rank-local layout: rank outside [0, R), missing counts, short workspace
    assert L.ep_layout_rank(fake, 16, 2, 8, 4, 4, fake, fake, 1 << 20, fake, 1 << 20, fake, None, None,
                            None) == tdh.EP_ERR_ARG
    assert L.ep_layout_rank(fake, 16, 2, 8, 4, 0, None, fake, 1 << 20, fake, 1 << 20, fake, None, None,
                            None) == tdh.EP_ERR_ARG
    assert L.ep_layout_rank(fake, 16, 2, 8, 4, 0, fake, fake, 1 << 20, fake, 8, fake, None, None,
                            None) == tdh.EP_ERR_CAPACITY
    # peer dispatch / combine: H not a multiple of 8, no peer table, K > 8 for combine, misaligned rows
    assert L.ep_dispatch_peer(fake, 16, 2, 12, fake, fake, None, 4, 32, 128, None, None) == tdh.EP_ERR_ARG
    assert L.ep_dispatch_peer(fake, 16, 2, 16, fake, None, None, 4, 32, 128, None, None) == tdh.EP_ERR_ARG
    assert L.ep_dispatch_peer(ctypes.c_void_p(0x1008), 16, 2, 16, fake, fake, None, 4, 32, 128, None,
                              None) == tdh.EP_ERR_ARG
    assert L.ep_combine_peer(fake, None, 4, 32, 128, fake, fake, 16, 9, 16, fake, None, None) == tdh.EP_ERR_ARG
    assert L.ep_combine_peer(None, None, 4, 32, 128, fake, fake, 16, 2, 16, fake, None, None) == tdh.EP_ERR_ARG
    assert L.ep_dispatch_peer(None, 0, 2, 16, None, fake, None, 4, 32, 0, None, None) == tdh.EP_OK
    # peer replica gradients: rank outside [0, R), negative rows, bad dtype, plan too small
    assert L.ep_replica_grad_reduce_peer(fake, fake, 8, 0, 16, 8, 4, 4, fake, 1 << 20, 0, None,
                                         None) == tdh.EP_ERR_ARG
    assert L.ep_replica_grad_reduce_peer(fake, fake, -1, 0, 16, 8, 4, 0, fake, 1 << 20, 0, None,
                                         None) == tdh.EP_ERR_ARG
    assert L.ep_replica_grad_reduce_peer(fake, fake, 8, 5, 16, 8, 4, 0, fake, 1 << 20, 0, None,
                                         None) == tdh.EP_ERR_ARG
    assert L.ep_replica_grad_reduce_peer(fake, fake, 8, 0, 16, 8, 4, 0, fake, 3, 0, None,
                                         None) == tdh.EP_ERR_CAPACITY
    # quota planner from the gathered matrix: B < 0, short workspace, plan too small
    assert L.ep_quota_counts_workspace_size(8, 4, ctypes.byref(n)) == tdh.EP_OK and n.value > 0
    assert L.ep_quota_counts_workspace_size(10, 4, ctypes.byref(n)) == tdh.EP_ERR_ARG
    assert L.ep_quota_plan_from_counts(fake, 4, 4, 2, 8, -1, fake, fake, 1 << 20, fake, 1 << 20, None,
                                       None) == tdh.EP_ERR_ARG
    assert L.ep_quota_plan_from_counts(fake, 4, 4, 2, 8, 1, fake, fake, 1 << 20, fake, 16, None,
                                       None) == tdh.EP_ERR_CAPACITY
    assert L.ep_quota_plan_from_counts(fake, 4, 4, 2, 8, 1, fake, fake, 3, fake, 1 << 20, None,
                                       None) == tdh.EP_ERR_CAPACITY
    assert L.ep_quota_layout_rank(fake, 16, 2, 8, 4, -1, fake, fake, 1 << 20, fake, 1 << 20, fake, None,
                                  None) == tdh.EP_ERR_ARG
    assert L.ep_quota_replica_grad_reduce_peer(fake, fake, 8, 0, 16, 8, 4, 0, fake, 3, 0, None,
                                               None) == tdh.EP_ERR_CAPACITY
    # quota route: T not R*S, B < 0, workspace too small
    assert L.ep_quota_route(fake, 17, 2, 8, 4, 4, 1, fake, fake, 1 << 20, fake, fake, fake, 1 << 20, None,
                            None) == tdh.EP_ERR_ARG
    assert L.ep_quota_route(fake, 16, 2, 8, 4, 4, -1, fake, fake, 1 << 20, fake, fake, fake, 1 << 20, None,
                            None) == tdh.EP_ERR_ARG
    assert L.ep_quota_route(fake, 16, 2, 8, 4, 4, 1, fake, fake, 1 << 20, fake, fake, fake, 16, None,
                            None) == tdh.EP_ERR_CAPACITY


def test_missing_library_fails_loudly_and_build_does_not_need_it():
    """Without libep.so the package does not import (no CPU fallback), and the
    build entry point reaches its build script without importing the package."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    hide = ("import os; real = os.path.exists; "
            "os.path.exists = lambda p: False if str(p).endswith('libep.so') else real(p); ")
    r = subprocess.run([sys.executable, "-c", hide + "import token_dispatch_histogram_b200"], cwd=root,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode != 0 and "ImportError" in r.stderr and "not built" in r.stderr
    probe = (hide + "import sys, __graft_entry__ as g; "
             "b = g._load_by_path('_b', os.path.join(g.ROOT, 'token_dispatch_histogram_b200', 'build.py')); "
             "assert callable(b.build) and 'token_dispatch_histogram_b200' not in sys.modules; print('ok')")
    r = subprocess.run([sys.executable, "-c", probe], cwd=root, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stderr
