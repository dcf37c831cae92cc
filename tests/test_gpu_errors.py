"""Failure detection on the GPU without a GPU fault (-m gpu).

Bad inputs are made on the host (ids outside [0, E), loads that do not add
up, row indices outside the buffer, buffers too small); the kernels report
them as EP_DEV_* bits in the caller's status word, write nothing out of
bounds, and the context stays usable.  The bounded look-back wait is made to
run out for real (a flag that nothing sets) and must report a timeout.
The dispatch kernel's wait on its own TMA copies has the same bound but cannot
be made to run out without a faulting copy, so it is not exercised here.
"""
import numpy as np
import pytest

import oracle as O
import workload as W

pytestmark = pytest.mark.gpu


def _t(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to("cuda") if dtype is None else t.to("cuda").view(dtype)


def test_bad_expert_ids_are_flagged_and_skipped():
    import torch
    import token_dispatch_histogram_b200 as tdh
    T, K, E = 5000, 4, 32
    topk, _ = W.routing_from(T, E, K, seed=3)
    topk[7, 1] = E
    topk[4000, 0] = -5
    d = _t(topk)
    loads = torch.zeros(E, dtype=torch.int32, device="cuda")
    mv = torch.zeros(1, dtype=torch.float64, device="cuda")
    ws = torch.zeros(tdh.ep_workspace_size(T, K, E), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tdh.ep_route_stats(d, E, loads, mv, ws, st)
    assert tdh.ep_status_read(st) & tdh.EP_DEV_BAD_EXPERT_ID
    ref, _, bad = O.route_stats(topk, E)
    assert bad == 2
    np.testing.assert_array_equal(loads.cpu().numpy(), ref)
    # the plan sees loads that no longer sum to R*S*K
    st.zero_()
    lay = tdh.ep_plan_layout(E, 4)
    plan = torch.zeros(lay["words"], dtype=torch.int32, device="cuda")
    tdh.ep_plan(loads, 4, T // 4, K, E, plan, st)
    assert tdh.ep_status_read(st) & tdh.EP_DEV_BAD_LOADS
    assert int(plan[lay["n_rep"]].item()) == 0
    # align-sort flags too and places only the valid pairs
    st.zero_()
    cap, capb = tdh.align_sort_capacity(T * K, E, 16)
    ids = torch.full((cap,), -9, dtype=torch.int32, device="cuda")
    eids = torch.full((capb,), -9, dtype=torch.int32, device="cuda")
    n = torch.zeros(1, dtype=torch.int32, device="cuda")
    tdh.ep_align_sort(d, E, 16, ids, eids, n, ws, st)
    assert tdh.ep_status_read(st) & tdh.EP_DEV_BAD_EXPERT_ID
    oids, oeids, on = O.align_sort(topk, E, 16)
    np.testing.assert_array_equal(ids.cpu().numpy(), oids)
    np.testing.assert_array_equal(eids.cpu().numpy(), oeids)


def test_rows_outside_the_buffer_are_flagged_and_skipped():
    import torch
    import token_dispatch_histogram_b200 as tdh
    T, K, H = 64, 2, 32
    x = W.hidden(T, H, seed=4)
    rng = np.random.default_rng(0)
    pos = rng.permutation(T * K).astype(np.int32)
    pos[3] = T * K + 11     # past the end
    pos[70] = -2            # negative
    buf = torch.full((T * K, H), 0x1234, dtype=torch.int16, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tdh.ep_dispatch(_t(x, torch.bfloat16), K, _t(pos), buf, st)
    assert tdh.ep_status_read(st) & tdh.EP_DEV_BAD_ROW
    got = buf.cpu().numpy().view(np.uint16)
    good = (pos >= 0) & (pos < T * K)
    np.testing.assert_array_equal(got[pos[good]], np.repeat(x, K, axis=0)[good])
    untouched = np.setdiff1d(np.arange(T * K), pos[good])
    assert np.all(got[untouched] == 0x1234)
    # combine: the same pairs contribute nothing
    st.zero_()
    w = rng.uniform(0, 1, (T, K)).astype(np.float32)
    y = W.hidden(T * K, H, seed=5)
    out = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
    tdh.ep_combine(_t(y, torch.bfloat16), _t(w), _t(pos), out, st)
    assert tdh.ep_status_read(st) & tdh.EP_DEV_BAD_ROW
    opos = np.where(good, pos, -1).astype(np.int32)
    np.testing.assert_array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), O.combine(y, w, opos, K))


def test_capacity_and_argument_errors_raise():
    import torch
    import token_dispatch_histogram_b200 as tdh
    d = _t(np.zeros((100, 2), dtype=np.int32))
    small = torch.zeros(8, dtype=torch.uint8, device="cuda")
    with pytest.raises(tdh.EpError) as e:
        tdh.ep_route_stats(d, 8, torch.zeros(8, dtype=torch.int32, device="cuda"),
                           torch.zeros(1, dtype=torch.float64, device="cuda"), small)
    assert e.value.code == tdh.EP_ERR_CAPACITY
    with pytest.raises(tdh.EpError) as e:
        tdh.ep_plan(torch.zeros(10, dtype=torch.int32, device="cuda"), 4, 25, 2, 10,
                    torch.zeros(10_000, dtype=torch.int32, device="cuda"))
    assert e.value.code == tdh.EP_ERR_ARG


def test_lookback_wait_runs_out_and_context_survives():
    import torch
    import token_dispatch_histogram_b200 as tdh
    T, K, E = 4096, 4, 16                  # 16,384 pairs: 8 tiles
    topk, _ = W.routing_from(T, E, K, seed=9)
    d = _t(topk)
    loads = torch.zeros(E, dtype=torch.int32, device="cuda")
    mv = torch.zeros(1, dtype=torch.float64, device="cuda")
    ws = torch.zeros(tdh.ep_workspace_size(T, K, E), dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    tdh.ep_selftest_lookback_timeout(d, E, loads, mv, ws, st)
    assert tdh.ep_status_read(st) & tdh.EP_DEV_LOOKBACK_TIMEOUT
    # the context is still usable: a normal call on the same workspace is exact
    st.zero_()
    tdh.ep_route_stats(d, E, loads, mv, ws, st)
    assert tdh.ep_status_read(st) == 0
    ref, ref_mv, _ = O.route_stats(topk, E)
    np.testing.assert_array_equal(loads.cpu().numpy(), ref)
    assert float(mv.item()) == ref_mv
