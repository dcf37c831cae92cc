"""Backward of dispatch and combine on the GPU vs the CPU oracle (-m gpu).

dx (backward of dispatch) and dy (backward of combine) are bit-exact: the same
fp32 operations in the same order.  dw is an fp32 reduction in the kernel's own
order, checked against the oracle's fp64 value within the summation bound
H * 2^-24 * sum_h |dout * y|.  Every case compares every element: the small
ones at once, the full-size workloads token chunk by token chunk.
"""
import numpy as np
import pytest

import oracle as O
import workload as W
from gpu_path import case_inputs

pytestmark = pytest.mark.gpu


def _dev(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a)).to("cuda")
    return t.view(dtype) if dtype is not None else t


def _run(topk, w, R, S, E, H, seed, rows_extra=0):
    import torch
    import token_dispatch_histogram_b200 as tdh
    T, K = topk.shape
    P = T * K
    layer = tdh.EpLayer(R, S, K, E, 8, 4, device="cuda")
    layer.topk_ids.copy_(torch.from_numpy(topk))
    layer.route()
    pos = layer.pos.cpu().numpy()
    rows = P + rows_extra
    dout = W.hidden(T, H, seed=seed)
    y = W.hidden(rows, H, seed=seed + 1)
    dbuf = W.hidden(rows, H, seed=seed + 2)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dx = torch.zeros((T, H), dtype=torch.int16, device="cuda")
    tdh.ep_dispatch_backward(_dev(dbuf.view(np.int16)), layer.pos, T, K, dx, st)
    dy = torch.full((rows, H), 0x1234, dtype=torch.int16, device="cuda")
    dw = torch.zeros((T, K), dtype=torch.float32, device="cuda")
    tdh.ep_combine_backward(_dev(dout.view(np.int16)), _dev(w), _dev(y.view(np.int16)), layer.pos, dy, dw, st)
    assert tdh.ep_status_read(st) == 0
    return pos, dout, y, dbuf, dx.cpu().numpy().view(np.uint16), dy.cpu().numpy().view(np.uint16), dw.cpu().numpy()


@pytest.mark.parametrize("case", [(4, 64, 2, 16, 128), (8, 256, 6, 64, 2048), (4, 97, 8, 32, 7168),
                                  (2, 50, 1, 4, 64), (3, 33, 5, 9, 24), (16, 64, 8, 256, 4096),
                                  # odd K with one token per warp: the per-warp shared-memory regions' alignment
                                  (4, 100, 3, 16, 2048), (4, 61, 5, 16, 1024), (2, 90, 7, 8, 520)],
                         ids=lambda c: "R{}_S{}_K{}_E{}_H{}".format(*c))
def test_backward_matches_oracle(case):
    R, S, K, E, H = case
    topk, w, _ = case_inputs(R, S, K, E, 0, seed=H + K)
    pos, dout, y, dbuf, dx, dy, dw = _run(topk, w, R, S, E, H, seed=H, rows_extra=3)
    T = R * S
    np.testing.assert_array_equal(dx, O.dispatch_backward(dbuf, pos, T, K))
    init = np.full_like(y, 0x1234)
    dy_ref, dw_ref = O.combine_backward(dout, w, y, pos, dy_init=init)
    np.testing.assert_array_equal(dy, dy_ref)  # including the 3 rows no pair addresses
    absum = np.einsum("th,tkh->tk", np.abs(O.bf16_to_f32(dout).astype(np.float64)),
                      np.abs(O.bf16_to_f32(y).astype(np.float64)[pos].reshape(T, K, H)))
    assert np.all(np.abs(dw.astype(np.float64) - dw_ref) <= H * 2.0 ** -24 * absum + 1e-30)


def _bwd_chunk_ok(t0, t1, rows, got_dx, got_dy, got_dw, dout_h, y_h, w, K, H):
    """One token chunk of the full-size backward against the oracle: dx of
    every token, the dy row of every pair, every dw (within the fp32 bound)."""
    y = y_h[rows]
    dout = dout_h[t0:t1]
    local = np.arange(len(rows), dtype=np.int32)
    np.testing.assert_array_equal(got_dx, O.dispatch_backward(y, local, t1 - t0, K))
    dy_ref, dw_ref = O.combine_backward(dout, w[t0:t1], y, local)
    np.testing.assert_array_equal(got_dy, dy_ref)
    absum = np.einsum("th,tkh->tk", np.abs(O.bf16_to_f32(dout).astype(np.float64)),
                      np.abs(O.bf16_to_f32(y).astype(np.float64)).reshape(t1 - t0, K, H))
    assert np.all(np.abs(got_dw.astype(np.float64) - dw_ref) <= H * 2.0 ** -24 * absum + 1e-30)


@pytest.mark.parametrize("cfg", [2, 3])
def test_backward_full_size(cfg):
    """Every output of both backward kernels at the workload's full size, in
    token chunks: the inputs (dout, y) regenerated on the host from the
    counter-based generator, the expected values from the oracle."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    import torch
    import token_dispatch_histogram_b200 as tdh
    c = W.shape(cfg)
    R, S, E, K, H, T, P = c["R"], c["S"], c["E"], c["K"], c["H"], c["T"], c["P"]
    topk, w = W.routing(cfg, 0)
    layer = tdh.EpLayer(R, S, K, E, H, c["block_m"], device="cuda")
    layer.topk_ids.copy_(torch.from_numpy(topk))
    layer.w.copy_(torch.from_numpy(w))
    layer.route()
    W.fill_device(layer.out, 0, 0x600)   # dout
    W.fill_device(layer.buf, 0, 0x601)   # y (and the dispatch backward's dbuf)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    dx = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    tdh.ep_dispatch_backward(layer.buf, layer.pos, T, K, dx, st)
    dy = torch.empty_like(layer.buf)
    dw = torch.empty((T, K), dtype=torch.float32, device="cuda")
    tdh.ep_combine_backward(layer.out, layer.w, layer.buf, layer.pos, dy, dw, st)
    assert tdh.ep_status_read(st) == 0
    pos = layer.pos.cpu().numpy().astype(np.int64)
    dout_h = W.normal_bf16(0, 0x600, 0, T * H).reshape(T, H)
    y_h = W.normal_bf16(0, 0x601, 0, P * H).reshape(P, H)
    dw_all = dw.cpu().numpy()
    ch = max(1, (1 << 24) // (K * H))
    workers = max(2, min(32, os.cpu_count() or 2))
    with ThreadPoolExecutor(workers) as ex:
        futs = []
        for t0 in range(0, T, ch):
            t1 = min(T, t0 + ch)
            rows = pos[t0 * K:t1 * K]
            trows = torch.from_numpy(rows).cuda()
            got_dx = dx[t0:t1].view(torch.int16).cpu().numpy().view(np.uint16)
            got_dy = dy.index_select(0, trows).view(torch.int16).cpu().numpy().view(np.uint16)
            futs.append(ex.submit(_bwd_chunk_ok, t0, t1, rows, got_dx, got_dy, dw_all[t0:t1], dout_h, y_h, w, K, H))
            while len(futs) > 2 * workers:
                futs.pop(0).result()
        for f in futs:
            f.result()
