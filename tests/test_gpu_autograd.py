"""Autograd through dispatch and combine (-m gpu): the gradients equal the
oracle's backward (dx and dy bit for bit, dw within the fp32 summation bound)
and agree with a plain PyTorch fp32 reference of the same forward."""
import numpy as np
import pytest

import oracle as O
from gpu_path import case_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("case", [(4, 200, 4, 16, 256), (8, 128, 6, 64, 2048), (2, 300, 8, 8, 64)],
                         ids=lambda c: "R{}_S{}_K{}_E{}_H{}".format(*c))
def test_dispatch_combine_autograd(case):
    import torch
    import token_dispatch_histogram_b200 as tdh
    from token_dispatch_histogram_b200.autograd import ep_combine_fn, ep_dispatch_fn
    R, S, K, E, H = case
    topk, w, x = case_inputs(R, S, K, E, H, seed=R + S, bias_scale=1.5)
    T, P = R * S, R * S * K
    layer = tdh.EpLayer(R, S, K, E, H, 4, device="cuda")
    layer.topk_ids.copy_(torch.from_numpy(topk))
    layer.route()
    pos = layer.pos
    dev = "cuda"
    xt = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16).requires_grad_(True)
    wt = torch.from_numpy(w).to(dev).requires_grad_(True)
    buf = torch.empty((P, H), dtype=torch.bfloat16, device=dev)
    rows = ep_dispatch_fn(xt, pos, K, buf)
    y = rows * 1.0  # stand-in expert: the identity (a new tensor, so combine saves its own y)
    out = ep_combine_fn(y, wt, pos)
    g = torch.from_numpy(case_inputs(R, S, K, E, H, seed=7 * S)[2].view(np.int16)).to(dev).view(torch.bfloat16)
    out.backward(g)
    assert layer.status() == 0

    # oracle: forward and backward of the same chain
    lo_pos = pos.cpu().numpy()
    ybuf = O.dispatch(x, lo_pos, K, P)
    want_out = O.combine(ybuf, w, lo_pos, K)
    np.testing.assert_array_equal(out.detach().view(torch.int16).cpu().numpy().view(np.uint16), want_out)
    gn = g.view(torch.int16).cpu().numpy().view(np.uint16)
    dy_ref, dw_ref = O.combine_backward(gn, w, ybuf, lo_pos)
    dx_ref = O.dispatch_backward(dy_ref, lo_pos, T, K)
    np.testing.assert_array_equal(xt.grad.view(torch.int16).cpu().numpy().view(np.uint16), dx_ref)
    absum = (np.abs(O.bf16_to_f32(gn).astype(np.float64)[:, None, :]) *
             np.abs(O.bf16_to_f32(ybuf[lo_pos.reshape(T, K)]).astype(np.float64))).sum(axis=2)
    assert np.all(np.abs(wt.grad.cpu().numpy().astype(np.float64) - dw_ref) <= H * 2.0 ** -24 * absum + 1e-30)

    # plain PyTorch fp32 reference of the same forward
    xr = torch.from_numpy(O.bf16_to_f32(x)).to(dev).requires_grad_(True)
    wr = torch.from_numpy(w).to(dev).requires_grad_(True)
    p = pos.long().view(T, K)
    src_tok = torch.empty(P, dtype=torch.long, device=dev)
    src_tok[pos.long()] = torch.arange(P, device=dev) // K
    bufr = xr[src_tok]
    outr = (wr[:, :, None] * bufr[p]).sum(dim=1)
    outr.backward(g.float())
    tol = dict(rtol=2 ** -7, atol=1e-2)
    torch.testing.assert_close(out.float(), outr.detach(), **tol)
    torch.testing.assert_close(xt.grad.float(), xr.grad, **tol)
    torch.testing.assert_close(wt.grad, wr.grad, rtol=1e-3, atol=1e-2)
