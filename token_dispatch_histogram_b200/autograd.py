"""Autograd functions for dispatch and combine (training).

The MoonEP page has the dispatched rows written straight into a static
communication buffer ("Online planning, zero copy και στατικά σχήματα"), which
the next dispatch or combine overwrites, so autograd must not keep such views
for the backward pass ("Ένα ρεαλιστικό πλαίσιο αξιολόγησης πριν από την
υιοθέτηση").  So:

- ep_dispatch_fn saves only the layout (pos); its backward is the unpermute,
  ep_dispatch_backward: dx[t] = sum_k dbuf[pos[t*K+k]] (fp32, one rounding).
- ep_combine_fn needs the expert rows y for the gate-weight gradient, so it
  saves y: the caller must keep y unchanged until the backward runs (a buffer
  per layer, or a copy).  Backward: ep_combine_backward, dy[pos[t*K+k]] =
  w[t,k] * dout[t] and dw[t,k] = <dout[t], y[pos[t*K+k]]>.

Every step runs in libep.so's kernels; these classes only allocate outputs and
route tensors.
"""
import torch

from . import ep_combine, ep_combine_backward, ep_dispatch, ep_dispatch_backward


class _Dispatch(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, pos, K, buf):
        ep_dispatch(x, K, pos, buf)
        ctx.save_for_backward(pos)
        ctx.K, ctx.T = K, x.shape[0]
        ctx.mark_dirty(buf)
        return buf

    @staticmethod
    def backward(ctx, dbuf):
        (pos,) = ctx.saved_tensors
        dx = torch.empty((ctx.T, dbuf.shape[1]), dtype=dbuf.dtype, device=dbuf.device)
        ep_dispatch_backward(dbuf.contiguous(), pos, ctx.T, ctx.K, dx)
        return dx, None, None, None


class _Combine(torch.autograd.Function):
    @staticmethod
    def forward(ctx, y, w, pos):
        T = w.shape[0]
        out = torch.empty((T, y.shape[1]), dtype=y.dtype, device=y.device)
        ep_combine(y, w, pos, out)
        ctx.save_for_backward(y, w, pos)
        return out

    @staticmethod
    def backward(ctx, dout):
        y, w, pos = ctx.saved_tensors
        dy = torch.zeros_like(y)  # rows no pair addresses get no gradient
        dw = torch.empty_like(w)
        ep_combine_backward(dout.contiguous(), w, y, pos, dy, dw)
        return dy, dw, None


def ep_dispatch_fn(x, pos, K, buf):
    """buf[pos[p]] = x[p // K] into the static buffer buf (returned); the
    backward gives dx.  buf is overwritten in place and must not be kept."""
    return _Dispatch.apply(x, pos, K, buf)


def ep_combine_fn(y, w, pos):
    """out[t] = sum_k w[t,k] * y[pos[t*K+k]]; the backward gives dy and dw.
    y is saved for the backward and must stay unchanged until then."""
    return _Combine.apply(y, w, pos)
