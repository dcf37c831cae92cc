"""The public end-to-end call (EpLayer.run_host) gives the same result as the
device-resident step, whether or not it pipelines the host copies in slices,
and matches the oracle (-m gpu)."""
import numpy as np
import pytest

import oracle as O
import workload as W
from gpu_path import case_inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("chunks", [1, 3, 8, 11])
def test_run_host_matches_oracle(chunks):
    import torch
    import token_dispatch_histogram_b200 as tdh
    c = W.shape(2)
    R, S, E, K, H, T = c["R"], c["S"], c["E"], c["K"], c["H"], c["T"]
    S2 = 512  # a smaller token count with the workload's shape
    T2 = R * S2
    topk, w = W.routing_from(T2, E, K, seed=3, bias_e=W.bias(2, 0))
    x = W.hidden(T2, H, seed=4)
    layer = tdh.EpLayer(R, S2, K, E, H, c["block_m"], device="cuda")
    topk_h = torch.from_numpy(topk).pin_memory()
    w_h = torch.from_numpy(w).pin_memory()
    x_h = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    out_h = torch.zeros((T2, H), dtype=torch.bfloat16).pin_memory()
    layer.run_host(topk_h, w_h, x_h, out_h, grads=False, chunks=chunks)
    torch.cuda.synchronize()
    assert layer.status() == 0
    loads, mv, _ = O.route_stats(topk, E)
    pl = O.plan(loads, R, S2, K, E)
    lo = O.layout(topk, pl, R, S2, E)
    buf = O.dispatch(x, lo["pos"], K, T2 * K)
    ref = O.combine(buf, w, lo["pos"], K)
    np.testing.assert_array_equal(out_h.view(torch.int16).numpy().view(np.uint16), ref)
    _ = (S, T)


def test_overlapped_step_matches_the_sequential_one():
    """EpLayer.step(overlap=True) runs the replica gradient reduction on a
    second stream beside combine: the same outputs, bit for bit."""
    import torch
    import token_dispatch_histogram_b200 as tdh
    R, S, K, E, H, n = 8, 300, 6, 64, 256, 4096 * 3 + 8
    topk, w, x = case_inputs(R, S, K, E, H, seed=11, bias_scale=1.5)
    lay = tdh.EpLayer(R, S, K, E, H, 16, device="cuda", grad_n=n)
    lay.topk_ids.copy_(torch.from_numpy(topk))
    lay.w.copy_(torch.from_numpy(w))
    lay.x.copy_(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16))
    g0 = torch.randn((E, n), device="cuda")
    W.fill_device(lay.g_rep, 3, W.STREAM_GREP)
    outs = []
    for overlap in (False, True):
        lay.g_home.copy_(g0)
        lay.out.zero_()
        lay.step(overlap=overlap)
        torch.cuda.synchronize()
        outs.append((lay.out.clone(), lay.g_home.clone()))
    assert lay.status() == 0
    assert int(lay.plan_view("n_rep", 1).item()) > 0
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


@pytest.mark.parametrize("chunks", [1, 5, 8])
def test_run_host_layers_matches_each_layer(chunks):
    """Three layers sharing their row buffers, fed from the host with the
    layers' copies overlapped (run_host_layers): each layer's combined rows
    equal the oracle's for that layer's routing, whether every layer has its
    own output buffer or all share one (which then holds the last layer's)."""
    import torch
    import token_dispatch_histogram_b200 as tdh
    from token_dispatch_histogram_b200.layer import run_host_layers
    R, S, K, E, H, bm = 8, 384, 6, 64, 512, 64
    T = R * S
    layers = []
    for _ in range(3):
        layers.append(tdh.EpLayer(R, S, K, E, H, bm, device="cuda", share=layers[0] if layers else None))
    routes = [W.routing_from(T, E, K, seed=20 + l, bias_e=W.bias(2, l)) for l in range(3)]
    xs = [W.hidden(T, H, seed=30 + l) for l in range(3)]
    pin = lambda a: torch.from_numpy(a).pin_memory()
    topk_hs = [pin(tk) for tk, _ in routes]
    w_hs = [pin(w) for _, w in routes]
    x_hs = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in xs]
    refs = []
    for (tk, w), x in zip(routes, xs):
        loads, _, _ = O.route_stats(tk, E)
        pl = O.plan(loads, R, S, K, E)
        lo = O.layout(tk, pl, R, S, E)
        refs.append(O.combine(O.dispatch(x, lo["pos"], K, T * K), w, lo["pos"], K))
    own = [torch.zeros((T, H), dtype=torch.bfloat16).pin_memory() for _ in range(3)]
    run_host_layers(layers, topk_hs, w_hs, x_hs, own, grads=False, chunks=chunks)
    torch.cuda.synchronize()
    assert all(ly.status() == 0 for ly in layers)
    for got, ref in zip(own, refs):
        np.testing.assert_array_equal(got.view(torch.int16).numpy().view(np.uint16), ref)
    shared = torch.zeros((T, H), dtype=torch.bfloat16).pin_memory()
    run_host_layers(layers, topk_hs, w_hs, x_hs, [shared] * 3, grads=False, chunks=chunks)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(shared.view(torch.int16).numpy().view(np.uint16), refs[-1])


def _oracle_chain(routes, x, R, S, K, E):
    """The oracle's forward chain: each layer dispatches the rows the one
    before combined, through its own routing."""
    T = x.shape[0]
    want = x
    for tk, w in routes:
        loads, _, _ = O.route_stats(tk, E)
        pl = O.plan(loads, R, S, K, E)
        lo = O.layout(tk, pl, R, S, E)
        want = O.combine(O.dispatch(want, lo["pos"], K, T * K), w, lo["pos"], K)
    return want


@pytest.mark.parametrize("chunks", [1, 5, 8])
@pytest.mark.parametrize("nl", [1, 2, 3])
def test_run_host_chain_matches_the_oracle_chain(nl, chunks):
    """Layers chained on two row buffers (layer l+1 dispatches the rows layer l
    combined), fed from the host (run_host_chain): the batch's hidden rows in,
    the last layer's combined rows out, equal to the oracle's chain of
    dispatch and combine through every layer's own routing; and equal to the
    same chain run on device-resident inputs."""
    import torch
    import token_dispatch_histogram_b200 as tdh
    from token_dispatch_histogram_b200.layer import chain_buffers, run_host_chain
    R, S, K, E, H, bm = 8, 384, 6, 64, 512, 64
    T = R * S
    layers = []
    for _ in range(nl):
        layers.append(tdh.EpLayer(R, S, K, E, H, bm, device="cuda", share=layers[0] if layers else None))
    chain_buffers(layers)
    assert nl == 1 or layers[1].x.data_ptr() == layers[0].out.data_ptr()
    routes = [W.routing_from(T, E, K, seed=40 + l, bias_e=W.bias(2, l)) for l in range(nl)]
    x = W.hidden(T, H, seed=50)
    want = _oracle_chain(routes, x, R, S, K, E)
    topk_hs = [torch.from_numpy(tk).pin_memory() for tk, _ in routes]
    w_hs = [torch.from_numpy(w).pin_memory() for _, w in routes]
    x_h = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    out_h = torch.zeros((T, H), dtype=torch.bfloat16).pin_memory()
    run_host_chain(layers, topk_hs, w_hs, x_h, out_h, grads=False, chunks=chunks)
    torch.cuda.synchronize()
    assert all(ly.status() == 0 for ly in layers)
    np.testing.assert_array_equal(out_h.view(torch.int16).numpy().view(np.uint16), want)
    # the same chain on the device
    layers[0].x.copy_(x_h)
    for ly, tk in zip(layers, topk_hs):
        ly.topk_ids.copy_(tk)
    for ly, w in zip(layers, w_hs):
        ly.w.copy_(w)
    for ly in layers:
        ly.step(grads=False)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(layers[-1].out.view(torch.int16).cpu().numpy().view(np.uint16), want)


@pytest.mark.parametrize("staged", [True, False], ids=["stage_buffers", "chain_buffers"])
@pytest.mark.parametrize("nl", [1, 2, 3])
def test_run_host_batches_matches_the_oracle_chain(nl, staged):
    """Three batches in flight through a chain of layers (run_host_batches),
    each with its own routing per layer and its own hidden rows: every batch's
    combined rows, copied to its own host buffer, equal the oracle's chain for
    that batch.  With separate stage buffers batch b+1's rows arrive while
    batch b's layers still run; with the defaults (the chain's own buffers)
    the batches wait for one another."""
    import torch
    import token_dispatch_histogram_b200 as tdh
    from token_dispatch_histogram_b200.layer import chain_buffers, run_host_batches
    R, S, K, E, H, bm = 8, 384, 6, 64, 512, 64
    T = R * S
    layers = []
    for _ in range(nl):
        layers.append(tdh.EpLayer(R, S, K, E, H, bm, device="cuda", share=layers[0] if layers else None))
    chain_buffers(layers)
    batches, wants = [], []
    for b in range(3):
        routes = [W.routing_from(T, E, K, seed=100 * b + l, bias_e=W.bias(2, l + b)) for l in range(nl)]
        x = W.hidden(T, H, seed=60 + b)
        wants.append(_oracle_chain(routes, x, R, S, K, E))
        batches.append(([torch.from_numpy(tk).pin_memory() for tk, _ in routes],
                        [torch.from_numpy(w).pin_memory() for _, w in routes],
                        torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory(),
                        torch.zeros((T, H), dtype=torch.bfloat16).pin_memory()))
    xs = torch.empty_like(layers[0].x) if staged else None
    os_ = torch.empty_like(layers[0].x) if staged else None
    run_host_batches(layers, batches, xs, os_, grads=False, chunks=5)
    torch.cuda.synchronize()
    assert all(ly.status() == 0 for ly in layers)
    for (_, _, _, out_h), want in zip(batches, wants):
        np.testing.assert_array_equal(out_h.view(torch.int16).numpy().view(np.uint16), want)
