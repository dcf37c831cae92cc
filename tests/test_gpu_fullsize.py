"""Parity at the full workload sizes (-m gpu), in the launch configuration the
benchmark uses (the same binding and EpLayer buffers).

  * loads, max_vio, plan, layout (pos, src, pair_slot), cu_seqlens, align-sort:
    compared in full, bit-exact, against the CPU oracle;
  * dispatch: sampled buffer rows (every slot's first and last row plus random
    rows) must equal the hidden row of their pair's token, bitwise, with x
    regenerated on the host from the counter-based generator;
  * combine (after the stand-in expert): sampled tokens against the layout-free
    closed form, within 1 bf16 ulp (and checked identical);
  * replica gradient reduction: sampled columns of every expert row, fp32 adds
    in match order, within 1e-6 relative (and checked identical).

Workloads: moderate EP8 (R=8, S=4096, E=64, K=6, H=2048), DeepSeek-V3-shaped
(R=32, S=4096, E=256, K=8, H=7168, bf16 replica grads), fine-grained 8-layer
(R=64, S=8192, E=384, K=8, H=7168, bias redrawn per layer), adversarial
prefill (R=16, S=16384, E=256, K=8, H=4096) with its uniform and single-expert
companions.
"""
import numpy as np
import pytest

import oracle as O
import workload as W
from gpu_path import bf16_ulp_diff

pytestmark = pytest.mark.gpu


def _layer(c, dev, grads=False):
    import torch
    import token_dispatch_histogram_b200 as tdh
    gdt = torch.bfloat16 if c["grad_dtype"] == "bf16" else torch.float32
    return tdh.EpLayer(c["R"], c["S"], c["K"], c["E"], c["H"], c["block_m"], device=dev,
                       grad_n=(c["grad_n"] if grads else 0), grad_dtype=gdt, with_pair_slot=True)


def _check_route(layer, c, topk):
    R, S, K, E = c["R"], c["S"], c["K"], c["E"]
    loads, mv, _ = O.route_stats(topk, E)
    pl = O.plan(loads, R, S, K, E)
    lo = O.layout(topk, pl, R, S, E)
    ids, eids, ntpp = O.align_sort(topk, E, c["block_m"])
    n = pl["n_rep"]
    assert np.array_equal(layer.loads.cpu().numpy(), loads)
    assert float(layer.max_vio.item()) == mv
    assert int(layer.plan_view("n_rep", 1).item()) == n
    for name in ("rep_expert", "rep_rank", "rep_count"):
        assert np.array_equal(layer.plan_view(name, n).cpu().numpy(), pl[name]), name
    assert np.array_equal(layer.plan_view("home_count", E).cpu().numpy(), pl["home_count"])
    assert np.array_equal(layer.plan_view("slot_order", E + n).cpu().numpy(), lo["slot_order"])
    assert np.array_equal(layer.plan_view("cu_seqlens", E + n + 1).cpu().numpy(), lo["cu_seqlens"])
    assert np.array_equal(layer.pos.cpu().numpy(), lo["pos"])
    assert np.array_equal(layer.src.cpu().numpy(), lo["src"])
    assert np.array_equal(layer.pair_slot.cpu().numpy(), lo["pair_slot"])
    assert np.array_equal(layer.sorted_token_ids.cpu().numpy(), ids)
    assert np.array_equal(layer.expert_ids.cpu().numpy(), eids)
    assert int(layer.num_tokens_post_pad.item()) == ntpp
    return pl, lo, mv


def _check_rows(layer, c, topk, w, lo, seed, layer_id, rng):
    import torch
    K, H, T, P = c["K"], c["H"], c["T"], c["P"]
    cu = lo["cu_seqlens"].astype(np.int64)
    edge = np.concatenate([cu[:-1][np.diff(cu) > 0], cu[1:][np.diff(cu) > 0] - 1])
    rows = np.unique(np.concatenate([edge, rng.integers(0, P, 2048)]))
    src = lo["src"].astype(np.int64)
    toks = src[rows] // K
    got = layer.buf.index_select(0, torch.from_numpy(rows).to(layer.buf.device)).view(torch.int16).cpu().numpy()
    want = W.hidden_rows(H, seed, layer_id, toks)
    assert np.array_equal(got.view(np.uint16), want), "dispatch rows differ"
    # stand-in expert, then combine; sampled tokens against the closed form
    scale = W.expert_scale(c["E"])
    layer.expert_standin(torch.from_numpy(scale).to(layer.buf.device))
    layer.combine()
    tok = np.unique(np.concatenate([rng.integers(0, T, 1024), toks[:512], [0, T - 1]]))
    got = layer.out.index_select(0, torch.from_numpy(tok).to(layer.out.device)).view(torch.int16).cpu().numpy()
    want = O.combine_closed(W.hidden_rows(H, seed, layer_id, tok), w[tok], topk[tok], scale)
    ulp = bf16_ulp_diff(got.view(np.uint16), want)
    assert ulp.max() <= 1
    assert np.count_nonzero(ulp) == 0


def _run_layer(cfg, seed, layer_id=0, variant="default", rows=True, grads=False, fused=True):
    import torch
    c = W.shape(cfg)
    dev = torch.device("cuda")
    topk, w = W.routing(cfg, seed, layer_id, variant)
    layer = _layer(c, dev, grads)
    layer.topk_ids.copy_(torch.from_numpy(topk))
    layer.w.copy_(torch.from_numpy(w))
    if rows:
        W.fill_device(layer.x, seed, W.STREAM_X + layer_id)
    layer.route(fused=fused)
    if rows:
        layer.dispatch()
    assert layer.status() == 0
    pl, lo, mv = _check_route(layer, c, topk)
    if rows:
        _check_rows(layer, c, topk, w, lo, seed, layer_id, np.random.default_rng(seed * 31 + layer_id))
    assert layer.status() == 0
    return layer, c, pl, lo, mv


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "separate"])
@pytest.mark.parametrize("cfg", [2, 3, 5])
def test_full_size_layer(cfg, fused):
    layer, c, pl, lo, mv = _run_layer(cfg, seed=0, rows=fused, fused=fused)
    assert pl["n_rep"] > 0
    del layer


def test_full_size_fine_grained_eight_layers():
    for layer_id in range(8):
        layer, c, pl, lo, mv = _run_layer(4, seed=0, layer_id=layer_id, rows=layer_id in (0, 7),
                                          fused=layer_id % 2 == 0)
        del layer


def test_full_size_adversarial_companions():
    # perfectly uniform routing: max_vio exactly 0 and no replica
    layer, c, pl, lo, mv = _run_layer(5, seed=0, variant="uniform")
    assert mv == 0.0 and pl["n_rep"] == 0
    del layer
    # every token's top-1 on expert 0
    layer, c, pl, lo, mv = _run_layer(5, seed=0, variant="single_expert")
    assert pl["home_count"][0] + pl["rep_count"][pl["rep_expert"] == 0].sum() == c["T"]
    del layer


@pytest.mark.parametrize("cfg", [2, 3, 5])
def test_full_size_grad_reduce(cfg):
    import torch
    seed = 0
    layer, c, pl, lo, mv = _run_layer(cfg, seed, rows=False, grads=True)
    n, E = c["grad_n"], c["E"]
    W.fill_device(layer.g_home, seed, W.STREAM_GHOME)
    W.fill_device(layer.g_rep, seed, W.STREAM_GREP)
    layer.grad_reduce(clear=False)
    assert layer.status() == 0
    rng = np.random.default_rng(cfg)
    cols = np.unique(np.concatenate([rng.integers(0, n, 96), [0, 1, n - 1]]))
    got = layer.g_home.index_select(1, torch.from_numpy(cols).to(layer.g_home.device)).cpu().numpy()
    home0 = np.stack([W.grad_elements(seed, W.STREAM_GHOME, n, e, cols) for e in range(E)])
    reps = pl["rep_expert"]
    dt = c["grad_dtype"]
    rep0 = [W.grad_elements(seed, W.STREAM_GREP, n, m, cols, dt) for m in range(len(reps))]
    want = home0.copy()
    for m, e in enumerate(reps):  # home first, then replicas in match order
        r = rep0[m] if dt == "f32" else O.bf16_to_f32(rep0[m])
        want[e] = (want[e] + r).astype(np.float32)
    rel = np.abs(got - want) / np.maximum(np.abs(want), 1e-30)
    assert rel.max() <= 1e-6
    assert np.array_equal(got, want)
    del layer
