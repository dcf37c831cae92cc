"""Parity at the full workload sizes (-m gpu), in the launch configuration the
benchmark uses (the same binding and EpLayer buffers), every output compared
in full:

  * loads, max_vio, plan, layout (pos, src, pair_slot), cu_seqlens, align-sort:
    bit-exact against the CPU oracle;
  * dispatch: every row of the dispatch buffer, bitwise.  The tokens are taken
    in chunks; a chunk's rows are gathered from the device buffer in row order
    and compared with the oracle's dispatch of that chunk (its hidden rows
    regenerated on the host from the counter-based generator, its pairs placed
    at their rank among the chunk's rows), so the whole buffer is covered
    without a host copy of it;
  * combine (after the stand-in expert): every output token against the
    oracle's layout-free closed form, within 1 bf16 ulp (and checked
    identical);
  * replica gradient reduction: every element of every replicated expert's
    home row against the oracle's reduction (fp32 adds in match order), within
    1e-6 relative (and checked identical); every other home row unchanged.

The host checks of a chunk run on a thread pool (the oracle and the generator
are C calls that release the interpreter lock; each oracle call is still one
single-threaded pass over its chunk).

Workloads: moderate EP8 (R=8, S=4096, E=64, K=6, H=2048), DeepSeek-V3-shaped
(R=32, S=4096, E=256, K=8, H=7168, bf16 replica grads), fine-grained 8-layer
(R=64, S=8192, E=384, K=8, H=7168, bias redrawn per layer; rows of layers 0
and 7), adversarial prefill (R=16, S=16384, E=256, K=8, H=4096) with its
uniform and single-expert companions.
"""
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest

import oracle as O
import workload as W
from gpu_path import bf16_ulp_diff

pytestmark = pytest.mark.gpu

WORKERS = max(2, min(32, os.cpu_count() or 2))
CHUNK_ELEMS = 1 << 26  # row elements per checked chunk (128 MB of bf16 rows)


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


def _token_chunks(c):
    ch = max(1, min(c["T"], CHUNK_ELEMS // (c["K"] * c["H"])))
    return [(t0, min(c["T"], t0 + ch)) for t0 in range(0, c["T"], ch)]


def _drain(futs, keep):
    """Wait until at most `keep` checks are in flight; raise the first failure."""
    while len(futs) > keep:
        futs.pop(0).result()


def _dispatch_chunk_ok(got, local, t0, t1, seed, layer_id, K, H):
    x = W.hidden(t1 - t0, H, seed, layer_id, t0, threads=1)
    want = O.dispatch(x, local, K, local.size)
    assert np.array_equal(got, want), f"dispatch rows of tokens [{t0}, {t1}) differ"


def _combine_chunk_ok(got, t0, t1, seed, layer_id, H, w, topk, scale):
    x = W.hidden(t1 - t0, H, seed, layer_id, t0, threads=1)
    want = O.combine_closed(x, w[t0:t1], topk[t0:t1], scale)
    ulp = bf16_ulp_diff(got, want)
    assert ulp.max() <= 1, f"combine of tokens [{t0}, {t1}): {ulp.max()} ulp"
    assert np.count_nonzero(ulp) == 0, f"combine of tokens [{t0}, {t1}) not identical"


def _check_rows(layer, c, topk, w, lo, seed, layer_id):
    import torch
    K, H, T, P = c["K"], c["H"], c["T"], c["P"]
    dev = layer.buf.device
    pos = lo["pos"].astype(np.int64)
    covered = np.zeros(P, dtype=bool)
    with ThreadPoolExecutor(WORKERS) as ex:
        futs = []
        for t0, t1 in _token_chunks(c):
            pc = pos[t0 * K:t1 * K]
            order = np.argsort(pc, kind="stable")
            rows = pc[order]
            local = np.empty(pc.size, dtype=np.int32)
            local[order] = np.arange(pc.size, dtype=np.int32)  # the pair's rank among the chunk's rows
            covered[rows] = True
            got = layer.buf.index_select(0, torch.from_numpy(rows).to(dev)).view(torch.int16).cpu().numpy()
            futs.append(ex.submit(_dispatch_chunk_ok, got.view(np.uint16), local, t0, t1, seed, layer_id, K, H))
            _drain(futs, 2 * WORKERS)
        _drain(futs, 0)
    assert covered.all(), "some buffer rows belong to no pair"
    # stand-in expert, then combine; every token against the closed form
    scale = W.expert_scale(c["E"])
    layer.expert_standin(torch.from_numpy(scale).to(dev))
    layer.combine()
    with ThreadPoolExecutor(WORKERS) as ex:
        futs = []
        for t0, t1 in _token_chunks(c):
            got = layer.out[t0:t1].view(torch.int16).cpu().numpy().view(np.uint16)
            futs.append(ex.submit(_combine_chunk_ok, got, t0, t1, seed, layer_id, H, w, topk, scale))
            _drain(futs, 2 * WORKERS)
        _drain(futs, 0)


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
        _check_rows(layer, c, topk, w, lo, seed, layer_id)
    assert layer.status() == 0
    return layer, c, pl, lo, mv


def test_device_generator_matches_host():
    """The full-size checks regenerate the device-filled inputs on the host:
    both generators give the same bits (fp32 and bf16, at offsets that are not
    multiples of the generator's four-value block)."""
    import torch
    t32 = torch.empty(100003, dtype=torch.float32, device="cuda")
    t16 = torch.empty(100003, dtype=torch.bfloat16, device="cuda")
    for off in (0, 1, 7, 123457):
        W.fill_device(t32, 5, W.STREAM_GHOME, off)
        W.fill_device(t16, 5, W.STREAM_X + 3, off)
        assert np.array_equal(t32.cpu().numpy(), W.normal_f32(5, W.STREAM_GHOME, off, t32.numel()))
        assert np.array_equal(t16.view(torch.int16).cpu().numpy().view(np.uint16),
                              W.normal_bf16(5, W.STREAM_X + 3, off, t16.numel()))


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


def _grad_row_ok(got, e, ms, seed, n, dt):
    home = W.normal_f32(seed, W.STREAM_GHOME, e * n, n, threads=1)[None]
    gen = W.normal_f32 if dt == "f32" else W.normal_bf16
    reps = np.stack([gen(seed, W.STREAM_GREP, int(m) * n, n, threads=1) for m in ms])
    want, _ = O.grad_reduce(home, reps, np.zeros(len(ms), dtype=np.int32))  # home first, then match order
    want = want[0]
    rel = np.abs(got - want) / np.maximum(np.abs(want), 1e-30)
    assert rel.max() <= 1e-6, f"expert {e}: relative error {rel.max()}"
    assert np.array_equal(got, want), f"expert {e}: not identical"


@pytest.mark.parametrize("cfg", [2, 3, 5])
def test_full_size_grad_reduce(cfg):
    import torch
    seed = 0
    layer, c, pl, lo, mv = _run_layer(cfg, seed, rows=False, grads=True)
    n, E, dt = c["grad_n"], c["E"], c["grad_dtype"]
    W.fill_device(layer.g_home, seed, W.STREAM_GHOME)
    W.fill_device(layer.g_rep, seed, W.STREAM_GREP)
    layer.grad_reduce(clear=False)
    assert layer.status() == 0
    reps = pl["rep_expert"]
    replicated = sorted(set(reps.tolist()))
    assert replicated
    with ThreadPoolExecutor(WORKERS) as ex:
        futs = []
        for e in replicated:
            got = layer.g_home[e].cpu().numpy()
            futs.append(ex.submit(_grad_row_ok, got, e, np.nonzero(reps == e)[0], seed, n, dt))
            _drain(futs, WORKERS)
        _drain(futs, 0)
    # every other home row is its input, unchanged (regenerated on the device)
    fresh = torch.empty(n, dtype=torch.float32, device=layer.g_home.device)
    for e in sorted(set(range(E)) - set(replicated)):
        W.fill_device(fresh, seed, W.STREAM_GHOME, e * n)
        assert torch.equal(fresh, layer.g_home[e]), f"expert {e} has no replica but its row changed"
    del layer
