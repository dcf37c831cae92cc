"""Fused layout + dispatch (ep_route_dispatch_fused) against the CPU oracle
and against the separate route + dispatch calls, through the C ABI (-m gpu).

Bar: every route output and every buffer row bit-exact.  Cases span one and
two CTAs per SM, tiles whose token rows straddle the tile boundary (K does not
divide the tile), rows from 16 bytes to 32 KB, K = 1 .. 8, degenerate routing,
and invalid expert ids (reported, their rows never written).
"""
import numpy as np
import pytest

import oracle as O
import workload as W
from gpu_path import assert_route_parity, case_inputs, run_cuda, run_oracle

pytestmark = pytest.mark.gpu

CASES = [
    # (R, S, K, E, H, kind, block_m)
    (4, 64, 2, 16, 128, "zipf", 4),          # the tiny workload
    (8, 4096, 6, 64, 2048, "skew", 64),      # the moderate EP8 workload's shape, one CTA per SM
    (16, 2048, 8, 256, 1024, "skew", 128),   # 262,144 pairs: two CTAs per SM
    (3, 777, 5, 9, 24, "skew", 3),           # odd sizes: token rows straddle tiles
    (2, 900, 1, 4, 8, "single", 1),          # K = 1, 16-byte rows
    (4, 1024, 8, 32, 7168, "uniform", 128),  # DeepSeek-V3 row width, no replica
    (2, 300, 4, 8, 16384, "skew", 16),       # 32 KB rows
    (1, 1000, 3, 7, 64, "skew", 16),         # one rank
    (64, 301, 8, 384, 256, "skew", 128),     # fine-grained expert count, ragged
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "R{}_S{}_K{}_E{}_H{}_{}".format(*c[:6]))
def test_route_dispatch_fused(case):
    R, S, K, E, H, kind, bm = case
    if kind == "zipf":
        topk, w = W.routing_from(R * S, E, K, seed=0, bias_e=W.bias(1, 0))
        x = W.hidden(R * S, H, seed=5)
    else:
        topk, w, x = case_inputs(R, S, K, E, H, seed=R * 17 + H, kind=kind, bias_scale=1.5)
    cu = run_cuda(topk, w, x, R, S, E, bm, with_y=False, fused="dispatch")
    orc = run_oracle(topk, None, None, R, S, E, bm)
    assert_route_parity(cu, orc, R, S, K, E)
    np.testing.assert_array_equal(cu["buf"], O.dispatch(x, orc["layout"]["pos"], K, R * S * K))
    sep = run_cuda(topk, w, x, R, S, E, bm, with_y=False, fused=True)
    np.testing.assert_array_equal(cu["buf"], sep["buf"])
    np.testing.assert_array_equal(cu["out"], sep["out"])


def test_route_dispatch_fused_fuzz():
    rng = np.random.default_rng(77)
    for it in range(24):
        R = int(rng.choice([1, 2, 3, 4, 8, 16]))
        E = R * int(rng.integers(1, 9))
        K = int(rng.integers(1, min(8, E) + 1))
        S = int(rng.integers(1, 2500 // R + 2))
        H = int(rng.choice([8, 16, 64, 200, 1024, 2048]))
        kind = ["skew", "uniform", "single"][it % 3]
        topk, w, x = case_inputs(R, S, K, E, H, seed=1000 + it, kind=kind, bias_scale=float(rng.uniform(0.2, 3)))
        bm = int(rng.choice([1, 16, 128]))
        cu = run_cuda(topk, w, x, R, S, E, bm, with_y=False, fused="dispatch")
        orc = run_oracle(topk, None, None, R, S, E, bm)
        assert_route_parity(cu, orc, R, S, K, E)
        np.testing.assert_array_equal(cu["buf"], O.dispatch(x, orc["layout"]["pos"], K, R * S * K), err_msg=str(it))


def test_route_dispatch_fused_invalid_ids():
    """An id outside [0, E) is reported, and the loads no longer add up to
    R*S*K, so the plan is empty and no pair gets a row: the same status bits,
    pos and (untouched) buffer as the fused route followed by ep_dispatch."""
    import torch
    import token_dispatch_histogram_b200 as tdh
    R, S, K, E, H = 4, 600, 4, 16, 64
    topk, w, x = case_inputs(R, S, K, E, H, seed=3)
    topk = topk.copy()
    topk[5, 1] = E + 3
    topk[1000, 0] = -1
    dev = torch.device("cuda")
    outs = {}
    for form in ("fused", "separate"):
        lay = tdh.EpLayer(R, S, K, E, H, 16, device=dev)
        lay.topk_ids.copy_(torch.from_numpy(topk))
        lay.x.copy_(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16))
        lay.buf.view(torch.int16).fill_(-1)
        if form == "fused":
            lay.route_dispatch()
        else:
            lay.route()
            lay.dispatch()
        outs[form] = (lay.status(), lay.pos.cpu().numpy(), lay.buf.view(torch.int16).cpu().numpy())
    st, pos, buf = outs["fused"]
    assert st & tdh.EP_DEV_BAD_EXPERT_ID and st & tdh.EP_DEV_BAD_ROW
    assert st == outs["separate"][0]
    assert st & tdh.EP_DEV_BAD_LOADS
    assert np.all(pos == -1)
    np.testing.assert_array_equal(pos, outs["separate"][1])
    np.testing.assert_array_equal(buf, outs["separate"][2])
    assert np.all(buf == -1)


def test_route_dispatch_fused_empty():
    import torch
    import token_dispatch_histogram_b200 as tdh
    lay = tdh.EpLayer(4, 0, 2, 16, 64, 4, device=torch.device("cuda"))
    lay.route_dispatch()
    assert lay.status() == 0
