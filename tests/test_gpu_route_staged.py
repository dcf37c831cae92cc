"""The one-launch route on problems whose tiles are large enough to be staged
in shared memory (-m gpu).

From 12,288 pairs per tile on, each tile CTA of ep_route_fused keeps its pairs
in shared memory in (expert, rank) order and writes the align-sort ids and the
src rows as runs, a warp per expert and all warps together on runs longer than
a warp's share.  These cases (3.9-4.2M pairs: tiles of 13.8-14.3K pairs on 148
SMs, two CTAs per SM) compare every route output with the oracle: skewed
routing, every top-1 on one expert (one run per tile far longer than a warp's
share), a ragged tail with block_m = 1, and ids outside [0, E).
"""
import numpy as np
import pytest

import oracle as O
from gpu_path import assert_route_parity, case_inputs, run_cuda, run_oracle

pytestmark = pytest.mark.gpu

CASES = [  # R, S, K, E, kind, bias_scale, block_m
    (8, 81920, 6, 64, "skew", 1.0, 16),
    (8, 81920, 6, 64, "single", 1.0, 16),
    (16, 32768, 8, 256, "skew", 2.5, 64),
    (4, 196613, 5, 40, "skew", 1.0, 1),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "R{}_S{}_K{}_E{}_{}_b{}_bm{}".format(*c))
def test_staged_route_matches_oracle(case):
    R, S, K, E, kind, bias, bm = case
    topk, w, _ = case_inputs(R, S, K, E, 0, seed=S + E, kind=kind, bias_scale=bias)
    cu = run_cuda(topk, w, None, R, S, E, bm, fused=True)
    orc = run_oracle(topk, w, None, R, S, E, bm)
    assert_route_parity(cu, orc, R, S, K, E)


def test_staged_route_invalid_ids():
    """Ids outside [0, E) in a staged tile: reported, their pairs get no row
    (pos = -1), the loads no longer add up so the plan is empty, and the
    align-sort still places every valid pair; the same outputs as the four
    separate entry points."""
    import token_dispatch_histogram_b200 as tdh
    R, S, K, E, bm = 8, 81920, 6, 64, 16
    topk, w, _ = case_inputs(R, S, K, E, 0, seed=11)
    topk = topk.copy()
    topk[17, 2] = E
    topk[300000, 0] = -3
    topk[-1, K - 1] = E + 100
    fused = run_cuda(topk, w, None, R, S, E, bm, fused=True)
    sep = run_cuda(topk, w, None, R, S, E, bm, fused=False)
    st = fused["status"]
    assert st & tdh.EP_DEV_BAD_EXPERT_ID and st & tdh.EP_DEV_BAD_LOADS
    assert st == sep["status"]
    loads, _, bad = O.route_stats(topk, E)
    assert bad == 3
    np.testing.assert_array_equal(fused["loads"], loads)
    assert np.all(fused["pos"] == -1)
    ids, eids, n = O.align_sort(topk, E, bm)
    np.testing.assert_array_equal(fused["sorted_ids"], ids)
    np.testing.assert_array_equal(fused["expert_ids"], eids)
    assert fused["ntpp"] == n
    from gpu_path import plan_field
    assert plan_field(fused, "n_rep", 1)[0] == 0
    for name in ("pos", "src", "pair_slot", "sorted_ids", "expert_ids"):
        np.testing.assert_array_equal(fused[name], sep[name], err_msg=name)
