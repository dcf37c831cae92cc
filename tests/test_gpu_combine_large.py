"""Combine and the backward of dispatch on problems of 2^28 row elements and
more, where ep_combine runs its shared-memory ring kernel (-m gpu): every
output element against the oracle, bit for bit (so within the 1-bf16-ulp bar),
for wide and narrow rows (one token per warp and several tokens per warp),
K = 1 ... 8, with and without gate weights, and a row index outside the
buffer that is reported and contributes nothing."""
import functools

import numpy as np
import pytest

import oracle as O
import workload as W

pytestmark = pytest.mark.gpu

CASES = [
    # T tokens, K, H   (T * H >= 2^28)
    (1 << 15, 3, 8192),    # one token per warp, 32 lanes per row
    (1 << 18, 8, 1024),
    (1 << 22, 1, 64),      # 8 lanes per token, four tokens per warp
    (1 << 19, 6, 520),     # 65 vectors per row: a ragged last job
]


@functools.lru_cache(maxsize=2)
def _inputs(T, K, H, seed):
    rng = np.random.default_rng(seed)
    rows = T * K
    pos = rng.permutation(rows).astype(np.int32)
    w = rng.random((T, K), dtype=np.float32)
    y = W.normal_bf16(seed, 0x700, 0, rows * H).reshape(rows, H)
    return pos, w, y


@pytest.mark.parametrize("weights", [True, False], ids=["combine", "dispatch_backward"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "T{}_K{}_H{}".format(*c))
def test_large_combine_matches_oracle(case, weights):
    import torch
    import token_dispatch_histogram_b200 as tdh
    T, K, H = case
    assert T * H >= 1 << 28
    pos, w, y = _inputs(T, K, H, seed=T + K + H)
    dev = torch.device("cuda")
    y_d = torch.from_numpy(y.view(np.int16)).to(dev).view(torch.bfloat16)
    pos_d = torch.from_numpy(pos).to(dev)
    out = torch.full((T, H), -1.0, dtype=torch.bfloat16, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    if weights:
        tdh.ep_combine(y_d, torch.from_numpy(w).to(dev), pos_d, out, st)
        want = O.combine(y, w, pos, K)
    else:
        tdh.ep_dispatch_backward(y_d, pos_d, T, K, out, st)
        want = O.dispatch_backward(y, pos, T, K)
    assert tdh.ep_status_read(st) == 0
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(got, want)


def test_large_combine_bad_row_is_reported():
    import torch
    import token_dispatch_histogram_b200 as tdh
    T, K, H = 1 << 15, 2, 8192
    pos, w, y = _inputs(T, K, H, seed=7)
    pos = pos.copy()
    pos[5] = T * K + 3  # past the buffer: skipped, flagged
    dev = torch.device("cuda")
    out = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    tdh.ep_combine(torch.from_numpy(y.view(np.int16)).to(dev).view(torch.bfloat16), torch.from_numpy(w).to(dev),
                   torch.from_numpy(pos).to(dev), out, st)
    assert tdh.ep_status_read(st) == tdh.EP_DEV_BAD_ROW
    pos_ok = pos.copy()
    pos_ok[5] = -1  # the oracle's "contributes nothing"
    want = O.combine(y, w, pos_ok, K)
    np.testing.assert_array_equal(out.view(torch.int16).cpu().numpy().view(np.uint16), want)
