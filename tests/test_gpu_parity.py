"""CUDA path vs CPU oracle, element by element, through the C ABI (-m gpu).

Bars: loads, max_vio, plan, layout, align-sort and dispatch bit-exact;
combine within 1 bf16 ulp per element (the kernel's arithmetic is the
oracle's, one fp32 multiply and one fp32 add per term in k order, so it is
also checked to be bit-exact); grad-reduce within 1e-6 relative (the same
adds in the same order, also checked bit-exact).

Sizes span several histogram tiles (2048-8192 pairs each) with ragged tails,
plus the degenerate cases: one rank, uniform routing (no replica), every
token's top-1 on one expert, an expert with no pair, T = 0.
"""
import numpy as np
import pytest

import oracle as O
import oracle_pins as PINS
import workload as W
from gpu_path import assert_route_parity, bf16_ulp_diff, case_inputs, plan_field, run_cuda, run_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
def test_hand_example_on_gpu(fused):
    g = PINS.golden()
    topk = np.array(g["topk_ids"], dtype=np.int32)
    R, S, K, E = g["R"], g["S"], g["K"], g["E"]
    cu = run_cuda(topk, None, None, R, S, E, g["block_m"], fused=fused)
    assert cu["status"] == 0
    assert cu["loads"].tolist() == g["loads"]
    assert cu["max_vio"] == g["max_vio"]
    assert cu["pos"].tolist() == g["pos"]
    assert plan_field(cu, "cu_seqlens", 12).tolist() == g["cu_seqlens"]
    assert plan_field(cu, "slot_order", 11).tolist() == g["slot_order"]
    assert cu["ntpp"] == g["align_num_tokens_post_pad"]
    assert cu["expert_ids"].tolist() == g["align_expert_ids"]


ROUTE_CASES = [
    # (R, S, K, E, kind, block_m)
    (4, 64, 2, 16, "zipf", 4),            # the tiny workload's shape
    (8, 4096, 6, 64, "skew", 64),         # the moderate EP8 workload's shape (96 tiles)
    (1, 1000, 3, 7, "skew", 16),          # one rank: no replica possible
    (4, 1024, 8, 32, "uniform", 128),     # uniform: max_vio 0, no replica
    (16, 613, 8, 256, "single", 128),     # every top-1 on expert 0; ragged tail
    (3, 777, 5, 9, "skew", 3),            # odd sizes, E/R = 3
    (2, 1, 1, 2, "skew", 1),
    (64, 301, 8, 384, "skew", 128),       # fine-grained, ragged
    (8, 2047, 4, 1024, "skew", 8),        # E at the library limit
    (1024, 4, 2, 1024, "skew", 4),        # R at the library limit, E/R = 1
    (4, 0, 2, 16, "skew", 4),             # T = 0
]


@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
@pytest.mark.parametrize("case", ROUTE_CASES, ids=lambda c: "R{}_S{}_K{}_E{}_{}".format(*c[:5]))
def test_route_plan_layout_align(case, fused):
    R, S, K, E, kind, bm = case
    if kind == "zipf":
        topk, w = W.routing_from(R * S, E, K, seed=0, bias_e=W.bias(1, 0))
    else:
        topk, w, _ = case_inputs(R, S, K, E, 0, seed=R * 131 + S, kind=kind, bias_scale=1.5)
    cu = run_cuda(topk, None, None, R, S, E, bm, fused=fused)
    orc = run_oracle(topk, None, None, R, S, E, bm)
    assert_route_parity(cu, orc, R, S, K, E)


@pytest.mark.parametrize("fused", [False, True], ids=["separate", "fused"])
def test_route_fuzz(fused):
    rng = np.random.default_rng(2024)
    for it in range(60):
        R = int(rng.choice([1, 2, 3, 4, 8, 16]))
        ER = int(rng.integers(1, 9))
        E = R * ER
        K = int(rng.integers(1, min(8, E) + 1))
        S = int(rng.integers(0, 3000 // max(1, R)))
        kind = ["skew", "uniform", "single"][it % 3]
        bm = int(rng.choice([1, 2, 16, 64, 128]))
        topk, w, _ = case_inputs(R, S, K, E, 0, seed=it, kind=kind, bias_scale=float(rng.uniform(0.2, 3)))
        cu = run_cuda(topk, None, None, R, S, E, bm, fused=fused)
        orc = run_oracle(topk, None, None, R, S, E, bm)
        assert_route_parity(cu, orc, R, S, K, E)


ROW_CASES = [
    # (R, S, K, E, H, kind)
    (4, 64, 2, 16, 128, "zipf"),       # tiny workload
    (8, 256, 6, 64, 2048, "skew"),     # moderate workload's row width, fewer tokens
    (4, 300, 8, 32, 7168, "skew"),     # DeepSeek-V3 row width, ragged
    (2, 50, 1, 4, 64, "skew"),         # K = 1
    (3, 33, 5, 9, 24, "single"),       # generic-K combine path, narrow rows
    (16, 64, 8, 256, 4096, "uniform"),
    (2, 40, 12, 16, 64, "skew"),       # K > 8: the generic combine kernel
    (8, 512, 8, 64, 7168, "single"),   # K = 8, wide rows, a dominant expert
    (2, 64, 4, 8, 16384, "skew"),      # 32 KB rows
    (4, 100, 3, 8, 8, "skew"),         # the narrowest row, one 16-byte vector
]


@pytest.mark.parametrize("case", ROW_CASES, ids=lambda c: "R{}_S{}_K{}_E{}_H{}_{}".format(*c))
def test_dispatch_expert_combine(case):
    R, S, K, E, H, kind = case
    if kind == "zipf":
        topk, w = W.routing_from(R * S, E, K, seed=0, bias_e=W.bias(1, 0))
        x = W.hidden(R * S, H, seed=5)
    else:
        topk, w, x = case_inputs(R, S, K, E, H, seed=H + S, kind=kind)
    scale = W.expert_scale(E)
    cu = run_cuda(topk, w, x, R, S, E, 4, scale=scale)
    orc = run_oracle(topk, w, x, R, S, E, 4, scale=scale)
    assert cu["status"] == 0
    np.testing.assert_array_equal(cu["pos"], orc["layout"]["pos"])
    np.testing.assert_array_equal(cu["buf"], orc["buf"])          # dispatch: bitwise
    np.testing.assert_array_equal(cu["y"], orc["y"])              # stand-in expert: bitwise
    ulp = bf16_ulp_diff(cu["out"], orc["out"])
    assert ulp.max() <= 1                                         # combine bar: 1 bf16 ulp
    assert np.count_nonzero(ulp) == 0                             # and in fact identical
    # combine against the layout-free closed form too
    cf = __import__("oracle").combine_closed(x, w, topk, scale)
    assert bf16_ulp_diff(cu["out"], cf).max() <= 1


def test_bf16_rounding_edges():
    """The row kernels round fp32 to bf16 with the hardware pair conversion.
    Through the stand-in expert (one fp32 multiply, one rounding) and combine
    (K = 1, unit weight), crafted values hit every class: exact ties to even,
    overflow to Inf, subnormal results, signed zeros, Inf in; each must equal
    the oracle's rounding bit for bit, and NaN in must give NaN out."""
    import torch
    import token_dispatch_histogram_b200 as tdh
    rng = np.random.default_rng(11)
    specials = np.array([0x7F7F, 0xFF7F, 0x0001, 0x8001, 0x0080, 0x007F, 0x0000, 0x8000, 0x7F80, 0xFF80,
                         0x3F81, 0x3FC1, 0x4001, 0xBF81, 0x3C01, 0x0100], dtype=np.uint16)
    H, E = 64, 4
    rows = 64
    x = rng.integers(0, 0x10000, size=(rows, H), dtype=np.uint16)
    x[(x & 0x7F80) == 0x7F80] = 0x3F80  # no NaN/Inf at random
    x[:, :len(specials)] = specials
    scale = np.array([1.5, 2.0 ** -10, 1.0 + 2.0 ** -8, 1.0 + 2.0 ** -23], dtype=np.float32)
    topk = (np.arange(rows) % E).astype(np.int32).reshape(rows, 1)
    src = np.arange(rows, dtype=np.int32)
    want = O.expert_standin(x, src, topk, scale)
    dev = "cuda"
    t_x = torch.from_numpy(x.view(np.int16)).to(dev).view(torch.bfloat16)
    y = torch.empty_like(t_x)
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    tdh.ep_expert_scale(t_x, torch.from_numpy(src).to(dev), torch.from_numpy(topk).to(dev),
                        torch.from_numpy(scale).to(dev), y, st)
    got = y.view(torch.int16).cpu().numpy().view(np.uint16)
    assert tdh.ep_status_read(st) == 0
    np.testing.assert_array_equal(got, want)
    assert np.any(got == 0x7F80) and np.any(got == 0xFF80)   # overflow to +-Inf happened
    assert np.any((got & 0x7F80) == 0) and np.any((got & 0x7FFF) != 0)  # subnormal results happened
    # combine of one unit-weight row per token: the row, except that -0 comes
    # out +0 (the accumulator starts at +0 and +0 + -0 = +0), as in the oracle
    out = torch.empty_like(y)
    w1 = torch.ones((rows, 1), dtype=torch.float32, device=dev)
    tdh.ep_combine(y, w1, torch.from_numpy(src).to(dev), out, st)
    got_c = out.view(torch.int16).cpu().numpy().view(np.uint16)
    np.testing.assert_array_equal(got_c, O.combine(got, np.ones((rows, 1), np.float32), src, 1))
    np.testing.assert_array_equal(got_c, np.where(got == 0x8000, 0, got))
    # NaN in, NaN out (the hardware writes the canonical NaN; the oracle keeps the payload)
    xn = x.copy()
    xn[:, 0] = 0x7FC1
    t_xn = torch.from_numpy(xn.view(np.int16)).to(dev).view(torch.bfloat16)
    tdh.ep_expert_scale(t_xn, torch.from_numpy(src).to(dev), torch.from_numpy(topk).to(dev),
                        torch.from_numpy(scale).to(dev), y, st)
    assert torch.isnan(y[:, 0].float()).all()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("clear", [False, True])
def test_grad_reduce(dtype, clear):
    R, S, K, E = 8, 512, 6, 64
    topk, w, _ = case_inputs(R, S, K, E, 0, seed=77, bias_scale=1.5)
    for n in (1000, 4096, 3 * 128 * 64 + 8):  # n % 8 != 0 takes the scalar path
        cap = E + R - 1
        g_home = W.grad_rows(3, W.STREAM_GHOME, n, E)
        g_rep = W.grad_rows(4, W.STREAM_GREP, n, cap, dtype)
        cu = run_cuda(topk, None, None, R, S, E, 4, g_home=g_home, g_rep=g_rep, clear=clear)
        orc = run_oracle(topk, None, None, R, S, E, 4, g_home=g_home, g_rep=g_rep, clear=clear)
        assert orc["plan"]["n_rep"] > 0
        rel = np.abs(cu["g_home"] - orc["g_home"]) / np.maximum(np.abs(orc["g_home"]), 1e-30)
        assert rel.max() <= 1e-6
        np.testing.assert_array_equal(cu["g_home"], orc["g_home"])  # same adds, same order
        np.testing.assert_array_equal(cu["g_rep"], orc["g_rep"])    # cleared rows (if asked), others untouched


@pytest.mark.parametrize("B", [0, 1, 3, 8])
def test_prefetch_slots(B):
    """Slot per replica, remote count and capped loads, bit-exact, on the hand
    example and the routings of three workloads."""
    import torch
    import token_dispatch_histogram_b200 as tdh
    import oracle as O
    g = PINS.golden()
    cases = [(g["R"], g["S"], g["K"], g["E"], 4, np.array(g["topk_ids"], dtype=np.int32))]
    for cfg in (1, 2, 5):
        c = W.shape(cfg)
        cases.append((c["R"], c["S"], c["K"], c["E"], c["block_m"], W.routing(cfg, 0)[0]))
    for R, S, K, E, block_m, topk in cases:
        layer = tdh.EpLayer(R, S, K, E, 8, block_m, device="cuda")
        layer.topk_ids.copy_(torch.from_numpy(topk))
        layer.route()
        cap = layer.plan_layout["cap"]
        slot = torch.full((cap,), -7, dtype=torch.int32, device="cuda")
        nrem = torch.full((R,), -7, dtype=torch.int32, device="cuda")
        capped = torch.full((R,), -7, dtype=torch.int64, device="cuda")
        tdh.ep_prefetch_slots(layer.plan, E, R, S * K, B, slot, nrem, capped)
        loads, _, _ = O.route_stats(topk, E)
        pl = O.plan(loads, R, S, K, E)
        ref, ref_rem, ref_capped = O.prefetch_slots(pl, E, R, B, S * K)
        got = slot.cpu().numpy()
        np.testing.assert_array_equal(got[:pl["n_rep"]], ref)
        assert np.all(got[pl["n_rep"]:] == -1)
        np.testing.assert_array_equal(nrem.cpu().numpy(), ref_rem)
        np.testing.assert_array_equal(capped.cpu().numpy(), ref_capped)
        tdh.ep_prefetch_slots(layer.plan, E, R, S * K, B, slot, nrem)  # load_capped is optional
        np.testing.assert_array_equal(slot.cpu().numpy()[:pl["n_rep"]], ref)
