"""Host-side logic of the layer and the benchmark, on CPU: the host-fed
pipeline's token slices, the algorithmic byte counts behind every roofline
fraction, the clock sampler's parsing, and the rule that a committed DRAM
traffic figure is used only for the source it was captured on."""
import hashlib
import json
import os

import pytest


def test_slice_bounds_cover_the_tokens_in_order():
    from token_dispatch_histogram_b200.layer import slice_bounds
    for T in (0, 1, 7, 100, 32768, 32769):
        for chunks in (1, 2, 4, 5, 8, 11, 16):
            b = slice_bounds(T, chunks)
            assert len(b) == chunks + 1 and b[0] == 0 and b[-1] == T
            assert all(x <= y for x, y in zip(b, b[1:]))
    # from five slices on, the outer slices are the small ones (weights 1, 2, 4, ..., 4, 2, 1)
    b = slice_bounds(22 * 1000, 8)
    sizes = [y - x for x, y in zip(b, b[1:])]
    assert sizes == [1000, 2000, 4000, 4000, 4000, 4000, 2000, 1000]


def test_algorithmic_bytes_of_the_moderate_workload():
    """The byte counts written out from their definitions: each x row read
    once and each buffer row written once (dispatch), each buffer row read
    once plus the gate weights and positions and each output row written once
    (combine), home rows read and written and each replica row read once
    (gradient reduction, 8 replicated experts with 10 replicas)."""
    import bench
    import workload as W
    c = W.shape(2)
    T, P, H, n = 32768, 196608, 2048, 3 * 2048 * 1024
    assert (c["T"], c["P"], c["H"], c["grad_n"]) == (T, P, H, n)
    ab = bench.algorithmic_bytes(c, 10, 8)
    assert ab["dispatch"] == T * H * 2 + P * H * 2 + P * 4 == 940310528
    assert ab["combine"] == P * H * 2 + P * 4 + P * 4 + T * H * 2 == 941096960
    assert ab["grad_reduce"] == 8 * n * 4 * 2 + 10 * n * 4 == 654311424
    # the committed ncu traffic records use the same per-launch figures
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    rec = json.load(open(os.path.join(root, "profiles", "traffic.json")))
    assert rec["k_dispatch"]["algorithmic_bytes_per_launch"] == ab["dispatch"]
    assert rec["k_combine"]["algorithmic_bytes_per_launch"] == ab["combine"]
    assert rec["k_grad_reduce"]["algorithmic_bytes_per_launch"] == ab["grad_reduce"]


def test_clock_sampler_parses_reasons_and_median():
    import bench
    cs = bench.ClockSampler(0)
    cs.proc = type("P", (), {"terminate": lambda self: None, "wait": lambda self, timeout=None: 0})()
    cs.lines = ["1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
                "1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
                "1900, 1965, 950.0, 0x0, Not Active, Not Active, Not Active, Not Active",
                "garbage"]
    out = cs.stop()
    assert out["sm_mhz"] == 1900 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] == 3


def test_traffic_record_only_for_the_captured_source(tmp_path, monkeypatch):
    import bench
    src = tmp_path / "k.cu"
    src.write_text("kernel source\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    rec = {"k_x": {"dram_bytes_per_launch": 123, "source": "k.cu", "source_sha": sha}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record("k_x")["dram_bytes_per_launch"] == 123
    assert bench.traffic_record("k_y") is None
    src.write_text("kernel source, changed\n")
    assert bench.traffic_record("k_x") is None
