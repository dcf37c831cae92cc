"""Host-side logic of the layer and the benchmark, on CPU: the host-fed
pipeline's token slices and the waits between host-fed batches, the algorithmic byte counts behind every roofline
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


def test_batch_gating_follows_the_buffers():
    """The waits between host-fed batches, from which storage each buffer is
    (A, B: the chain's two row buffers; C, D: stage buffers of their own)."""
    from token_dispatch_histogram_b200.layer import batch_gating
    A, B, C, D = 1, 2, 3, 4
    # one layer with stage buffers apart, or its own x and out: slice by slice both ways
    for xs, os_ in ((C, D), (A, B)):
        g = batch_gating([(A, B)], xs, os_)
        assert g == {"x_last_use": 0, "out_first_write": 0, "x_waits_sent": False, "x_by_slice": True,
                     "out_by_slice": True}
    # one layer whose stage buffers are one storage: everything waits for the rows to have left
    g = batch_gating([(A, B)], C, C)
    assert g["x_waits_sent"] and not g["x_by_slice"] and not g["out_by_slice"]
    # a chain of two on its own buffers: x_stage = layer 0's x = A = layer 1's out = out_stage
    g = batch_gating([(A, B), (B, A)], A, A)
    assert g["x_waits_sent"] and g["x_last_use"] == 1 and g["out_first_write"] == 1
    assert not g["x_by_slice"] and not g["out_by_slice"]
    # a chain of three on its own buffers: A is used up to the last layer, B is written from layer 0 on
    g = batch_gating([(A, B), (B, A), (A, B)], A, B)
    assert not g["x_waits_sent"] and g["x_last_use"] == 2 and g["out_first_write"] == 0
    assert not g["x_by_slice"] and not g["out_by_slice"]
    # eight chained layers with stage buffers apart: rows in after the first layer, out slice by slice
    chain = [(A, B) if l % 2 == 0 else (B, A) for l in range(8)]
    g = batch_gating(chain, C, D)
    assert g == {"x_last_use": 0, "out_first_write": 7, "x_waits_sent": False, "x_by_slice": False,
                 "out_by_slice": True}
    # a stage buffer that is one of the chain's: waits for the last layer using it
    g = batch_gating(chain, B, D)
    assert g["x_last_use"] == 7 and not g["x_by_slice"]
    with pytest.raises(ValueError):
        batch_gating([], C, D)


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
    assert rec["k_dispatch@moderate_ep8"]["algorithmic_bytes_per_launch"] == ab["dispatch"]
    assert rec["k_combine@moderate_ep8"]["algorithmic_bytes_per_launch"] == ab["combine"]
    assert rec["k_grad_reduce@moderate_ep8"]["algorithmic_bytes_per_launch"] == ab["grad_reduce"]
    for k, r in rec.items():  # every record names the pairs of the launch it was captured on
        assert k.split("@")[1] == r["workload"] and r["pairs_per_launch"] > 0


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
    """A record is used only at the source it was captured on, and only for
    its own workload shape, scaled by pairs per launch."""
    import bench
    src = tmp_path / "k.cu"
    src.write_text("kernel source\n")
    sha = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    rec = {"k_x@fine": {"dram_bytes_per_launch": 1000, "source": "k.cu", "source_sha": sha, "capture": "cap",
                        "pairs_per_launch": 100, "workload": "fine"}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    got = bench.traffic_record("k_x", {"name": "fine", "P": 1600})
    assert got["dram_bytes_per_launch"] == 16000 and got["scaled_by"] == 16.0
    assert bench.traffic_record("k_x", {"name": "other", "P": 1600}) is None
    assert bench.traffic_record("k_y", {"name": "fine", "P": 1600}) is None
    src.write_text("kernel source, changed\n")
    assert bench.traffic_record("k_x", {"name": "fine", "P": 1600}) is None


def test_both_arms_print_the_same_config():
    """The reference arm and ours describe the workload with one function of
    the workload alone (nothing about the timing method in it)."""
    import bench
    for cfg in (1, 2, 3, 4, 5):
        c = bench.workload_shape(cfg)
        a, b = bench.config_obj(c), bench.config_obj(bench.workload_shape(cfg))
        assert a == b and "l2" not in a
        assert a["pairs_per_step"] == c["P"] * c["layers"]
    c4 = bench.workload_shape(4)
    assert (c4["R"], c4["S"], c4["E"], c4["K"], c4["H"], c4["layers"]) == (64, 8192, 384, 8, 7168, 8)
    assert bench.parse([]).config == 4          # the largest single-GPU workload is the default


def test_smaller_case_overrides():
    import bench
    c = bench.workload_shape(4, tokens_per_rank=512, layers=1)
    assert (c["S"], c["T"], c["P"], c["layers"]) == (512, 64 * 512, 64 * 512 * 8, 1)
    assert c["name"] == "fine_grained_ep64_8layers"


def test_oracle_sample_extrapolation():
    """The CPU baseline's layer time: the route ran over the whole layer, the
    rows over Ts tokens, the gradients over nc columns; each phase's time per
    unit times the layer's units."""
    import bench
    c = bench.workload_shape(3)
    Ts, nc = bench.sample_tokens(c), bench.sample_cols(c)
    assert Ts * c["K"] * c["H"] <= (1 << 28) < (Ts + 1) * c["K"] * c["H"]
    assert nc == 1 << 22
    s = bench.layer_seconds(c, 0.5, 2.0, 1.0, Ts, nc)
    assert s == pytest.approx(0.5 + 2.0 * c["T"] / Ts + 1.0 * c["grad_n"] / nc)
    c1 = bench.workload_shape(1)
    assert bench.sample_tokens(c1) == c1["T"] and bench.sample_cols(c1) == c1["grad_n"]
    assert bench.layer_seconds(c1, 0.5, 2.0, 1.0, c1["T"], c1["grad_n"]) == pytest.approx(3.5)


def test_side_measurement_replays():
    import bench
    assert bench.side_steps(20, 0.4) == 20          # short steps: all of them
    assert bench.side_steps(20, 163.0) == 15        # 2.5 s of replays
    assert bench.side_steps(20, 5000.0) == 3        # at least three


def test_reference_arm_runs_on_the_host():
    """bench.py --impl reference (the CPU oracle on a sample of the workload)
    runs on a machine without a GPU and prints one JSON line whose config is
    the one our arm prints for the same workload."""
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    out = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--config", "1",
                          "--steps", "2", "--warmup", "1"], capture_output=True, text=True, timeout=600, cwd=root)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    import bench
    assert line["impl"] == "reference" and line["steps"] == 2 and line["value"] > 0
    assert line["config"] == bench.config_obj(bench.workload_shape(1))
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
