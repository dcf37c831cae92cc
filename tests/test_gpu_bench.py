"""The benchmark's JSON line on a GPU (-m gpu), on the tiny workload so the
run takes seconds: every key the line promises is there and consistent, for
the default arm and for the rank-local form."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                         timeout=900, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-3000:]
    return json.loads(out.stdout.strip().splitlines()[-1])


def test_bench_line_has_every_field():
    line = _run("--config", "1", "--others=", "--steps", "4", "--warmup", "3")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks", "cpu_baseline"):
        assert key in line, key
    assert line["steps"] == 4 and line["warmup"] == 3 and line["n_gpus"] == 1
    assert line["value"] > 0 and line["gpu_launches"] > 0
    P = line["config"]["pairs_per_step"]
    assert line["value"] == pytest.approx(P / (line["ms_per_step"] / 1e3), rel=1e-6)
    r = line["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert abs(r["frac"] - r["achieved"] / r["peak"]) <= 1e-4 + 1e-3 * r["frac"]  # both rounded in the line
    e = line["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert e["value"] == pytest.approx(P / (e["ms_per_step"] / 1e3), rel=1e-6)
    assert "run_host_batches" in e["what"] and e["one_batch_at_a_time"]["value"] > 0  # batches in flight, and alone
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 1


def test_bench_rank_local_line():
    line = _run("--rank-local", "--config", "1", "--steps", "3", "--warmup", "2")
    assert line["value"] > 0 and line["scaling"] == "strong" and line["n_gpus"] == 1
    assert "every peer buffer local" in line["form"]
