"""bench.py on the GPU: one short run prints one JSON line that keeps the
bench contract -- the metric and config of the workload, the roofline of the
attention kernel (its launch time inside the step, so 28 launches fit in a
step), the GPU-vs-oracle parity check of the timed call, the end-to-end
figure with its copies declared, the clock record and the launch count."""
import json
import os
import subprocess
import sys

import pytest

from gpu_util import require_gpu

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_line_keeps_the_contract():
    require_gpu()
    r = subprocess.run([sys.executable, "bench.py", "--steps", "5", "--warmup", "3", "--no-extras",
                        "--cpu-seconds", "1"], cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    sys.path.insert(0, ROOT)
    import bench
    assert j["metric"] == bench.METRIC and j["unit"] == bench.UNIT and j["n_gpus"] == 1
    assert j["steps"] == 5 and j["warmup"] == 3 and j["value"] > 0 and j["higher_is_better"] is True
    assert j["config"] == bench.config_dict(1)
    rf = j["roofline"]
    assert rf["bound"] == "tensor" and rf["unit"] == "TFLOP/s" and 0 < rf["frac"] < 1.2
    assert abs(rf["achieved"] - bench.ATTN_FLOP / (rf["avg_launch_us"] * 1e-6) / 1e12) < 0.01 * rf["achieved"]
    assert bench.BLOCKS * rf["avg_launch_us"] * 1e-3 <= rf["run_ms"] / 5 * 1.0001
    assert j["gpu_launches"] == 5 * (1 + bench.BLOCKS)
    e = j["e2e"]
    assert e["h2d_bytes_per_step"] == 3 * bench.BLOCKS * bench.R * bench.HEADS * bench.D * 2
    assert e["d2h_bytes_per_step"] == bench.BLOCKS * bench.R * bench.HEADS * bench.D * 2
    assert 0 < e["value"] <= j["value"] * 1.05
    par = j["cpu_baseline"]["gpu_parity"]
    assert par["buffers"] == "bit-exact" and par["rel_l2"] <= 5e-3 and par["max_abs"] <= 2e-2
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["cores"] >= 1
    assert "sm_mhz" in j["clocks"] and "reasons" in j["clocks"]
