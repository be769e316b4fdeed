"""The benchmark's reference arm, run on the CPU: one JSON line with the
contract's keys, the same metric, unit and workload config as the GPU arm,
and the oracle's sample described (no GPU needed)."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "1", "--cpu-tokens", "1"], capture_output=True, text=True, timeout=600,
                         cwd=ROOT, env=dict(os.environ, CUDA_VISIBLE_DEVICES=""))
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["config"] == bench.step_config(1)
    assert d["value"] > 0 and d["steps"] == 1 and d["warmup"] == 1
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and "1 of 8192" in cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_step_accounting():
    # six GEMMs of 2 x 8192 x 8192 x 2048 FLOP each; casts read fp32/bf16 and write y only
    assert bench.STEP_GEMMS == 6
    assert abs(bench.STEP_FLOP - 6 * 2.0 * 8192 * 8192 * 2048) < 1
    assert bench.STEP_CAST_BYTES_FUSED == 3 * 8192 * 2048 * 5 + 8192 * 2048 * 3
    assert bench.LAUNCHES_PER_STEP == 9 and bench.LAUNCHES_PER_STEP_UNFUSED == 12
