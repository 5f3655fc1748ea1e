"""bench.py on a GPU prints the contract's JSON line: one line, the metric,
value and unit, the roofline object with its fields, the end-to-end object
with the copied bytes, the launch count and the clock record.  Runs the tiny
head for a few steps, without the sweeps and the CPU baseline."""
import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_prints_the_contract_line():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "tiny",
                          "--batch", "1", "--steps", "5", "--warmup", "3", "--no-sweep",
                          "--no-cpu-baseline"], capture_output=True, text=True, timeout=600,
                         cwd=ROOT)
    assert out.returncode == 0, out.stderr[-3000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    r = json.loads(lines[0])
    import bench
    assert r["metric"] == bench.METRIC and r["unit"] == bench.UNIT
    assert r["n_gpus"] == 1 and r["steps"] == 5 and r["warmup"] == 3
    assert r["higher_is_better"] is False and r["value"] > 0
    assert r["ms_per_step"] == pytest.approx(r["value"] / 1e3, rel=1e-3)
    rf = r["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic", "regime", "fracs"):
        assert k in rf
    assert rf["bound"] in ("hbm", "tensor") and rf["frac"] == pytest.approx(
        rf["achieved"] / rf["peak"])
    e = r["e2e"]
    assert e["unit"] == bench.UNIT and e["value"] > 0
    assert e["h2d_bytes_per_step"] == 1 * 256 * 2 and e["d2h_bytes_per_step"] == 4
    assert r["gpu_launches"] == 5
    assert set(r["clocks"]) >= {"sm_mhz", "sm_max_mhz", "reasons"}
    assert r["config"]["workload"].startswith("tiny") and r["dtype"] == "bf16"
