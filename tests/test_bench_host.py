"""bench.py's measurement arithmetic and its reference arm, on the CPU.

The roofline figures the benchmark reports are algorithmic: bytes that must
cross HBM (W once, H once, the tokens, the mask if any) and the matmul's
flops per call, divided by the measured kernel time and compared with the
measured peak of the bound that is larger for that shape.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

PEAKS = {"hbm_gbs": 6457.7, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1391.4}


def test_algorithmic_bytes_and_flops():
    """Qwen3-8B-shaped head, B=64: W once (1,244,659,712 bytes), H once, four
    bytes per token; a mask adds one bit per (row, token) in 32-bit words."""
    nbytes, flops = bench.algorithmic(64, 4096, 151936, False)
    assert nbytes == 151936 * 4096 * 2 + 64 * 4096 * 2 + 64 * 4
    assert flops == 2 * 64 * 151936 * 4096
    masked, _ = bench.algorithmic(3, 4096, 151937, True)
    assert masked - bench.algorithmic(3, 4096, 151937, False)[0] == 3 * 4749 * 4


def test_roofline_picks_the_larger_bound():
    """At the measured peaks, streaming W takes longer than the matmul at B=64
    (HBM-bound) and shorter at B=256 (tensor-bound); the fraction is the
    achieved rate over that bound's peak."""
    r = bench.roofline(64, 4096, 151936, False, 200.0, PEAKS, "measured", 123)
    nbytes, _ = bench.algorithmic(64, 4096, 151936, False)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] == PEAKS["hbm_gbs"]
    assert r["achieved"] == pytest.approx(nbytes / 200e-6 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / PEAKS["hbm_gbs"])
    assert r["traffic"] == 123
    t = bench.roofline(256, 4096, 151936, False, 340.0, PEAKS, "measured", None)
    assert t["bound"] == "tensor" and t["unit"] == "TFLOP/s"
    assert t["regime"] == "burst" and t["peak"] == PEAKS["bf16_tflops"]
    assert t["achieved"] == pytest.approx(2 * 256 * 151936 * 4096 / 340e-6 / 1e12)
    assert t["traffic"] is None
    assert t["fracs"]["tensor_burst"] == pytest.approx(t["achieved"] / PEAKS["bf16_tflops"], abs=1e-4)
    assert t["fracs"]["tensor_sustained"] == pytest.approx(
        t["achieved"] / PEAKS["bf16_tflops_sustained"], abs=1e-4)
    u = bench.roofline(256, 4096, 151936, False, 340.0, PEAKS, "measured", None, "sustained")
    assert u["regime"] == "sustained" and u["peak"] == PEAKS["bf16_tflops_sustained"]


def test_regime_follows_the_region_length():
    """A region of a second or more runs at the board's power limit (the
    sustained bf16 peak); shorter ones take the burst peak."""
    assert bench.regime_of(0.004) == "burst"
    assert bench.regime_of(0.999) == "burst"
    assert bench.regime_of(1.0) == "sustained"
    assert bench.regime_of(2.5) == "sustained"


def test_percentiles_and_median():
    """Nearest-rank percentiles: the ceil(q n / 100)-th smallest value."""
    assert bench.percentiles(list(range(100, 0, -1))) == [10, 50, 90]
    assert bench.percentiles([5, 1, 4, 2, 3, 7, 6]) == [1, 4, 7]
    assert bench.percentiles([42]) == [42, 42, 42]
    assert bench.median([3.0, 1.0, 2.0]) == 2.0


def test_workload_config_names_the_workload():
    from lm_head_exact_fmms_b200 import synth
    wl = synth.WORKLOADS["qwen3-8b"]
    c = bench.workload_config(wl, 64, 1)
    assert c["batch_per_gpu"] == 64 and c["global_batch"] == 64
    assert c["d"] == 4096 and c["V"] == 151936
    assert "exceeds the 126 MB L2" in c["l2"]
    assert "model" not in c
    c8 = bench.workload_config(wl, 64, 8, tp=True, fused_tp=True)
    assert c8["global_batch"] == 512 and "fused peer-memory exchange" in c8["parallelism"]


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` (the CPU oracle) on the tiny head: one JSON
    line with the metric, unit and config of the GPU arm, `impl` reference,
    a cpu_baseline describing the run and an e2e object with no copies."""
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--batch", "1", "--steps", "3", "--warmup", "1"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    r = json.loads(lines[0])
    assert r["impl"] == "reference" and r["metric"] == bench.METRIC and r["unit"] == bench.UNIT
    assert r["steps"] == 3 and r["warmup"] == 1 and r["higher_is_better"] is False
    assert r["value"] > 0 and r["dtype"] == "f64" and r["n_gpus"] == 1
    assert r["cpu_baseline"]["kind"] == "oracle" and r["cpu_baseline"]["cores"] >= 1
    assert r["cpu_baseline"]["value"] == r["value"]
    assert r["e2e"] == {"value": r["value"], "unit": bench.UNIT, "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert r["config"]["V"] == 4096 and r["config"]["d"] == 256


def test_nvtx_sections_are_transparent():
    """The NVTX section wrapper runs its body and lets its exceptions through."""
    ran = []
    with bench.nvtx("section"):
        ran.append(1)
    with pytest.raises(KeyError):
        with bench.nvtx("failing section"):
            raise KeyError("k")
    assert ran == [1]


def test_clock_sampler_keeps_only_samples_inside_the_region():
    """The sampler starts before the warm-up; the summary counts only samples
    stamped inside the timed region's host window, and their reasons."""
    s = bench.ClockSampler(0)
    s._nvml = object()          # as if NVML answered (no GPU here)
    s.max_mhz = 1965
    s.stamped = [(0.5, 1965, 0x1), (1.0, 1500, 0x4), (1.5, 1480, 0x4), (2.5, 1965, 0x8)]
    s.set_window(0.9, 2.0)
    r = s.summary()
    assert r["samples"] == 2 and r["sm_mhz"] in (1480, 1500)
    assert r["reasons"] == ["sw_power_cap"] and r["sm_max_mhz"] == 1965


def test_clock_sampler_samples_from_the_polling_thread():
    """sample_now() queries from the calling thread and stamps the sample at
    the middle of its queries, so a region shorter than one query of a slow
    NVML still holds the sample taken while it drained."""
    import types
    import time as _time

    calls = []

    def clock(h, which):
        calls.append("clock")
        _time.sleep(0.002)
        return 1700

    def reasons(h):
        calls.append("reasons")
        _time.sleep(0.002)
        return 0x4

    s = bench.ClockSampler(0)
    s._nvml = types.SimpleNamespace(nvmlDeviceGetClockInfo=clock, NVML_CLOCK_SM=1,
                                    nvmlDeviceGetCurrentClocksEventReasons=reasons)
    s._h = None
    s.max_mhz = 1965
    t0 = _time.perf_counter()
    s.sample_now()
    t1 = _time.perf_counter()
    assert calls == ["clock", "reasons"] and len(s.stamped) == 1
    t, mhz, bits = s.stamped[0]
    assert t0 < t < t1 and mhz == 1700 and bits == 0x4
    # A window that opens after the first query began and closes before
    # the last one ended still keeps it.
    s.set_window(t0 + 0.001, t1 - 0.001)
    r = s.summary()
    assert r["samples"] == 1 and r["sm_mhz"] == 1700 and r["reasons"] == ["sw_power_cap"]
