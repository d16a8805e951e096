"""bench.py's reference arm (the fp64 oracle on the host cores) needs no GPU:
run it and check the JSON line the driver reads."""
from __future__ import annotations

import json
import os
import subprocess
import sys
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("workload", ["tiny", "qkv_proj_qknorm", "tp_qknorm"])
def test_reference_arm_json_line(workload):
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", workload,
                        "--steps", "1", "--warmup", "0"], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "higher_is_better", "scaling",
                "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["dtype"] == "f64" and d["data"] == "synthetic"
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["config"]["workload"] == workload
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["ms_per_step"] > 0
    # the same metric string as the GPU arm's line for this workload, so the two lines compare
    sys.path.insert(0, ROOT)
    import bench
    expected = {"tiny": bench.METRIC_QK, "qkv_proj_qknorm": bench.METRIC_QKV, "tp_qknorm": bench.METRIC_TP}
    assert d["metric"] == expected[workload]


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1")
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0"],
                       cwd=ROOT, capture_output=True, text=True, timeout=120, env=env)
    assert r.returncode == 0 and not [l for l in r.stdout.splitlines() if l.startswith("{")]


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _sampler_with(rows, t0, t1):
    """A ClockSampler whose nvidia-smi output is `rows` (timestamp, sm MHz, reasons)."""
    import tempfile
    sys.path.insert(0, ROOT)
    import bench
    fd, path = tempfile.mkstemp(suffix=".csv")
    with os.fdopen(fd, "w") as f:
        for ts, sm, cap, thermal in rows:
            stamp = time.strftime("%Y/%m/%d %H:%M:%S", time.localtime(ts)) + f".{int(round((ts % 1) * 1000)):03d}"
            f.write(f"{stamp}, 0, {sm}, 1965, 700.0, 0x0, Not Active, {thermal}, Not Active, {cap}\n")
    cs = bench.ClockSampler()
    cs.proc, cs.path, cs.t0, cs.t1 = _FakeProc(), path, t0, t1
    return cs


def test_clock_sampler_keeps_the_timed_window():
    base = 1_700_000_000.0
    rows = [(base + 0.1 * i, 1965 if i < 10 else 1500, "Not Active" if i < 10 else "Active", "Not Active")
            for i in range(30)]
    # window 1.0 .. 1.5 s: samples 9 .. 16 with one period of margin; 1500 MHz and sw_power_cap dominate
    clk = _sampler_with(rows, base + 1.0, base + 1.5).stop(gpu_index=0)
    assert clk["sm_mhz"] == 1500.0 and clk["sm_max_mhz"] == 1965.0
    assert clk["reasons"] == ["sw_power_cap"]
    assert 6 <= clk["samples"] <= 8


def test_clock_sampler_short_window_takes_the_nearest_samples():
    base = 1_700_000_000.0
    rows = [(base + 0.5 * i, 1965 - 10 * i, "Not Active", "Not Active") for i in range(10)]
    # a 10 ms window between two samples 0.5 s apart: the two nearest samples
    clk = _sampler_with(rows, base + 2.20, base + 2.21).stop(gpu_index=0)
    assert clk["samples"] == 2 and clk["sm_mhz"] == (1965 - 40 + 1965 - 50) / 2


def test_clock_sampler_reports_thermal_slowdown():
    base = 1_700_000_000.0
    rows = [(base + 0.1 * i, 1800, "Not Active", "Active" if i == 3 else "Not Active") for i in range(8)]
    clk = _sampler_with(rows, base, base + 0.7).stop(gpu_index=0)
    assert "hw_thermal_slowdown" in clk["reasons"]


def test_at_max_clock_scales_by_the_sampled_clock():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.at_max_clock(600.0, {"sm_mhz": 1474.0, "sm_max_mhz": 1965.0}) == 600.0 * 1474.0 / 1965.0
    assert bench.at_max_clock(600.0, {"sm_mhz": None, "sm_max_mhz": 1965.0}) is None
    assert bench.at_max_clock(600.0, None) is None
