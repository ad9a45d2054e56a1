"""The bench's CPU-side legs without a GPU: the reference arm (the float64 oracle
timed on the host cores) prints one well-formed JSON line, in every sampler mode,
at a reduced vocabulary so that it runs in seconds."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("extra", [[], ["--accept", "sample"], ["--rule", "group"], ["--logits", "e4m3"]])
def test_reference_arm_json_line(extra):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--vocab", "4096",
           "--steps", "2", "--warmup", "3"] + extra
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "positions/s" and d["higher_is_better"] is True
    assert d["value"] > 0 and d["steps"] == 2 and d["warmup"] == 3 and d["dtype"] == "f64"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert "V=4096" in d["config"]["workload"]
    if extra == ["--accept", "sample"]:
        assert "Gumbel-max" in d["config"]["workload"]
    if extra == ["--rule", "group"]:
        assert "cumulative entropy" in d["config"]["workload"]
    if extra == ["--logits", "e4m3"]:
        assert "E4M3" in d["config"]["workload"]


def test_warmup_floor():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "2"], capture_output=True,
                         text=True, timeout=120, cwd=ROOT)
    assert out.returncode != 0 and "warmup" in out.stderr


def test_peak_follows_the_timed_regime():
    """The roofline peak is the burst bf16 figure unless the timed region lasted a second or more
    with the power cap active, where the sustained (seconds-long loop) figure applies."""
    sys.path.insert(0, ROOT)
    import bench
    pk = {"bf16_tflops": 1644.9, "bf16_tflops_sustained": 1403.3}
    assert bench.choose_peak(pk, 0.013, {"reasons": []}) == (1644.9, "burst")
    assert bench.choose_peak(pk, 0.013, {"reasons": ["sw_power_cap"]}) == (1644.9, "burst")
    assert bench.choose_peak(pk, 2.4, {"reasons": []}) == (1644.9, "burst")
    assert bench.choose_peak(pk, 2.4, {"reasons": ["sw_power_cap"]}) == (1403.3, "sustained")


def test_clock_summary_keeps_the_timed_window():
    sys.path.insert(0, ROOT)
    import bench
    c = bench.ClockSampler(0)
    c.max_mhz = 1965
    c.rows = [(1.0, 1965, 300.0, 0x0), (2.0, 1900, 900.0, 0x4), (2.5, 1850, 950.0, 0x4), (4.0, 1000, 300.0, 0x8)]
    s = c.summary(1.5, 3.0)
    assert s["samples"] == 2 and s["sm_mhz"] == 1875 and s["reasons"] == ["sw_power_cap"] and s["sm_max_mhz"] == 1965
    assert c.summary(5.0, 6.0)["reasons"] == ["no samples"]
