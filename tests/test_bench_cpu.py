"""The bench's CPU-side legs without a GPU: the reference arm (the float64 oracle
timed on the host cores) prints one well-formed JSON line, in every sampler mode,
at a reduced vocabulary so that it runs in seconds."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("extra", [[], ["--accept", "sample"], ["--rule", "group"]])
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


def test_warmup_floor():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "2"], capture_output=True,
                         text=True, timeout=120, cwd=ROOT)
    assert out.returncode != 0 and "warmup" in out.stderr
