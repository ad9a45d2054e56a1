"""The bench's GPU arm prints the one JSON line its readers parse, with every key they read.

Runs `bench.py` as a subprocess at the default workload for a few steps (the CPU
baseline leg included, on its bounded sample) and checks the line's shape and the
consistency of its numbers: the metric, the roofline block (the measured kernel time,
FLOPs and the fraction that follows from them, and the committed DRAM traffic while the
library source matches its profile), the CPU baseline, the end-to-end block with its
copy sizes, the launch count and both clock readings.
"""

import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, timeout=900):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True, text=True,
                         timeout=timeout, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-3000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


def test_bench_line_has_the_contract_keys():
    d = _run(["--steps", "5", "--warmup", "3"])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e", "gpu_launches", "clocks"):
        assert k in d, k
    assert d["metric"].startswith("canvas positions/s per denoise step") and d["unit"] == "positions/s"
    assert d["n_gpus"] == 1 and d["steps"] == 5 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["scaling"] == "weak" and d["dtype"] == "bf16" and d["data"] == "synthetic"
    assert "workload" in d["config"] and d["config"]["vocab"] == 262144 and d["config"]["hidden"] == 2816
    assert abs(d["value"] - 256 / (d["ms_per_step"] * 1e-3)) <= 1e-6 * d["value"]
    r = d["roofline"]
    for k in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert k in r, k
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert abs(r["achieved"] - r["flops_per_launch"] / (r["kernel_ms"] * 1e-3) / 1e12) <= 1e-6 * r["achieved"]
    assert abs(r["frac"] - r["achieved"] / r["peak"]) <= 1e-9
    assert r["kernel_ms"] <= d["ms_per_step"]
    sys.path.insert(0, ROOT)
    import bench
    assert r["traffic"] == bench.profiled_traffic()            # committed capture, or null once stale
    c = d["cpu_baseline"]
    assert c["kind"] == "oracle" and c["cores"] >= 1 and c["value"] > 0 and c["unit"] == "positions/s"
    e = d["e2e"]
    assert e["unit"] == "positions/s" and e["value"] > 0
    assert e["h2d_bytes_per_step"] == 256 * 2816 * 2                       # h, bf16
    assert e["d2h_bytes_per_step"] == 13 * 256 + 256 * 2816 * 4            # packed results + self-conditioning
    assert d["gpu_launches"] == 3 * 5
    k = d["clocks"]
    assert "sm_mhz" in k and "sm_max_mhz" in k and "reasons" in k
    assert 300.0 < k["kernel_sm_mhz"] < 2200.0
