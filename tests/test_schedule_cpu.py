"""The fused kernel's work schedule, checked on the host (no GPU): exact coverage,
slot bounds, balance, and agreement between the fused kernel and the combine."""

import os
import subprocess
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_schedule_exact_cover_and_slots():
    src = os.path.join(ROOT, "tests", "csrc", "schedule_check.cu")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "schedule_check")
        nvcc = "/usr/local/cuda/bin/nvcc" if os.path.exists("/usr/local/cuda/bin/nvcc") else "nvcc"
        subprocess.run([nvcc, "-std=c++17", "-O1", "-o", exe, src], check=True, capture_output=True)
        res = subprocess.run([exe], capture_output=True, text=True)
        assert res.returncode == 0, res.stdout[-2000:]
        assert "fails=0" in res.stdout
