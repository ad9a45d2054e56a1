"""Build-time guards (no GPU): the hot kernels compile for sm_100a without register spills or
a stack frame, as reported by ptxas (-Xptxas -v).  A spill in the fused pass would put the
softmax's 64-logit register tiles through local memory."""

import os
import re
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "discrete_diffusion_decoding_b200", "csrc")


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    pytest.skip("nvcc not available")


def _ptxas_report(src, tmp_path):
    out = subprocess.run([_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                          "-Xptxas", "-v", "-c", "-o", str(tmp_path / "k.o"), os.path.join(CSRC, src)],
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    report, current = {}, None
    for line in out.stderr.splitlines():
        m = re.search(r"Function properties for (\S+)", line)
        if m:
            current = m.group(1)
            continue
        m = re.search(r"(\d+) bytes stack frame, (\d+) bytes spill stores, (\d+) bytes spill loads", line)
        if m and current:
            report[current] = tuple(int(x) for x in m.groups())
    return report


def test_fused_and_combine_kernels_do_not_spill(tmp_path):
    rep = _ptxas_report("dg_fused.cu", tmp_path)
    wanted = {"dg_fused_kernel": None, "dg_fused_sample_kernel": None, "dg_combine_kernel": None}
    for name, frame in rep.items():
        for k in wanted:
            if k in name:
                wanted[k] = frame
    for k, frame in wanted.items():
        assert frame is not None, f"{k} missing from the ptxas report"
        assert frame == (0, 0, 0), f"{k}: stack frame / spill stores / spill loads = {frame}"


def test_small_kernels_do_not_spill(tmp_path):
    rep = _ptxas_report("dg_small.cu", tmp_path)
    assert rep, "no kernels in the ptxas report"
    for name, frame in rep.items():
        assert frame[1:] == (0, 0), f"{name}: spill stores / loads = {frame[1:]}"
