import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long CPU-side oracle run")


def pytest_terminal_summary(terminalreporter):
    """Rows compared with the oracle and rows excluded by the near-tie / near-bound rule, per check."""
    mod = sys.modules.get("gpu_case")
    rows = getattr(mod, "REPORT", None) if mod else None
    if not rows:
        return
    tr = terminalreporter
    tr.section("oracle comparisons (rows compared / excluded)")
    tot_r = tot_x = 0
    for tag, n, x, extra in rows:
        tr.write_line(f"{tag}: {n} rows, {x} excluded {extra}".rstrip())
        tot_r += n
        tot_x += x
    tr.write_line(f"total: {tot_r} rows compared, {tot_x} excluded")
