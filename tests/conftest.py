"""Shared pytest configuration: the ``gpu`` marker and repository imports."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line(
        "markers", "slow: a CPU test that takes more than a few seconds")


def pytest_terminal_summary(terminalreporter):
    """The largest |y - y_ref| / tolerance of each test that compared fp32
    outputs (1.0 would be at the bound); also written to the file named by
    NVQ_MARGIN_LOG when set."""
    try:
        from parity import MARGINS
    except ImportError:
        return
    if not MARGINS:
        return
    worst = {}
    for test, ratio in MARGINS:
        worst[test] = max(ratio, worst.get(test, 0.0))
    lines = [f"{ratio:.4f}  {test}" for test, ratio in sorted(worst.items(), key=lambda kv: -kv[1])]
    terminalreporter.write_sep("-", "max err / tolerance per test (largest first)")
    for line in lines[:25]:
        terminalreporter.write_line(line)
    path = os.environ.get("NVQ_MARGIN_LOG")
    if path:
        with open(path, "w") as f:
            f.write("\n".join(lines) + "\n")
