import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")


def _cuda_available():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if _cuda_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device on this machine")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


# (workload, dtype, max abs error, mean abs error) of the named-workload parity
# checks, printed after the run so a log carries the achieved accuracy
PARITY_REPORT = []


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    if not PARITY_REPORT:
        return
    terminalreporter.write_sep("-", "parity against the fp64 oracle (named workloads)")
    for name, dtype, mx, mean in PARITY_REPORT:
        terminalreporter.write_line(f"{name:12s} {dtype:9s} max abs {mx:.3e}  mean abs {mean:.3e}")
