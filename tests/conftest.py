import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def gpu_available() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if gpu_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    try:
        import parity
    except ImportError:
        return
    if not parity.REPORT:
        return
    terminalreporter.write_sep("-", "parity coverage (groups)")
    for where, counts in parity.REPORT:
        terminalreporter.write_line(f"{where}: " + ", ".join(f"{k}={v}" for k, v in counts.items()))
