import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def has_gpu() -> bool:
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if has_gpu():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """How many near-tie exceptions each byte comparison used (tests/parity.py)."""
    try:
        import parity
    except Exception:
        return
    if not parity.EXCEPTIONS:
        return
    tr = terminalreporter
    tr.section("near-tie exceptions in byte comparisons")
    for test, kind, count, total in parity.EXCEPTIONS:
        tr.write_line(f"{count:8d} of {total:11d}  {kind:18s} {test}")
