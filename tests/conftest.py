import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200); parity and kernel tests")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Report the largest elementwise relative errors the parity tests saw."""
    mod = sys.modules.get("flhelpers")
    if mod is None or not getattr(mod, "ELEMENTWISE", None):
        return
    ELEMENTWISE, ELEM_FLOOR = mod.ELEMENTWISE, mod.ELEM_FLOOR
    terminalreporter.write_sep("-", f"elementwise relative error (floor {ELEM_FLOOR:g} x ||ref||_inf per head)")
    for label in sorted(ELEMENTWISE):
        terminalreporter.write_line(f"{label}: {ELEMENTWISE[label]:.3e}")
