import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built library")
    config.addinivalue_line("markers", "slow: full-size parity case (minutes of oracle time)")


def _has_cuda():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if _has_cuda():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """Print every GPU-vs-oracle layer comparison (mismatches before and after the
    near-tie replay, forced decisions and their largest distance from a tie, scale
    and loss differences), so that the achieved tolerances are on record even in
    a quiet run."""
    mod = sys.modules.get("tests.parity")
    lines = getattr(mod, "REPORT", None) if mod is not None else None
    if not lines:
        return
    terminalreporter.write_sep("-", "parity against the float64 oracle")
    for line in lines:
        terminalreporter.write_line(line)
