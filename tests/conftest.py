import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a) and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device visible")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """Largest parity errors observed in the session, per quantity."""
    try:
        from s6_testutil import OBSERVED
    except ImportError:  # pragma: no cover
        return
    if not OBSERVED:
        return
    terminalreporter.write_sep("-", "largest observed max|got-ref|/(1+|ref|)")
    for k in sorted(OBSERVED):
        terminalreporter.write_line(f"{k:40s} {OBSERVED[k]:.3e}")
