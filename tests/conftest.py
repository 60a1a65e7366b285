import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device in this process")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter):
    """The errors of every GPU-vs-oracle comparison of the run."""
    try:
        from helpers import STATS
    except ImportError:  # pragma: no cover
        return
    if not STATS:
        return
    tr = terminalreporter
    tr.section("parity errors against the float64 oracle")
    for what, s in STATS:
        tr.write_line(f"{what:<60s} max_abs {s['max_abs']:.3e}  mean_abs {s['mean_abs']:.3e}  "
                      f"rel {s['rel']:.3e}")
