import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
HERE = os.path.dirname(os.path.abspath(__file__))
if HERE not in sys.path:
    sys.path.insert(0, HERE)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: full-size case, minutes of oracle time")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Parity counts per configuration: requests compared bit-exactly with the
    oracle, compared after resolving near ties toward the GPU's nodes, and
    excluded (not matched either way)."""
    try:
        from gpu_util import REPORT
    except Exception:  # pragma: no cover
        return
    if not REPORT:
        return
    terminalreporter.write_line("parity (requests: exact / near-tie resolved / excluded):")
    for label, (n, ex, res, exc) in REPORT.items():
        terminalreporter.write_line(f"  {label}: {n}: {ex} / {res} / {exc}")
