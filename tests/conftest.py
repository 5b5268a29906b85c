import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built libfocus.so")


def pytest_collection_modifyitems(config, items):
    # A gpu test without a GPU is a setup problem, not a pass: skip it with a reason
    # only when CUDA is absent (the CPU suite is run with -m "not gpu").
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


def pytest_terminal_summary(terminalreporter):
    """One line per workload with the parity counts the GPU tests recorded: elements
    (or blocks) checked, the populations of the rounding bands and the mismatches,
    which the tests hold at or below 1e-6 of the elements."""
    from tests.parity import RECORD
    if not RECORD:
        return
    terminalreporter.write_sep("-", "parity counts")
    for name in sorted(RECORD):
        c = RECORD[name]
        terminalreporter.write_line(name + ": " + ", ".join(f"{k} {v}" for k, v in c.items()))
