import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")
    config.addinivalue_line("markers", "slow: full-size workloads")


def pytest_collection_modifyitems(config, items):
    # GPU tests are skipped (not failed) when no CUDA device is visible, so the
    # CPU suite can run with -m "not gpu" or without a marker filter.
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    # the parity figures the GPU tests reported (tests/_cases.py: report), one per line
    mod = sys.modules.get("_cases")
    lines = getattr(mod, "PARITY_REPORT", None) if mod is not None else None
    if lines:
        terminalreporter.section("parity against the oracle: beyond-rounding and raw max|err|/RMS")
        for line in lines:
            terminalreporter.write_line(line)
