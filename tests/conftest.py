import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA B200 (sm_100a) device")


def _cuda_available():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def pytest_collection_modifyitems(config, items):
    if _cuda_available():
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


# Error figures of the parity tests on the named workloads, printed at the end
# of the run so that a record of the run carries the margins, not only a
# pass/fail bit.
PARITY_RECORDS = []


def pytest_terminal_summary(terminalreporter):
    if not PARITY_RECORDS:
        return
    terminalreporter.write_sep("-", "parity against the float64 oracle (error / bar)")
    for label, e, bar in PARITY_RECORDS:
        figs = "  ".join(f"{k}={e[k]:.3e} ({e[k] / b:.2f})" for k, b in bar.items())
        terminalreporter.write_line(f"{label}: {figs}")
