import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU; parity tests of the CUDA path")
    config.addinivalue_line("markers", "slow: full-size workloads")
    config.addinivalue_line(
        "markers", "late: collected after all unmarked tests, so that under -x a failure in one "
        "of these cases stops none of the others")


def pytest_collection_modifyitems(config, items):
    # "late" cases last, the order otherwise unchanged (a stable sort)
    items.sort(key=lambda it: "late" in it.keywords)
    # GPU tests need a device; without one they are reported as skipped rather
    # than silently passing.
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    if have_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)
