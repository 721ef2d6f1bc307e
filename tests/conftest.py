import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size systems (minutes of CPU work)")


def pytest_collection_modifyitems(config, items):
    # GPU tests on a machine without a GPU are skipped only when not explicitly
    # selected with -m gpu; when selected, a missing GPU is a failure.
    markexpr = config.getoption("-m") or ""
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:
        have_gpu = False
    if have_gpu or "gpu" in markexpr and "not gpu" not in markexpr:
        return
    skip = pytest.mark.skip(reason="no CUDA GPU on this machine")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)
