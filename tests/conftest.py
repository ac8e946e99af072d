import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def pytest_collection_modifyitems(config, items):
    # gpu tests are skipped, not failed, when no GPU is present and the run
    # did not select them explicitly
    if config.option.markexpr.strip() == "not gpu":
        return  # deselected anyway: no need to import torch to ask for a GPU
    try:
        import torch
        have_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        have_gpu = False
    # an explicit "-m gpu" run must fail loudly without a GPU, never skip
    if have_gpu or config.option.markexpr.strip() == "gpu":
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
