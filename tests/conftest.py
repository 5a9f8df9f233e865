import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA (B200, sm_100a) device")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")


def pytest_collection_modifyitems(config, items):
    """Skip GPU tests on a machine without a CUDA device only when they were not asked for.

    ``-m gpu`` on a machine without a GPU fails loudly instead of skipping, so
    that a missing device or extension can never pass as green.
    """
    import torch
    markexpr = config.getoption("-m") or ""
    if torch.cuda.is_available() or "gpu" in markexpr.replace("not gpu", ""):
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)
