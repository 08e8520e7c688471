import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: full-size workloads (large device memory)")


def pytest_runtest_setup(item):
    # A GPU test on a machine without a GPU is a failure, not a skip: the CUDA
    # path has no CPU fallback and must not pass silently.
    if item.get_closest_marker("gpu") is not None:
        import torch
        if not torch.cuda.is_available():
            pytest.fail("GPU test needs a CUDA device; none is visible")
