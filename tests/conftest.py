import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: oracle runs of several seconds")


def pytest_runtest_setup(item):
    if item.get_closest_marker("gpu") is None:
        return
    import torch
    if not torch.cuda.is_available():
        if os.path.exists("/dev/nvidiactl"):
            pytest.fail("a GPU test found a driver node but no usable CUDA device")
        pytest.skip("no CUDA device on this machine")
