"""Shared pytest configuration: markers and the repository import path."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built libtq.so")


def require_cuda():
    """GPU tests fail loudly (never skip) when no device is present."""
    import torch
    if not torch.cuda.is_available():
        pytest.fail("this test needs a CUDA device (run the -m gpu tests on a machine with one)")


GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
