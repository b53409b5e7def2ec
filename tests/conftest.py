import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a)")


@pytest.fixture(scope="session")
def fd():
    """The C-ABI binding (loads libfd.so; builds it first if it is missing)."""
    from streaming_autoregressive_video_b200 import binding
    binding.load()
    return binding
