import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_sessionstart(session):
    """The tests call the in-tree libdsa.so; a checkout without it (the library is not tracked) builds it once
    with nvcc, which needs no GPU.  An existing library is used as it is."""
    lib = os.path.join(ROOT, "sparse_attention_long_dsa_b200", "libdsa.so")
    if not os.path.exists(lib):
        from sparse_attention_long_dsa_b200 import build
        build.build()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU case")
