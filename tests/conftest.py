import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def lib():
    """The built C-ABI library (built in-tree on first use if it is missing or stale)."""
    from quantized_kv_cache_19_b200 import build as qbuild
    qbuild.build_library(quiet=True)
    from quantized_kv_cache_19_b200 import api
    return api.load_library()
