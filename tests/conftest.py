import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the CUDA library")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session", autouse=True)
def _cuda_library_built(request):
    """GPU sessions build the in-tree CUDA library first (a no-op when it is up to date),
    so a fresh checkout runs the parity tests on the library of its own sources."""
    if any(item.get_closest_marker("gpu") for item in request.session.items):
        from sparse_moe_transformer_b200 import build
        build.build()
