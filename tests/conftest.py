import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a) and the built library")


@pytest.fixture(scope="session", autouse=True)
def _built_library():
    """Build librssm.so in-tree if it is missing or stale (nvcc, no GPU needed)."""
    from hybrid_ssm_decode_replayssm_b200 import build
    build.build()
