import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


@pytest.fixture(scope="session", autouse=True)
def _built_library():
    """Compile libmla.so in-tree (nvcc, sm_100a) when it is missing or older than its sources."""
    from mla_latent_kv_window_b200 import build
    build.build()
    yield
