import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


@pytest.fixture(scope="session", autouse=True)
def _built_library():
    """Compile liblora_gemm.so if it is missing or older than its sources."""
    from lora_gemm_b200 import build

    build.build()
    yield
