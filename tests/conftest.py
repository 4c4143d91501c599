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
    """Compile liblora_gemm.so if it is missing or older than its sources.

    The build script is loaded by path: importing the package would load the
    (possibly stale) library first."""
    import importlib.util

    spec = importlib.util.spec_from_file_location("_lg_build", os.path.join(ROOT, "lora_gemm_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    yield
