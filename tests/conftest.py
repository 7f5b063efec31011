import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)
TESTS = os.path.dirname(os.path.abspath(__file__))
if TESTS not in sys.path:
    sys.path.insert(0, TESTS)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle

    oracle.lib()  # builds oracle/libkvqref.so if it is missing or stale
    return oracle


def build_library():
    """Build libkvq.so when it is missing or stale, without importing the package first
    (the package's __init__ loads the library); returns the imported package."""
    import importlib.util

    spec = importlib.util.spec_from_file_location(
        "kvq_build", os.path.join(ROOT, "kv_cache_quantization_fp16_b200", "_build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import kv_cache_quantization_fp16_b200

    return kv_cache_quantization_fp16_b200


@pytest.fixture(scope="session")
def kvq_built():
    return build_library()

