import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    oracle._load()
    return oracle


def build_library():
    """Compile libpa_b200.so if stale, loading the build script by path (importing the
    package itself needs the library to exist already)."""
    import importlib.util
    path = os.path.join(ROOT, "paged_kv_cache_389_b200", "build.py")
    spec = importlib.util.spec_from_file_location("pa_b200_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


@pytest.fixture(scope="session")
def pa():
    build_library()
    import paged_kv_cache_389_b200 as pa
    return pa
