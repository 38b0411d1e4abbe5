import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: takes more than a few seconds")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


def pytest_sessionstart(session):
    # Build (or refresh) the native libraries once per session; nvcc cross-compiles
    # sm_100a without a GPU.  Nothing falls back if this fails.
    from paged_kv_cache_403_b200 import build
    import oracle.build
    build.build_all()
    oracle.build.build()
