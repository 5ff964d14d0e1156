import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_sessionstart(session):
    # build the CUDA library (nvcc cross-compiles without a GPU) and the C
    # oracle if they are missing or stale
    import importlib.util

    spec = importlib.util.spec_from_file_location(
        "_spkv_build", os.path.join(ROOT, "compressed_kv_decode_ada_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import oracle

    oracle.build()


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle

    oracle.build()
    return oracle
