import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity cases")


def load_builder():
    """block_sparse_causal_b200/build.py loaded by path (the package import needs libuf.so)."""
    import importlib.util
    path = os.path.join(ROOT, "block_sparse_causal_b200", "build.py")
    spec = importlib.util.spec_from_file_location("uf_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.fixture(scope="session")
def built_lib():
    """Build libuf.so when stale, then import the binding."""
    load_builder().build()
    import block_sparse_causal_b200 as uf
    return uf
