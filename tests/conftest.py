import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _build_library():
    """Compile libpoem.so if it is missing or stale, loading the build script by path:
    importing the package first would fail (it refuses to import without the library)."""
    import importlib.util

    path = os.path.join(ROOT, "block_sparse_attention_poem_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_poem_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    _build_library()


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle

    oracle.build()
    return oracle
