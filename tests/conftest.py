import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (sm_100a B200)")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")


def build_library():
    """Compile libhinm.so if a source is newer (loaded by path: importing the package
    needs the library to exist)."""
    import importlib.util
    path = os.path.join(ROOT, "pruning_hinm_spmm_b200", "build_lib.py")
    spec = importlib.util.spec_from_file_location("hinm_build_lib", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()
