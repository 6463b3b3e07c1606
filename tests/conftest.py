import importlib.util
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running host test")


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def build_library():
    """Compile libtasq.so if stale and return the imported package. The build script is loaded
    by its path: importing the package first would load the library it is about to build."""
    spec = importlib.util.spec_from_file_location(
        "_tasq_build", os.path.join(ROOT, "timestep_adaptive_bit_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import timestep_adaptive_bit_b200
    return timestep_adaptive_bit_b200
