import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_sessionstart(session):
    """Build libloopkv.so (nvcc, sm_100a) when a source is newer than it, so
    that a fresh checkout tests what it builds.  The build module is loaded
    from its file: importing the package needs the library first."""
    import importlib.util
    path = os.path.join(ROOT, "mixed_precision_kv_loopkv_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_loopkv_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")
