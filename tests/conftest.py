import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def build_library():
    """Build libmoe_b200.so (if stale) without importing the package first."""
    import importlib.util
    path = os.path.join(ROOT, "sparse_mixture_experts_24_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_moe_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


import pytest  # noqa: E402


@pytest.fixture(scope="session", autouse=True)
def _library_built():
    """Every test session starts with an up-to-date libmoe_b200.so."""
    build_library()
    yield
