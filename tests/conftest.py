import importlib.util
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _ensure_built():
    """Build libbnb4.so in-tree if it is missing or stale (nvcc cross-compiles without a GPU)."""
    path = os.path.join(ROOT, "bit_blockwise_weight_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_bnb4_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


_ensure_built()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")
