import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")


def _ensure_library():
    """Build libpagedkv.so if it is missing (nvcc cross-compiles; no GPU needed)."""
    lib = os.path.join(ROOT, "paged_kv_cache_440_b200", "libpagedkv.so")
    if not os.path.exists(lib):
        # load build.py by path: importing the package needs the library itself
        import importlib.util
        spec = importlib.util.spec_from_file_location(
            "_pagedkv_build", os.path.join(ROOT, "paged_kv_cache_440_b200", "build.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod.build()


_ensure_library()
