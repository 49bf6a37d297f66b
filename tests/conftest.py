import importlib.util
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a) and the built library")
    config.addinivalue_line("markers", "slow: longer CPU test")
    # a tree that was never built (a fresh checkout): compile liblsa.so first, by the build script's
    # path (importing the package would load the library it is about to build)
    lib = os.path.join(ROOT, "sparse_kv_cache_memoryindexer_b200", "liblsa.so")
    if not os.path.exists(lib) and shutil.which("nvcc"):
        spec = importlib.util.spec_from_file_location(
            "_lsa_build", os.path.join(ROOT, "sparse_kv_cache_memoryindexer_b200", "build.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod.build()
