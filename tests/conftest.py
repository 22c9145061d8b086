import importlib.util
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _build_cuda_library():
    # build.py is loaded by path: importing the package needs the library.
    path = os.path.join(ROOT, "paged_kv_cache_group_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_fp8q_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


_build_cuda_library()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built CUDA library")
