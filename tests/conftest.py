import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built library")


def build_library():
    """Compile liblcsa.so if stale (build script loaded by path) and import the binding."""
    import importlib.util
    path = os.path.join(ROOT, "long_context_compressed_softmax_b200", "build.py")
    spec = importlib.util.spec_from_file_location("lcsa_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    import long_context_compressed_softmax_b200 as m
    return m
