import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _build_native():
    """Build libmoe.so (by the build script's path) before any test imports the package, which loads it."""
    import importlib.util
    import shutil

    if shutil.which("nvcc") is None:
        return
    path = os.path.join(ROOT, "mixture_experts_ffn_11_b200", "build.py")
    spec = importlib.util.spec_from_file_location("_moe_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


_build_native()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a); runs the CUDA path through the C-ABI")
