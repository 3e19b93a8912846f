"""pytest configuration: the `gpu` marker, and building the native libraries before tests import them."""
import importlib.util
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def load_build_module():
    """The package's build script, loaded by path (importing the package needs the built library)."""
    path = os.path.join(ROOT, "linear_attention_attn_b200", "build.py")
    spec = importlib.util.spec_from_file_location("la_b200_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    load_build_module().build()
