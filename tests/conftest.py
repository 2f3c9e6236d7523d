import importlib.util
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 and the built CUDA library")


def pytest_sessionstart(session):
    """Build the CUDA library (nvcc, no GPU needed) before any test module is
    imported: several modules import the package, which refuses to load
    without it. A no-op when the library is up to date."""
    spec = importlib.util.spec_from_file_location(
        "exact_attn_cuda_build", os.path.join(ROOT, "exact_io_aware_70_b200", "build.py"))
    build = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(build)
    build.build()
