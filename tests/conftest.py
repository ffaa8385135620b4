import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))
for p in (ROOT, HERE):
    if p not in sys.path:
        sys.path.insert(0, p)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the CUDA library")
    config.addinivalue_line("markers", "slow: full-size workloads (minutes)")


def ensure_library_built():
    """Build libdg.so if it is missing or older than its sources (loads the
    build script by path: importing the package needs the built library)."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "dg_build", os.path.join(ROOT, "moe_grouped_gemm_09_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
