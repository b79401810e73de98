import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _build_library_if_stale():
    # loaded by path: importing the package would load the library itself
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "hq_build", os.path.join(ROOT, "fp8_dynamic_quantization_amax_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")
    _build_library_if_stale()
