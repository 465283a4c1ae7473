import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    # Rebuild the CUDA library and the oracle if a source is newer than the build
    # (a no-op when they are current; nvcc cross-compiles without a GPU).
    import shutil
    if shutil.which("nvcc") or os.path.exists("/usr/local/cuda/bin/nvcc"):
        # load build.py by path: importing the package would load the stale library
        import importlib.util
        spec = importlib.util.spec_from_file_location(
            "_fp8q_build", os.path.join(ROOT, "fp8_quantized_linear_rms_b200", "build.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod.build()
    import oracle
    oracle.build()


@pytest.fixture(scope="session")
def golden():
    import json
    with open(os.path.join(ROOT, "tests", "golden", "closed_forms.json")) as f:
        return json.load(f)
