import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def load_build_module():
    """extreme_bit_weight_b200/build.py, loaded by its path: importing the package itself needs the
    library to be built already (and current)."""
    import importlib.util

    spec = importlib.util.spec_from_file_location("_ccq_build", os.path.join(ROOT, "extreme_bit_weight_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.fixture(scope="session")
def built_lib():
    """Builds libccq.so if any source is newer than it; returns its path."""
    return load_build_module().build()


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


@pytest.fixture(scope="session")
def golden():
    import json

    def load(name):
        with open(os.path.join(ROOT, "tests", "golden", name)) as f:
            return json.load(f)

    return load
