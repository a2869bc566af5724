import json
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (a B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running case")


def build_cuda_lib():
    """Compile libmoe_route.so if stale.  build.py is loaded by path: importing
    the package itself needs the library to exist already."""
    import importlib.util
    path = os.path.join(ROOT, "combine_moe_route_08_b200", "build.py")
    spec = importlib.util.spec_from_file_location("moe_route_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


def load_golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle
