import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")


def pytest_sessionstart(session):
    # (re)build the in-tree CUDA library when a source is newer than it; the
    # build script is loaded by path, since importing the package loads the library
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_lcl_build", os.path.join(ROOT, "long_context_linear_b200", "build.py"))
    b = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(b)
    b.build()


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle
