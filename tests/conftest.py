import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_sessionstart(session):
    # a fresh checkout has no libdqgemm.so (built files are not versioned):
    # build it once, in-tree, so the ABI tests have a library to load (nvcc
    # cross-compiles for sm_100a without a GPU)
    from weight_only_quantized_prologue_b200 import build

    if not os.path.exists(build.LIB):
        build.build()


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")
