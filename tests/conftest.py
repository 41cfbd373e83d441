import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_sessionstart(session):
    # build (or rebuild after a source edit) libdqgemm.so in-tree so the tests
    # load the library of the sources they test; build() returns at once when
    # the library is newer than every source.  nvcc cross-compiles for sm_100a
    # without a GPU; without nvcc the oracle-only tests still run.
    import shutil
    import warnings

    from weight_only_quantized_prologue_b200 import build

    if shutil.which(build.nvcc()) is None and not os.path.exists(build.nvcc()):
        warnings.warn("nvcc not found: libdqgemm.so is not (re)built; the ABI tests use whatever library exists")
        return
    build.build()


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")
