import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running; opt-in via ZERO_SLOW=1")
    # a fresh checkout has no built library yet: build it (nvcc cross-compiles
    # for sm_100a without a GPU) before any test module imports the package
    lib = os.path.join(ROOT, "zero_partitioned_mixed_reduce_b200", "libzero_b200.so")
    if not os.path.exists(lib) and not os.environ.get("ZERO_B200_LIB"):
        import __graft_entry__
        __graft_entry__.build()


def pytest_collection_modifyitems(config, items):
    if os.environ.get("ZERO_SLOW") == "1":
        return
    skip = pytest.mark.skip(reason="slow test; set ZERO_SLOW=1 to run")
    for item in items:
        if "slow" in item.keywords:
            item.add_marker(skip)


@pytest.fixture(scope="session")
def golden_dir():
    return os.path.join(ROOT, "tests", "golden")
