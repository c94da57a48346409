import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")
    # the library is a build artefact (not in version control): build it once
    # when a fresh checkout runs the tests before anything else did (nvcc
    # cross-compiles without a GPU)
    lib_path = os.path.join(ROOT, "eagle_tree_verification_dynamic_b200", "libeagle_tree.so")
    if not os.path.exists(lib_path):
        from eagle_tree_verification_dynamic_b200 import build
        build.build()


@pytest.fixture(scope="session")
def golden_dir():
    return GOLDEN
