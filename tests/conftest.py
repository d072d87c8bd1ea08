import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity case (minutes of CPU oracle time)")


def pytest_collection_modifyitems(config, items):
    # A gpu-marked test on a machine without CUDA is a failure of the run, not
    # a skip: the product path has no CPU fallback.
    pass


@pytest.fixture(scope="session")
def golden_dir():
    return GOLDEN
