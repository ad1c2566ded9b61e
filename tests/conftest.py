import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    # a GPU test on a machine without a GPU is an error, not a skip, unless the
    # run deselected it with -m "not gpu"
    pass


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle
