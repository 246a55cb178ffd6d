import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def pytest_collection_modifyitems(config, items):
    # Tests that need the GPU are marked explicitly; nothing is auto-skipped, so a GPU test run
    # on a box without a GPU fails loudly instead of passing vacuously.
    pass


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.lib()
    return oracle
