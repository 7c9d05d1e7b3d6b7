import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built libgdn.so")


def pytest_collection_modifyitems(config, items):
    # GPU tests are selected with -m gpu; without a device they fail loudly rather than
    # silently passing, so only skip them when the run did not ask for them.
    pass


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle

    oracle.build()
    return oracle
