import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU")


def pytest_collection_modifyitems(config, items):
    # A test marked gpu that runs where there is no GPU is an error, not a skip.
    pass


@pytest.fixture(scope="session")
def oracle_lib():
    import oracle
    return oracle.lib()
