import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (sm_100a) and the built CUDA library")


def pytest_collection_modifyitems(config, items):
    # GPU tests fail loudly (not skip) when the device is missing but a GPU run was asked for;
    # in a CPU-only run they are deselected with -m "not gpu".
    pass


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.build()
    return oracle
