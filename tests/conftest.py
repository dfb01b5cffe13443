import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA B200 (sm_100a) device")


def pytest_collection_modifyitems(config, items):
    # GPU tests fail loudly when the device or library is missing; nothing is skipped silently.
    pass


@pytest.fixture(scope="session")
def root_dir():
    return ROOT
