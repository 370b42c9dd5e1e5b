import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line(
        "markers", "gpu: needs a B200 (sm_100a) and the built libssq.so")


def pytest_collection_modifyitems(config, items):
    # GPU tests are opt-in by marker; when no GPU is visible they fail loudly
    # inside the test rather than silently passing on a fallback.
    pass


@pytest.fixture(scope="session")
def oref():
    import oracle
    oracle.build()
    return oracle
