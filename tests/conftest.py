import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


@pytest.fixture(scope="session", autouse=True)
def _oracle_threads():
    """The oracle's parallel loops use every processor (results are
    bit-identical for any thread count)."""
    import oracle
    oracle.set_threads(oracle.max_threads())
    yield
