import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (runs the sm_100a library)")


@pytest.fixture(scope="session")
def orc():
    """The float64 oracle (built with gcc on first use)."""
    from oracle import oracle
    oracle.build()
    return oracle
