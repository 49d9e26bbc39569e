import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size parity cases (minutes)")


def pytest_collection_modifyitems(config, items):
    """GPU tests fail loudly when no GPU is present (they are deselected with -m "not gpu")."""
    return


@pytest.fixture(scope="session")
def orc():
    import oracle
    oracle.build()
    return oracle
