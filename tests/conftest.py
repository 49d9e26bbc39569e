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


@pytest.fixture(scope="session")
def sbg():
    """The CUDA library on a B200; fails loudly (no fallback) when either is missing."""
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device (deselect with -m 'not gpu')"
    major, minor = torch.cuda.get_device_capability()
    assert major == 10, f"libsixbit targets sm_100a (B200); found sm_{major}{minor}"
    from video_diffusion_mixed_b200 import build
    build.build()
    from video_diffusion_mixed_b200 import sixbit
    sixbit.lib()
    return sixbit
