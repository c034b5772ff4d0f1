import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")
    config.addinivalue_line("markers", "slow: full-size workload checks")


@pytest.fixture(scope="session")
def ora():
    import oracle
    oracle.build()
    return oracle


@pytest.fixture(scope="session")
def bl():
    """The CUDA path through its C-ABI binding; fails loudly when it cannot load."""
    import torch
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    import bit_ternary_qat_b200 as pkg
    lib = pkg.load()
    return pkg
