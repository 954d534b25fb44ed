import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) GPU; calls the CUDA path through the C ABI")
    config.addinivalue_line("markers", "slow: takes more than a few seconds on the CPU")


@pytest.fixture(scope="session")
def oracle_lib():
    """Build (if stale) and return the oracle package."""
    import oracle
    oracle._load()
    return oracle


@pytest.fixture(scope="session")
def gdn_lib():
    """Build the CUDA library if its sources are newer (nvcc cross-compiles
    without a GPU) and load it through the binding."""
    from gated_deltanet_recurrent_sigmoid_b200 import binding, build
    build.build()
    return binding.load()
