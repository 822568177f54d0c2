import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: oracle work at N=2^16 (seconds)")


@pytest.fixture(scope="session")
def ks_lib():
    """The CUDA library, built in-tree (nvcc cross-compiles for sm_100a without a GPU)."""
    from fhe_key_switching_b200 import build as _build
    _build.build()
    import fhe_key_switching_b200 as ks
    return ks


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.lib()
    return oracle
