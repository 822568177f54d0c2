import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: oracle work at N=2^16 (seconds)")


def build_library(debug=None):
    """Builds the CUDA library in-tree (nvcc cross-compiles for sm_100a without a GPU): the build the
    package loads (FHE_KS_B200_BUILD), or the one `debug` names.  The build script is loaded by
    path, since importing the package needs the built library."""
    import importlib.util
    spec = importlib.util.spec_from_file_location(
        "_ckks_ks_build", os.path.join(ROOT, "fhe_key_switching_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    if debug is None:
        debug = os.environ.get("FHE_KS_B200_BUILD", "release") == "debug"
    return mod.build(debug=debug)


@pytest.fixture(scope="session")
def ks_lib():
    """The CUDA library, built in-tree."""
    build_library()
    import fhe_key_switching_b200 as ks
    return ks


@pytest.fixture(autouse=True)
def _debug_bounds_clean(request):
    """Under the debug-bounds build, a GPU test fails when any kernel's index check failed during it."""
    yield
    ks = sys.modules.get("fhe_key_switching_b200")
    if ks is None or ks.BUILD != "debug" or request.node.get_closest_marker("gpu") is None:
        return
    count, site, addr, nbytes = ks.ckks_debug_bounds_report(clear=True)
    assert count == 0, f"{count} failed index checks; the first at {site}: {nbytes} bytes at {addr:#x}"


@pytest.fixture(scope="session")
def oracle_mod():
    import oracle
    oracle.lib()
    return oracle
