"""The debug-bounds build (the same sources compiled with -DCKKS_DEBUG_BOUNDS): every kernel checks
each group of global-memory accesses against the running call's buffers and the context's tables,
and shared memory is poisoned at kernel start.

- In the release build the debug entry points answer CKKS_ERR_UNSUPPORTED.
- In the debug build a check that fails (the self-test's, which makes no access) is recorded with its
  site and size, reported by ckks_sync_status as CKKS_ERR_BOUNDS, and cleared.
- The GPU parity suite (every non-slow GPU test, this file included) runs again in a child process
  on the debug build: every output must still equal the oracle's, and conftest fails any test
  during which an index check failed."""
import glob
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _ctx(ks):
    q, p = ks.ckks_gen_primes(12, 4, 1)
    return ks.Context(12, q, p, 2)


def test_release_build_has_no_checks(ks_lib):
    ks = ks_lib
    if ks.BUILD == "debug":
        pytest.skip("release-build behaviour")
    assert not ks.ckks_debug_bounds_enabled()
    ctx = _ctx(ks)
    for call in (lambda: ks.ckks_selftest_bounds(ctx), lambda: ks.ckks_debug_bounds_report()):
        with pytest.raises(ks.CkksError) as e:
            call()
        assert e.value.code == ks.CKKS_ERR_UNSUPPORTED


def test_selftest_is_recorded_and_reported(ks_lib):
    ks = ks_lib
    if ks.BUILD != "debug":
        pytest.skip("runs in the debug-bounds child process of test_gpu_suite_under_debug_bounds")
    assert ks.ckks_debug_bounds_enabled()
    ctx = _ctx(ks)
    ks.ckks_debug_bounds_report(clear=True)
    ks.ckks_selftest_bounds(ctx)
    count, site, addr, nbytes = ks.ckks_debug_bounds_report(clear=True)
    assert (count, site, nbytes) == (1, "selftest", 4) and addr % 256 == 4
    assert ks.ckks_debug_bounds_report(clear=True)[0] == 0
    ks.ckks_selftest_bounds(ctx)
    assert ks.ckks_sync_status(ctx, None, 10000) == ks.CKKS_ERR_BOUNDS
    assert ks.ckks_sync_status(ctx, None, 10000) == ks.CKKS_OK          # the record was cleared
    assert ks.ckks_debug_bounds_report(clear=True)[0] == 0


def test_gpu_suite_under_debug_bounds(ks_lib):
    """Every non-slow GPU test again, on the debug-bounds build, in a child process."""
    if ks_lib.BUILD == "debug":
        pytest.skip("already the debug-bounds build")
    from conftest import build_library
    build_library(debug=True)
    files = sorted(glob.glob(os.path.join(ROOT, "tests", "test_gpu_*.py")))
    files.append(os.path.join(ROOT, "tests", "test_zz_no_alloc.py"))
    env = dict(os.environ, FHE_KS_B200_BUILD="debug")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-rs", "-m", "gpu and not slow", "-p",
                        "no:cacheprovider", *files], cwd=ROOT, env=env, capture_output=True, text=True, timeout=3000)
    tail = r.stdout[-6000:] + "\n" + r.stderr[-3000:]
    assert r.returncode == 0, tail
    # the debug-only self-test ran there (its skip reason would be listed under -rs otherwise)
    assert " passed" in r.stdout and "debug-bounds child process" not in r.stdout, tail
