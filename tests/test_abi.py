"""The C-ABI library loads and exports every entry point its header declares; host-only logic
(prime chain rule, argument checks that run before any CUDA call) works without a GPU."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "ckks_ks.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(ckks_[a-z0-9_]+)\s*\(", src)))


def test_header_symbols_exported(ks_lib):
    lib = ctypes.CDLL(ks_lib.LIB_PATH)
    names = _declared()
    assert len(names) >= 18
    for name in names:
        assert hasattr(lib, name), name
    assert set(names) == set(ks_lib.EXPORTED)


def test_debug_build_exports_the_same_symbols(ks_lib):
    """The debug-bounds build exports the header's entry points too and says which build it is;
    neither question needs a GPU."""
    from conftest import build_library
    lib = ctypes.CDLL(build_library(debug=True))
    for name in _declared():
        assert hasattr(lib, name), name
    rel = ctypes.CDLL(os.path.join(os.path.dirname(ks_lib.LIB_PATH), "libckks_ks.so"))
    assert lib.ckks_debug_bounds_enabled() == 1 and rel.ckks_debug_bounds_enabled() == 0
    for l in (lib, rel):
        l.ckks_debug_bounds_site_name.restype = ctypes.c_char_p
        assert l.ckks_debug_bounds_site_name(1) == b"selftest"
        assert l.ckks_debug_bounds_site_name(10 ** 6) == b"unknown"
    count = ctypes.c_uint64()
    rel.ckks_debug_bounds_report.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int]
    assert rel.ckks_debug_bounds_report(ctypes.byref(count), None, None, None, 1) == ks_lib.CKKS_ERR_UNSUPPORTED
    lib.ckks_debug_bounds_report.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int]
    assert lib.ckks_debug_bounds_report(None, None, None, None, 1) == ks_lib.CKKS_ERR_ARG


@pytest.mark.parametrize("log_n,n_q,n_p", [(12, 4, 1), (14, 12, 4), (16, 36, 12), (13, 3, 2), (15, 5, 5)])
def test_gen_primes_matches_oracle(ks_lib, oracle_mod, log_n, n_q, n_p):
    q, p = ks_lib.ckks_gen_primes(log_n, n_q, n_p)
    oq, op = oracle_mod.chain(log_n, n_q, n_p)
    assert q == oq and p == op


def test_host_argument_errors(ks_lib):
    q, p = ks_lib.ckks_gen_primes(12, 4, 1)
    with pytest.raises(ks_lib.CkksError) as e:
        ks_lib.Context(11, q, p, 2)
    assert e.value.code == ks_lib.CKKS_ERR_UNSUPPORTED
    with pytest.raises(ks_lib.CkksError) as e:
        ks_lib.Context(12, [q[0] + 2] + q[1:], p, 2)        # not a prime = 1 mod 2N
    assert e.value.code == ks_lib.CKKS_ERR_UNSUPPORTED
    with pytest.raises(ks_lib.CkksError) as e:
        ks_lib.Context(12, q, p, 0)
    assert e.value.code == ks_lib.CKKS_ERR_UNSUPPORTED
    with pytest.raises(ks_lib.CkksError) as e:
        ks_lib.Context(12, [q[0], q[0]] + q[2:], p, 2)      # repeated modulus
    assert e.value.code == ks_lib.CKKS_ERR_UNSUPPORTED
    lib = ctypes.CDLL(ks_lib.LIB_PATH)
    lib.ckks_gen_primes.argtypes = [ctypes.c_uint32] * 3 + [ctypes.c_void_p] * 2
    assert lib.ckks_gen_primes(12, 2, 1, None, None) == ks_lib.CKKS_ERR_ARG
    assert ks_lib.galois_element(16, -1) == pow(5, 2**15 - 1, 2**17)
