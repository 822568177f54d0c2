"""Pins for the CKKS encoding: direct O(N^2) evaluation at the slot roots and round trip."""
import numpy as np
import pytest


@pytest.mark.parametrize("log_n", [2, 4, 7])
def test_encode_direct(oracle_mod, log_n):
    n = 1 << log_n
    rng = np.random.default_rng(log_n)
    z = rng.uniform(-1, 1, n // 2) + 1j * rng.uniform(-1, 1, n // 2)
    scale = 2.0 ** 40
    m = oracle_mod.encode(z, n, scale)
    zeta = np.exp(1j * np.pi / n)
    for j in range(n // 2):
        x = zeta ** pow(5, j, 2 * n)
        val = sum(float(m[i]) * x ** i for i in range(n))
        assert abs(val / scale - z[j]) < 1e-9
        xc = zeta ** (2 * n - pow(5, j, 2 * n))       # conjugate slot
        valc = sum(float(m[i]) * xc ** i for i in range(n))
        assert abs(valc / scale - np.conj(z[j])) < 1e-9


@pytest.mark.parametrize("log_n", [12, 16])
def test_roundtrip(oracle_mod, log_n):
    n = 1 << log_n
    rng = np.random.default_rng(3)
    z = rng.uniform(-1, 1, n // 2) + 1j * rng.uniform(-1, 1, n // 2)
    scale = 2.0 ** 28
    m = oracle_mod.encode(z, n, scale)
    assert m.dtype == np.int64
    # rounding error of each coefficient <= 1/2 -> slot error <= N/2 / scale
    assert np.abs(oracle_mod.decode(m, n, scale) - z).max() < n / 2 / scale
