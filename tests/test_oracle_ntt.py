"""Pins for the oracle's negacyclic NTT: the O(N^2) definition, negacyclic convolution,
the closed form for monomials at N=2^16, and inverse o forward = identity."""
import numpy as np
import pytest


def brv(x, bits):
    return int(format(x, f"0{bits}b")[::-1], 2) if bits else 0


@pytest.mark.parametrize("log_n", [1, 2, 3, 5, 7])
def test_definition_small(oracle_mod, log_n):
    n = 1 << log_n
    ctx = oracle_mod.Ctx(log_n, 3, 1)
    rng = np.random.default_rng(log_n)
    for t in range(4):
        q, psi = ctx.mod[t], ctx.psi(t)
        a = rng.integers(0, q, n, dtype=np.uint64).astype(np.uint32)
        got = ctx.ntt_fwd(a, first_limb=t)
        want = [sum(int(a[i]) * pow(psi, (2 * brv(k, log_n) + 1) * i, q) for i in range(n)) % q
                for k in range(n)]
        assert got.tolist() == want


@pytest.mark.parametrize("log_n", [4, 6, 8])
def test_negacyclic_convolution(oracle_mod, log_n):
    """iNTT(NTT(a) * NTT(b)) = a*b mod (X^N + 1): independent of the storage order."""
    n = 1 << log_n
    ctx = oracle_mod.Ctx(log_n, 2, 1)
    rng = np.random.default_rng(11)
    for t in range(3):
        q = ctx.mod[t]
        a = rng.integers(0, q, n, dtype=np.uint64)
        b = rng.integers(0, q, n, dtype=np.uint64)
        fa = ctx.ntt_fwd(a.astype(np.uint32), t).astype(np.uint64)
        fb = ctx.ntt_fwd(b.astype(np.uint32), t).astype(np.uint64)
        got = ctx.ntt_inv(((fa * fb) % q).astype(np.uint32), t)
        want = [0] * n
        al, bl = a.tolist(), b.tolist()
        for i in range(n):
            for j in range(n):
                k = i + j
                if k < n:
                    want[k] += al[i] * bl[j]
                else:
                    want[k - n] -= al[i] * bl[j]
        assert got.tolist() == [w % q for w in want]


def test_monomials_n65536(oracle_mod):
    log_n = 16
    n = 1 << log_n
    ctx = oracle_mod.Ctx(log_n, 2, 1)
    rng = np.random.default_rng(5)
    for t in range(3):
        q, psi = ctx.mod[t], ctx.psi(t)
        for i in [0, 1, 2, 777, n - 1]:
            a = np.zeros(n, dtype=np.uint32)
            a[i] = 1
            got = ctx.ntt_fwd(a, t)
            for k in rng.integers(0, n, 12):
                k = int(k)
                assert int(got[k]) == pow(psi, (2 * brv(k, log_n) + 1) * i, q)


def test_definition_sampled_n65536(oracle_mod):
    """Random input at N=2^16: selected outputs evaluated straight from the definition."""
    log_n = 16
    n = 1 << log_n
    ctx = oracle_mod.Ctx(log_n, 1, 1)
    q, psi = ctx.mod[0], ctx.psi(0)
    a = np.random.default_rng(9).integers(0, q, n, dtype=np.uint64)
    got = ctx.ntt_fwd(a.astype(np.uint32), 0)
    al = a.tolist()
    for k in [0, 1, 12345, n - 1]:
        w = pow(psi, 2 * brv(k, log_n) + 1, q)
        acc, pw = 0, 1
        for x in al:
            acc = (acc + x * pw) % q
            pw = pw * w % q
        assert int(got[k]) == acc


@pytest.mark.parametrize("log_n", [12, 14, 16])
def test_roundtrip(oracle_mod, log_n):
    n = 1 << log_n
    ctx = oracle_mod.Ctx(log_n, 3, 1)
    rng = np.random.default_rng(2)
    a = np.stack([rng.integers(0, q, n, dtype=np.uint64) for q in ctx.mod]).astype(np.uint32)
    f = ctx.ntt_fwd(a, 0)
    assert not np.array_equal(f, a)
    assert np.array_equal(ctx.ntt_inv(f, 0), a)
    assert np.array_equal(ctx.ntt_fwd(ctx.ntt_inv(a, 0), 0), a)
