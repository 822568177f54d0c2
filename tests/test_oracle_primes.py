"""Pins for the prime chain rule and the choice of psi (checked with sympy and pow)."""
import pytest
import sympy


@pytest.mark.parametrize("log_n,count", [(12, 5), (14, 16), (16, 48), (5, 10)])
def test_prime_scan(oracle_mod, log_n, count):
    pr = oracle_mod.gen_primes(log_n, count)
    two_n = 2 << log_n
    assert len(pr) == count
    assert all(p < 2**30 and p % two_n == 1 and sympy.isprime(p) for p in pr)
    assert pr == sorted(pr, reverse=True)
    # nothing skipped: every x = 1 mod 2N from the top down to the last prime is listed or composite
    x = (1 << 30) - two_n + 1
    listed = set(pr)
    while x >= pr[-1]:
        assert (x in listed) == sympy.isprime(x)
        x -= two_n


def test_is_prime(oracle_mod):
    import random
    rnd = random.Random(3)
    xs = [0, 1, 2, 3, 4, 9, 25, 2**30 - 35, 65537, 2**31 - 1] + [rnd.randrange(2**30) for _ in range(300)]
    for x in xs:
        assert oracle_mod.is_prime(x) == sympy.isprime(x), x


@pytest.mark.parametrize("log_n", [3, 12, 14, 16])
def test_psi_rule(oracle_mod, log_n):
    n = 1 << log_n
    for q in oracle_mod.gen_primes(log_n, 6):
        psi = oracle_mod.find_psi(q, log_n)
        assert pow(psi, n, q) == q - 1 and pow(psi, 2 * n, q) == 1
        e = (q - 1) // (2 * n)
        h = next(h for h in range(2, q) if pow(h, e, q) == psi)
        # smallest h whose power is a primitive 2N-th root
        for h2 in range(2, h):
            assert pow(pow(h2, e, q), n, q) != q - 1
