"""Pins for the automorphism kappa_g: polynomial substitution by brute force, commutation
with the NTT, composition, the Galois elements of rotations, and slot rotation on decode."""
import numpy as np
import pytest


@pytest.mark.parametrize("log_n", [3, 6])
def test_coef_brute_force(oracle_mod, log_n):
    n = 1 << log_n
    ctx = oracle_mod.Ctx(log_n, 2, 1)
    q = ctx.mod[0]
    a = np.random.default_rng(1).integers(0, q, n, dtype=np.uint64).astype(np.uint32)
    for g in [1, 3, 5, 2 * n - 1, 25 % (2 * n)]:
        got = ctx.automorph_coef(a, 0, g)
        want = [0] * n
        for i in range(n):          # a(X^g) mod X^N + 1, term by term
            e = i * g
            sign = -1 if (e // n) % 2 else 1
            want[e % n] += sign * int(a[i])
        assert got.tolist() == [w % q for w in want]


@pytest.mark.parametrize("log_n", [4, 12, 16])
def test_eval_commutes_with_ntt(oracle_mod, log_n):
    n = 1 << log_n
    ctx = oracle_mod.Ctx(log_n, 2, 1)
    rng = np.random.default_rng(4)
    for t in range(2):
        q = ctx.mod[t]
        a = rng.integers(0, q, n, dtype=np.uint64).astype(np.uint32)
        for g in [5, 25, oracle_mod.galois_elt(log_n, -1), 2 * n - 1, 3]:
            lhs = ctx.ntt_fwd(ctx.automorph_coef(a, t, g), t)
            rhs = ctx.automorph_eval(ctx.ntt_fwd(a, t), g)
            assert np.array_equal(lhs, rhs)


def test_composition(oracle_mod):
    log_n = 10
    n = 1 << log_n
    ctx = oracle_mod.Ctx(log_n, 1, 1)
    a = np.random.default_rng(0).integers(0, ctx.mod[0], n, dtype=np.uint64).astype(np.uint32)
    for g, h in [(5, 25), (3, 2 * n - 1), (125, 7)]:
        lhs = ctx.automorph_eval(ctx.automorph_eval(a, h), g)
        assert np.array_equal(lhs, ctx.automorph_eval(a, (g * h) % (2 * n)))
    assert np.array_equal(ctx.automorph_eval(a, 1), a)


@pytest.mark.parametrize("log_n", [12, 14, 16])
def test_galois_elements(oracle_mod, log_n):
    n = 1 << log_n
    for r in [0, 1, 2, 8, 16, 272, n // 2 - 1, -1, -8]:
        assert oracle_mod.galois_elt(log_n, r) == pow(5, r % (n // 2), 2 * n)
    assert pow(5, n // 2, 2 * n) == 1


def test_rotation_on_slots(oracle_mod):
    """kappa_{5^r} on an encoded plaintext moves slot j+r to slot j (a left rotation)."""
    log_n = 8
    n = 1 << log_n
    ctx = oracle_mod.Ctx(log_n, 3, 1)
    rng = np.random.default_rng(8)
    z = rng.uniform(-1, 1, n // 2) + 1j * rng.uniform(-1, 1, n // 2)
    scale = 2.0 ** 30
    m = oracle_mod.encode(z, n, scale)
    for r in [1, 3, -2]:
        g = oracle_mod.galois_elt(log_n, r)
        res = np.stack([np.array([int(x) % q for x in m], dtype=np.uint32) for q in ctx.q])
        rot = np.stack([ctx.automorph_coef(res[t], t, g) for t in range(3)])
        mm = ctx.crt_centered(rot, range(3))
        zr = oracle_mod.decode(mm, n, scale)
        assert np.abs(zr - np.roll(z, -r)).max() < 1e-6
