"""Pins for the oracle's rescale and conjugation.

Rescale (full-RNS CKKS, Cheon-Han-Kim-Kim-Song, SAC 2018): per component with integer
polynomial C over q_0..q_l, the result is (C - [C]_{q_l}) / q_l modulo q_0..q_{l-1}, with the
centred residue [C]_{q_l} in (-q_l/2, q_l/2].  The oracle computes it limb by limb through
NTTs; the pin below recomputes it from the composite integer C (Python integers, CRT), a
different route, so a wrong prime, a missing transform, an unsigned lift or a wrong inverse
fails it.  Decoding pins check the plaintext meaning: rescaling a product at scale Delta^2
gives the product at scale Delta^2 / q_l.

Conjugation is the automorphism kappa_g with g = 2N - 1 (X -> X^-1), which conjugates every
slot; its key-switching key has key_id g like any rotation key.
"""
import numpy as np
import pytest

import workloads as W
from oracle.scenario import Scenario


def _coef_ints(ctx, limbs, n_limbs):
    """Centred CRT integers of a residue polynomial (evaluation domain) over q_0..q_{n_limbs-1}."""
    coef = ctx.ntt_inv(np.ascontiguousarray(limbs[:n_limbs]), 0)
    return ctx.crt_centered(coef, range(n_limbs))


@pytest.fixture(scope="module")
def sc1b():
    return Scenario(W.CONFIGS["n12-dnum4"])


@pytest.mark.parametrize("level", [3, 2, 1])
def test_rescale_exact_division(sc1b, level):
    ctx, n = sc1b.ctx, sc1b.n
    rng = np.random.default_rng(100 + level)
    ct = np.stack([np.stack([rng.integers(0, ctx.mod[t], n, dtype=np.uint64) for t in range(level + 1)])
                   for _ in range(2)]).astype(np.uint32)
    out = ctx.rescale(ct, level)
    assert out.shape == (2, level, n)
    ql = ctx.mod[level]
    for comp in range(2):
        C = _coef_ints(ctx, ct[comp], level + 1)
        got = ctx.ntt_inv(np.ascontiguousarray(out[comp]), 0)
        for k in range(0, n, 7):                      # every 7th coefficient, all limbs
            r = C[k] % ql
            if r > (ql - 1) // 2:
                r -= ql
            e = (C[k] - r) // ql
            assert (C[k] - r) % ql == 0
            for i in range(level):
                assert int(got[i, k]) == e % ctx.mod[i], (comp, k, i)


def test_rescale_centred_not_unsigned(sc1b):
    """A coefficient whose residue mod q_l lies above q_l/2 rounds up, not down."""
    ctx, n, level = sc1b.ctx, sc1b.n, 2
    ql = ctx.mod[level]
    coef = np.zeros((level + 1, n), dtype=np.uint32)
    v = 5 * ql + (ql - 3)                              # = 6 q_l - 3: centred residue -3
    for t in range(level + 1):
        coef[t, 0] = v % ctx.mod[t]
    ev = ctx.ntt_fwd(coef, 0)
    out = ctx.rescale(ev[None], level)[0]
    got = ctx.ntt_inv(np.ascontiguousarray(out), 0)
    for i in range(level):
        assert int(got[i, 0]) == 6                     # (6 q_l - 3 - (-3)) / q_l
        assert not got[i, 1:].any()


@pytest.mark.parametrize("key,tol", [("n12-dnum4", 2.0 ** -9), ("n14-hoisted8", 2.0 ** -13)])
def test_tensor_relin_rescale_decode(key, tol):
    sc = Scenario(W.CONFIGS[key])
    ctx, lvl = sc.ctx, sc.level
    z1, x = sc.ciphertext(0)
    z2, y = sc.ciphertext(1)
    d = ctx.tensor(x, y, lvl)
    r = ctx.relin(d, lvl, sc.alpha, sc.key(0), sc.seed_bytes, 0)
    out = ctx.rescale(r, lvl)
    scale = sc.scale ** 2 / ctx.mod[lvl]
    err = np.abs(sc.decrypt_slots(out, level=lvl - 1, scale=scale) - z1 * z2).max()
    assert err < tol
    # decoding at the unrescaled scale is wrong by the factor q_l
    assert np.abs(sc.decrypt_slots(out, level=lvl - 1, scale=sc.scale ** 2) - z1 * z2).max() > 0.1


@pytest.mark.parametrize("key", ["n12-dnum4", "n14-hoisted8"])
def test_conjugation_decode(key):
    sc = Scenario(W.CONFIGS[key])
    g = 2 * sc.n - 1
    z, ct = sc.ciphertext(0)
    out = sc.ctx.rotate(ct, sc.level, sc.alpha, g, sc.key(g), sc.seed_bytes, g)
    assert np.abs(sc.decrypt_slots(out) - np.conj(z)).max() < 2.0 ** -9.5
    # conjugating twice is the identity on the slots
    out2 = sc.ctx.rotate(out, sc.level, sc.alpha, g, sc.key(g), sc.seed_bytes, g)
    assert np.abs(sc.decrypt_slots(out2) - z).max() < 2.0 ** -9
