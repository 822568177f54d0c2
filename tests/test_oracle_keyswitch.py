"""Pins for key generation, key switching, rotation (single and hoisted), relinearisation and
the tensor product: decryption identities and decoding against the plaintext slot operations.

Decoding tolerances come from the key-switching noise model
  std(slot error) ~ sqrt(N) * sqrt(N) * sigma * sqrt(beta) * (D_j / P) / Delta,
which gives max errors of about 2^-10 at n12-dnum4 and n14-hoisted8 and about 2^-8 at N=2^16
(n16-full);
a wrong sign, term or index anywhere in the pipeline gives errors of order 1 or larger.
"""
import numpy as np
import pytest

import workloads as W
from oracle.scenario import Scenario


def _noise(ctx, vals, level):
    """max |centred CRT lift| of a residue polynomial in the coefficient domain."""
    coef = ctx.crt_centered(ctx.ntt_inv(vals, 0), range(level + 1))
    return max(abs(v) for v in coef)


@pytest.fixture(scope="module")
def sc1b():
    return Scenario(W.CONFIGS["n12-dnum4"])


def test_keyswitch_identity(sc1b):
    """KS(c) = (u0, u1) with u0 + u1*s = c*s' + small, for s' = s^2 and s' = kappa_g(s)."""
    sc, ctx = sc1b, sc1b.ctx
    lvl, n = sc.level, sc.n
    rng = np.random.default_rng(1)
    c = np.stack([rng.integers(0, ctx.mod[t], n, dtype=np.uint64) for t in range(lvl + 1)]).astype(np.uint32)
    mods = np.array(ctx.q[: lvl + 1], dtype=np.uint64)[:, None]
    se = sc.s_eval[: lvl + 1].astype(np.uint64)
    for key_id in [0, sc.galois(1)]:
        b = sc.key(key_id)
        out = ctx.keyswitch(c, lvl, sc.alpha, b, sc.seed_bytes, key_id)
        s2 = (se * se) % mods if key_id == 0 else ctx.automorph_eval(sc.s_eval[: lvl + 1], key_id).astype(np.uint64)
        lhs = (out[0].astype(np.uint64) + out[1].astype(np.uint64) * se) % mods
        rhs = (c.astype(np.uint64) * s2) % mods
        diff = ((lhs + mods - rhs) % mods).astype(np.uint32)
        assert _noise(ctx, diff, lvl) < 2 ** 14
        # a wrong key (other seed) breaks it
        bad = ctx.keyswitch(c, lvl, sc.alpha, b, bytes(32), key_id)
        lhs = (bad[0].astype(np.uint64) + bad[1].astype(np.uint64) * se) % mods
        diff = ((lhs + mods - rhs) % mods).astype(np.uint32)
        assert _noise(ctx, diff, lvl) > 2 ** 60


def test_stored_a_equals_regenerated(sc1b):
    sc, ctx = sc1b, sc1b.ctx
    g = sc.galois(1)
    b, a = sc.key(g, want_a=True)
    for j in range(a.shape[0]):
        for t in range(a.shape[1]):
            assert np.array_equal(a[j, t], ctx.chacha_expand(sc.seed_bytes, g, j, t))
    z, ct = sc.ciphertext(0)
    o1 = ctx.rotate(ct, sc.level, sc.alpha, g, b, sc.seed_bytes, g)
    o2 = ctx.rotate(ct, sc.level, sc.alpha, g, b, bytes(32), g, a_stored=a)
    assert np.array_equal(o1, o2)


@pytest.mark.parametrize("key,tol", [("n12-dnum4", 2.0 ** -9.5), ("n14-hoisted8", 2.0 ** -9.5)])
def test_rotations_decode(key, tol):
    sc = Scenario(W.CONFIGS[key])
    z, ct = sc.ciphertext(0)
    for r in sc.cfg.rot_steps[:4]:
        g = sc.galois(r)
        out = sc.ctx.rotate(ct, sc.level, sc.alpha, g, sc.key(g), sc.seed_bytes, g)
        assert np.abs(sc.decrypt_slots(out) - np.roll(z, -r)).max() < tol


@pytest.mark.parametrize("key", ["n12-dnum4", "n14-hoisted8"])
def test_hoisted_decode_and_equals_single(key):
    """With centred fast base conversion, BConv(-x) = -BConv(x) coefficient-wise, and kappa_g
    only permutes coefficients with sign changes, so ModUp commutes with kappa_g: hoisted and
    single rotations give identical bits."""
    sc = Scenario(W.CONFIGS[key])
    ctx = sc.ctx
    z, ct = sc.ciphertext(0)
    steps = [1, -1, 3]
    gs = [sc.galois(r) for r in steps]
    keys = [sc.key(g) for g in gs]
    out = ctx.rotate_hoisted(ct, sc.level, sc.alpha, gs, keys, [sc.seed_bytes] * 3, gs)
    for i, r in enumerate(steps):
        assert np.abs(sc.decrypt_slots(out[i]) - np.roll(z, -r)).max() < 2.0 ** -9.5
        single = ctx.rotate(ct, sc.level, sc.alpha, gs[i], keys[i], sc.seed_bytes, gs[i])
        assert np.array_equal(single, out[i])


@pytest.mark.parametrize("key", ["n12-dnum4", "n14-hoisted8"])
def test_tensor_relin_decode(key):
    sc = Scenario(W.CONFIGS[key])
    z1, x = sc.ciphertext(0)
    z2, y = sc.ciphertext(1)
    d = sc.ctx.tensor(x, y, sc.level)
    zz = sc.decrypt_slots(d, scale=sc.scale ** 2)   # 3-component decryption
    assert np.abs(zz - z1 * z2).max() < 2.0 ** -12
    out = sc.ctx.relin(d, sc.level, sc.alpha, sc.key(0), sc.seed_bytes, 0)
    assert np.abs(sc.decrypt_slots(out, scale=sc.scale ** 2) - z1 * z2).max() < 2.0 ** -9.5


def test_n12_dnum2_noise_is_large():
    """n12-dnum2 (dnum=2, one special prime): P ~ 2^30 << D_j ~ 2^60, so the output is bit-exact
    material only; its decode error is far above 2^-10 (recorded, not a failure)."""
    sc = Scenario(W.CONFIGS["n12-dnum2"])
    z, ct = sc.ciphertext(0)
    g = sc.galois(1)
    out = sc.ctx.rotate(ct, sc.level, sc.alpha, g, sc.key(g), sc.seed_bytes, g)
    assert np.abs(sc.decrypt_slots(out) - np.roll(z, -1)).max() > 1.0


@pytest.mark.slow
def test_n16_full_rotation_relin_decode():
    sc = Scenario(W.CONFIGS["n16-full"])
    z1, x = sc.ciphertext(0)
    g = sc.galois(1)
    out = sc.ctx.rotate(x, sc.level, sc.alpha, g, sc.key(g), sc.seed_bytes, g)
    err = np.abs(sc.decrypt_slots(out) - np.roll(z1, -1))
    assert err.max() < 2.0 ** -6 and np.median(err) < 2.0 ** -10
