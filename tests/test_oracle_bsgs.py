"""Pins for the oracle's baby-step giant-step linear transform with double hoisting.

The transform computes sum_j rot_{G_j}( sum_k pt_{j,k} * rot_{B_k}(ct) ), with the baby
rotations kept in the extended basis PQ and the plaintext products summed there before one
ModDown per giant step.  Exact pins: ModDown(P c) = c and ModDown(P a + acc) = a + ModDown(acc)
hold bit for bit, so a transform whose only non-zero plaintext is the constant 1 at (j, k)
must equal the hoisted rotation by B_k followed by the single rotation by G_j, and the identity
diagonal must return the input.  Decoding pins check the slot meaning against numpy.
"""
import numpy as np
import pytest

import workloads as W
from oracle import encode
from oracle.scenario import Scenario


def _ext_limbs(ctx, level):
    return list(range(level + 1)) + list(range(ctx.n_q, ctx.n_q + ctx.n_p))


def _ones(ctx, level, n_giant, n_baby, at):
    """Plaintexts [n_giant][n_baby][ext][N]: the constant 1 at the positions in `at`, else 0."""
    ext = level + 1 + ctx.n_p
    pt = np.zeros((n_giant, n_baby, ext, ctx.n), dtype=np.uint32)
    for j, k in at:
        pt[j, k] = 1                      # the constant polynomial 1 is 1 at every evaluation point
    return pt


@pytest.fixture(scope="module")
def sc1b():
    return Scenario(W.CONFIGS["n12-dnum4"])


def _keys(sc, gs):
    return [None if g == 1 else (sc.key(g), g) for g in gs]


def test_bsgs_identity(sc1b):
    sc, ctx, lvl = sc1b, sc1b.ctx, sc1b.level
    _, ct = sc.ciphertext(0)
    baby = [1, sc.galois(1)]
    giant = [1]
    out = ctx.bsgs(ct, lvl, sc.alpha, baby, _keys(sc, baby), giant, _keys(sc, giant),
                   _ones(ctx, lvl, 1, 2, [(0, 0)]), sc.seed_bytes)
    assert np.array_equal(out, ct)


@pytest.mark.parametrize("j,k", [(0, 1), (1, 2), (1, 0)])
def test_bsgs_single_diagonal_is_rotation(sc1b, j, k):
    sc, ctx, lvl = sc1b, sc1b.ctx, sc1b.level
    _, ct = sc.ciphertext(0)
    baby = [1, sc.galois(1), sc.galois(2)]
    giant = [1, sc.galois(3)]
    out = ctx.bsgs(ct, lvl, sc.alpha, baby, _keys(sc, baby), giant, _keys(sc, giant),
                   _ones(ctx, lvl, 2, 3, [(j, k)]), sc.seed_bytes)
    want = ct
    if baby[k] != 1:
        want = ctx.rotate_hoisted(ct, lvl, sc.alpha, [baby[k]], [sc.key(baby[k])], [sc.seed_bytes], [baby[k]])[0]
    if giant[j] != 1:
        want = ctx.rotate(want, lvl, sc.alpha, giant[j], sc.key(giant[j]), sc.seed_bytes, giant[j])
    assert np.array_equal(out, want)


def test_bsgs_decode():
    """A 12-diagonal transform (baby 0..3, giant 0, 4, 8) on n14-hoisted8 decodes to
    sum_i d_i * rot_i(z); the plaintexts are the diagonals pre-rotated by -G_j."""
    sc = Scenario(W.CONFIGS["n14-hoisted8"])
    ctx, lvl, n = sc.ctx, sc.level, sc.n
    z, ct = sc.ciphertext(0)
    n1, n2 = 4, 3
    baby = [sc.galois(k) if k else 1 for k in range(n1)]
    giant = [sc.galois(n1 * j) if j else 1 for j in range(n2)]
    rng = np.random.default_rng(7)
    d = rng.uniform(-1, 1, (n1 * n2, n // 2)) + 1j * rng.uniform(-1, 1, (n1 * n2, n // 2))
    scale_p = 2.0 ** 20
    limbs = _ext_limbs(ctx, lvl)
    pt = np.empty((n2, n1, len(limbs), n), dtype=np.uint32)
    for j in range(n2):
        for k in range(n1):
            m = encode(np.roll(d[n1 * j + k], n1 * j), n, scale_p)
            pt[j, k] = ctx.signed_to_eval(m, limbs)
    out = ctx.bsgs(ct, lvl, sc.alpha, baby, _keys(sc, baby), giant, _keys(sc, giant), pt, sc.seed_bytes)
    want = sum(d[i] * np.roll(z, -i) for i in range(n1 * n2))
    err = np.abs(sc.decrypt_slots(out, scale=sc.scale * scale_p) - want).max()
    # each of the 12 terms carries one rotation's key-switching noise (max about 2^-10.3 at
    # n14-hoisted8); their sum stays below 2^-7.5, while a misplaced diagonal errs by order 1
    assert err < 2.0 ** -7.5
    # the same plaintexts without the -G_j pre-rotation give a different transform
    assert np.abs(sc.decrypt_slots(out, scale=sc.scale * scale_p)
                  - sum(d[i] * np.roll(z, -i) for i in range(n1))).max() > 0.1
