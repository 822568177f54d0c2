"""Pins of the bootstrapping linear maps in oracle/bootstrap.py (CPU).

The special DFT V (z = V t, t_k = m_k + i m_(k+n)) is pinned against the oracle's CKKS decoding
of a plaintext polynomial, which is itself pinned by direct evaluation; its radix-2 stage
factorization against the explicit O(n^2) matrix; the inverse stages against V^-1; the levels,
their compositions and the baby-step giant-step plan against stage-by-stage application."""
import numpy as np
import pytest

import oracle
from oracle import bootstrap as bt


def _rand_c(n, seed):
    g = np.random.default_rng(seed)
    return g.uniform(-1, 1, n) + 1j * g.uniform(-1, 1, n)


@pytest.mark.parametrize("log_n", [3, 4, 6, 8])
def test_dft_matrix_is_decoding(log_n):
    """V t equals the decoding of the real polynomial with m_k = Re t_k, m_(k+n) = Im t_k."""
    n, ns = 1 << log_n, 1 << (log_n - 1)
    t = _rand_c(ns, log_n)
    m = np.concatenate([t.real, t.imag])
    z = oracle.decode(m, n, 1.0)
    assert np.allclose(bt.dft_matrix(log_n) @ t, z, atol=1e-9)


@pytest.mark.parametrize("log_n", [3, 5, 7, 9])
def test_stages_factor_the_dft(log_n):
    ns = 1 << (log_n - 1)
    t = _rand_c(ns, 10 + log_n)
    x = bt.bitrev(t)
    for length in bt.stage_lengths(log_n):
        x = bt.apply_diagonals(x, bt.stage_diagonals(log_n, length))
    assert np.allclose(x, bt.dft_matrix(log_n) @ t, atol=1e-9)


@pytest.mark.parametrize("log_n", [3, 5, 7])
def test_inverse_stages_invert(log_n):
    ns = 1 << (log_n - 1)
    z = _rand_c(ns, 20 + log_n)
    t = np.linalg.solve(bt.dft_matrix(log_n), z)
    assert np.allclose(bt.coeff_to_slot(z, log_n, 1), bt.bitrev(t), atol=1e-9)
    for length in bt.stage_lengths(log_n):
        d, di = bt.stage_diagonals(log_n, length), bt.stage_diagonals(log_n, length, inverse=True)
        assert np.allclose(bt.apply_diagonals(bt.apply_diagonals(z, d), di), z, atol=1e-12)


@pytest.mark.parametrize("log_n,levels", [(7, 2), (9, 3), (12, 3), (12, 4)])
def test_levels_equal_stages(log_n, levels):
    ns = 1 << (log_n - 1)
    z = _rand_c(ns, 30 + log_n)
    split = bt.split_levels(log_n, levels, True)
    assert sum(len(s) for s in split) == log_n - 1
    x = z
    for length in sorted(bt.stage_lengths(log_n), reverse=True):
        x = bt.apply_diagonals(x, bt.stage_diagonals(log_n, length, inverse=True))
    assert np.allclose(bt.coeff_to_slot(z, log_n, levels), x, atol=1e-9)
    y = bt.slot_to_coeff(x, log_n, levels)
    assert np.allclose(y, z, atol=1e-9)
    # a level of r stages has at most 2^(r+1) - 1 diagonals
    for lens in split:
        assert len(bt.level_diagonals(log_n, lens, True)) <= 2 ** (len(lens) + 1) - 1


@pytest.mark.parametrize("n1", [2, 4, 8])
def test_bsgs_plan_matches_diagonals(n1):
    log_n = 10
    ns = 1 << (log_n - 1)
    x = _rand_c(ns, 40 + n1)
    for lens in bt.split_levels(log_n, 3, False):
        d = bt.level_diagonals(log_n, lens, False)
        babies, giants, pt = bt.bsgs_plan(d, ns, n1)
        assert len(babies) == n1 and babies[0] == 0
        assert np.allclose(bt.apply_bsgs(x, babies, giants, pt), bt.apply_diagonals(x, d), atol=1e-9)


def test_modraise_crt_identity():
    """Every coefficient of the raised polynomial, CRT-reconstructed over q_0..q_L (Python
    integers), equals the centred lift of the level-0 coefficient; and the raised ciphertext
    decrypts to m + q_0 I with a small integer polynomial I."""
    import workloads as W
    from oracle.scenario import Scenario
    cfg = W.CONFIGS["n12-dnum4"]
    sc = Scenario(cfg)
    ctx = sc.ctx
    _, ct = sc.ciphertext(0, level=0)
    L = cfg.level
    up = bt.modraise(ctx, ct, L)
    q0 = ctx.q[0]
    for comp in range(2):
        coef0 = ctx.ntt_inv(ct[comp], 0)[0].astype(np.int64)
        want = np.where(coef0 > (q0 - 1) // 2, coef0 - q0, coef0)
        res = np.stack([ctx.ntt_inv(up[comp][i][None], i)[0] for i in range(L + 1)])
        got = ctx.crt_centered(res, range(L + 1))
        assert got == [int(x) for x in want]
    m0 = np.array(ctx.decrypt(ct, 0, sc.s_eval), dtype=object)
    m1 = np.array(ctx.decrypt(up, L, sc.s_eval), dtype=object)
    diff = m1 - m0
    assert all(d % q0 == 0 for d in diff)
    assert max(abs(d // q0) for d in diff) <= cfg.h // 2 + 2


@pytest.mark.parametrize("direction", ["coeff_to_slot", "slot_to_coeff"])
def test_homomorphic_levels_decode(direction):
    """The levels evaluated homomorphically on the oracle (encrypted slots, one baby-step
    giant-step transform and one rescale per level, diagonals encoded at scale q_level) decode
    to the numpy maps: CoeffToSlot(z) = bitrev(V^-1 z), SlotToCoeff(x) = V x for x given in
    bit-reversed order; at N=2^12, 4 + 1 primes, dnum 4 (the key-switching noise of this chain
    is below 2^-10 per slot).  CoeffToSlot's stages halve their inputs, so its error stays near
    the key-switching noise: max error below 2^-8.  SlotToCoeff's stages do not (V / sqrt(n) is
    unitary), so they amplify the earlier levels' noise up to sqrt(n) = 45 times: its error is
    pinned relative to the output, below 2^-9 of the largest slot (measured 8e-4).  A wrong
    twiddle, sign or shift gives errors of the order of the values themselves."""
    import workloads as W
    from oracle.scenario import Scenario
    cfg = W.CONFIGS["n12-dnum4"]
    sc = Scenario(cfg)
    ctx, log_n, ns = sc.ctx, cfg.log_n, cfg.n // 2
    levels, n1 = 3, 4
    inverse = direction == "coeff_to_slot"
    z, ct = sc.ciphertext(0)
    if not inverse:
        z = z / 4.0                    # V's entries have modulus 1: keep V z inside [-4, 4]
        ct = sc.encrypt_slots(z, 0)
    lvl = cfg.level
    keys = {}
    for lens in bt.split_levels(log_n, levels, inverse):
        babies, giants, pt = bt.bsgs_plan(bt.level_diagonals(log_n, lens, inverse), ns, n1)
        for s in babies + giants:
            g = bt.galois_of_shift(ctx, s)
            if g != 1 and g not in keys:
                keys[g] = sc.key(g)
        enc = bt.encode_plan(ctx, pt, lvl, float(ctx.q[lvl]))
        ct = bt.linear_level(ctx, ct, lvl, cfg.alpha, babies, giants, enc, keys, cfg.chacha_seed)
        lvl -= 1
    got = sc.decrypt_slots(ct, lvl)
    want = bt.coeff_to_slot(z, log_n, levels) if inverse else bt.slot_to_coeff(z, log_n, levels)
    err = np.max(np.abs(got - want))
    if inverse:
        assert err < 2.0 ** -8, err
    else:
        assert err < 2.0 ** -9 * np.max(np.abs(want)), (err, np.max(np.abs(want)))


def test_llround_is_half_away_from_zero():
    for x, want in [(2.5, 3), (-2.5, -3), (0.49999999999999994, 0), (-0.5, -1), (1e15 + 0.5, int(1e15) + 1),
                    (3.2, 3), (-3.7, -4), (0.0, 0)]:
        assert bt.llround(x) == want, x


@pytest.mark.slow
def test_evalmod_decodes_to_scaled_sine():
    """EvalMod (cosine Taylor polynomial of degree 12 in theta = 2 pi (x - 1/4) / 8, three double
    angles) on an encryption of real slots x in [-2, 2] at N=2^16, dnum 4, level 35, scale q_35,
    decodes to sin(2 pi x) / (2 pi): the polynomial itself is within 4.3e-8 of it; the measured
    error (CKKS noise of the input amplified up to 64 times by the double angles) has median
    1.9e-6 and maximum 1.1e-3 (2^-9.85) over the 32768 slots.  Pinned: median below 2^-17 and
    maximum below 2^-9; a wrong coefficient, sign or step gives errors of order 0.1."""
    import workloads as W
    from oracle.scenario import Scenario
    cfg = W.CONFIGS["n16-stream64"]
    sc = Scenario(cfg)
    ctx = sc.ctx
    L = 35
    S = float(ctx.q[L])
    x = np.random.default_rng(5).uniform(-2, 2, cfg.n // 2)
    m = oracle.encode(x.astype(complex), cfg.n, S)
    e = W.gaussian_error(cfg.n, cfg.sigma, W.rng(cfg.seed, W.TAG_ENC_ERR, 77))[0]
    a = W.uniform_residues(ctx.q[: L + 1], cfg.n, W.rng(cfg.seed, W.TAG_ENC_A, 77))
    ct = ctx.encrypt(sc.s, m, e, a, L)
    out, lv, so = bt.evalmod(ctx, ct, L, S, 3, 6, cfg.alpha, sc.key(0), cfg.chacha_seed)
    assert lv == L - (6 + 3 + 3)
    err = np.abs(sc.decrypt_slots(out, lv, so).real - np.sin(2 * np.pi * x) / (2 * np.pi))
    assert np.median(err) < 2.0 ** -17 and err.max() < 2.0 ** -9, (np.median(err), err.max())


def test_constant_ops_by_definition():
    """mul_const and add_const against the slot values they must produce (decoded), and the
    residue arithmetic against Python integers."""
    import workloads as W
    from oracle.scenario import Scenario
    cfg = W.CONFIGS["n12-dnum4"]
    sc = Scenario(cfg)
    ctx = sc.ctx
    z, ct = sc.ciphertext(0)
    lvl = cfg.level
    m3 = bt.mul_const(ctx, ct, lvl, -3)
    for i in range(lvl + 1):
        qi = ctx.q[i]
        assert int(m3[1, i, 5]) == (int(ct[1, i, 5]) * -3) % qi
    assert np.max(np.abs(sc.decrypt_slots(m3) - (-3) * z)) < 1e-3
    c = bt.add_const(ctx, ct, lvl, bt.llround(0.75 * sc.scale))
    assert np.array_equal(c[1], ct[1])
    assert np.max(np.abs(sc.decrypt_slots(c) - (z + 0.75))) < 1e-3
