"""Pins of the oracle's whole bootstrap (ModRaise, CoeffToSlot, the split into real and imaginary
halves, EvalMod, recombination, SlotToCoeff) and of the monomial product the split uses.

The bootstrap's defining property: the output decrypts to the input's message, although the
raised plaintext m + q_0 I carries a nonzero multiple of q_0.  The chain is the n12-boot test
chain (N=2^12, 24 + 6 primes, secret of weight 2, so |I| <= 1)."""
import numpy as np
import pytest

import workloads as W


@pytest.fixture(scope="module")
def boot_case(oracle_mod):
    from oracle import bootstrap as bt
    from oracle.scenario import Scenario
    cfg = W.CONFIGS["n12-boot"]
    sc = Scenario(cfg)
    return cfg, sc, bt


def test_monomial_half_multiplies_slots_by_i(boot_case):
    """X^(N/2) moves every slot value z_j to i z_j (decoded from a fresh encryption: up to double
    rounding, since the product is exact, and within the encryption noise of i times the message),
    and applied twice it negates the ciphertext exactly (X^N = -1)."""
    cfg, sc, bt = boot_case
    octx, lv = sc.ctx, 7
    z, ct = sc.ciphertext(3, level=lv)
    got = sc.decrypt_slots(bt.mul_monomial_half(octx, ct, lv), lv)
    assert np.max(np.abs(got - 1j * sc.decrypt_slots(ct, lv))) < 1e-9
    assert np.max(np.abs(got - 1j * z)) < 2.0 ** -16
    twice = bt.mul_monomial_half(octx, bt.mul_monomial_half(octx, ct, lv), lv)
    assert np.array_equal(twice, bt.mul_const(octx, ct, lv, -1))


def test_bootstrap_levels_consumed():
    from oracle import bootstrap as bt
    c2s, s2c, out = bt.bootstrap_levels(23, 3, 3, 3, 6)
    assert c2s == [23, 22, 21] and s2c == [8, 7, 6] and out == 5


def test_bootstrap_decodes_to_input(boot_case):
    """A level-0 encryption of uniform complex slots, bootstrapped to level 5 (CoeffToSlot and
    SlotToCoeff in 3 levels of 8 baby steps each, EvalMod of degree 12 with three double angles),
    decodes to the input slots.  The raised plaintext has I = +-1 in many coefficients, so the
    modular reduction really removes multiples of q_0.  Measured error: 2^-8.25 at most (median
    2^-10); the bound 2^-6 leaves a factor 4.  Planted mistakes give errors of order 1 or more
    (the subtraction of the split reversed: 2.7; the monomial left out: 5.8e3)."""
    cfg, sc, bt = boot_case
    octx = sc.ctx
    r, d, levels, n1 = 3, 6, 3, 8
    c2s_p, s2c_p = bt.bootstrap_plans(cfg.log_n, levels, n1)
    lc, ls, lout = bt.bootstrap_levels(cfg.level, levels, levels, r, d)
    c2s, g1 = bt.encoded_plans(octx, c2s_p, lc)
    s2c, g2 = bt.encoded_plans(octx, s2c_p, ls)
    keys = {g: sc.key(g) for g in sorted(set(g1) | set(g2))}
    z, ct = sc.ciphertext(0, level=0)
    raised = octx.decrypt(bt.modraise(octx, ct, cfg.level), cfg.level, sc.s_eval)
    I = np.array([round(float(x) / octx.q[0]) for x in raised])
    assert I.min() == -1 and I.max() == 1 and np.count_nonzero(I) > 100
    out, lv, ratio = bt.bootstrap(octx, ct, cfg.level, cfg.alpha, c2s, s2c, keys, sc.key(2 * cfg.n - 1),
                                  sc.key(0), cfg.chacha_seed, r, d)
    assert lv == lout and out.shape == (2, lv + 1, cfg.n)
    got = sc.decrypt_slots(out, lv, sc.scale * ratio)
    assert np.max(np.abs(got - z)) < 2.0 ** -6


def test_bootstrap_plans_are_the_dft_maps():
    """The plans bootstrap_plans builds, applied in the clear level by level (baby-step giant-step
    form), are half the CoeffToSlot map (the 1/2 of the real/imaginary split) and the SlotToCoeff
    map of the oracle's stage factorisation, at N=2^7 with 2 and 3 levels."""
    from oracle import bootstrap as bt
    rng = np.random.default_rng(11)
    for log_n, levels, n1 in ((7, 2, 4), (7, 3, 2)):
        ns = 1 << (log_n - 1)
        z = rng.normal(size=ns) + 1j * rng.normal(size=ns)
        c2s, s2c = bt.bootstrap_plans(log_n, levels, n1)
        x = z
        for babies, giants, pt in c2s:
            x = bt.apply_bsgs(x, babies, giants, pt)
        assert np.allclose(x, 0.5 * bt.coeff_to_slot(z, log_n, levels), atol=1e-12)
        y = z
        for babies, giants, pt in s2c:
            y = bt.apply_bsgs(y, babies, giants, pt)
        assert np.allclose(y, bt.slot_to_coeff(z, log_n, levels), atol=1e-9)


def test_monomial_half_is_the_negacyclic_product(oracle_mod):
    """mul_monomial_half at N=2^4 (2 primes) against the negacyclic product with X^(N/2) by brute
    force: c_k = sum_{i+j = k} a_i m_j - sum_{i+j = k+N} a_i m_j, m the monomial."""
    from oracle import bootstrap as bt
    log_n = 4
    n = 1 << log_n
    octx = oracle_mod.Ctx(log_n, 2, 1)
    rng = np.random.default_rng(12)
    level = 1
    comps = [np.stack([rng.integers(0, q, size=n) for q in octx.q[: level + 1]]).astype(np.uint32)
             for _ in range(2)]
    ct = np.stack([octx.ntt_fwd(c, 0) for c in comps])
    got = bt.mul_monomial_half(octx, ct, level)
    for comp in range(2):
        a = octx.ntt_inv(ct[comp], 0).astype(np.int64)
        out = octx.ntt_inv(got[comp], 0).astype(np.int64)
        for t, q in enumerate(octx.q[: level + 1]):
            want = np.zeros(n, dtype=object)
            for i in range(n):
                k = i + n // 2
                if k < n:
                    want[k] += int(a[t, i])
                else:
                    want[k - n] -= int(a[t, i])
            assert [int(v) % q for v in want] == [int(v) for v in out[t]]
