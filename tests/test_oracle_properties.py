"""Randomised properties of the oracle (hypothesis): small rings, random chains, levels, digit
widths and inputs, each property checked against its mathematical definition (Python integers
or brute force), independently of the fixed cases of the other pins.

- NTT: multiplication in the evaluation domain is the negacyclic convolution of the
  coefficients, and the inverse undoes the forward transform;
- automorphism: kappa_g kappa_h = kappa_(gh mod 2N) in the evaluation domain;
- ModUp: every converted coefficient is a lift of the digit's residues within alpha/2 digit
  moduli of the centred CRT value;
- rescale: the exact division (C - [C]_q_l) / q_l, recomputed from the composite integer C.
"""
import numpy as np
import pytest

hypothesis = pytest.importorskip("hypothesis")
from hypothesis import given, settings, strategies as st  # noqa: E402

SETTINGS = settings(max_examples=25, deadline=None, derandomize=True)


def _ctx(oracle_mod, log_n, n_q, n_p):
    return oracle_mod.Ctx(log_n, n_q, n_p)


def _rand(ctx, t, seed):
    return np.random.default_rng(seed).integers(0, ctx.mod[t], ctx.n, dtype=np.uint64).astype(np.uint32)


@SETTINGS
@given(log_n=st.integers(3, 6), t=st.integers(0, 3), seed=st.integers(0, 2**31))
def test_ntt_is_negacyclic_convolution(oracle_mod, log_n, t, seed):
    ctx = _ctx(oracle_mod, log_n, 3, 1)
    n, q = ctx.n, ctx.mod[t]
    a, b = _rand(ctx, t, seed), _rand(ctx, t, seed + 1)
    prod = (ctx.ntt_fwd(a[None], t)[0].astype(np.uint64) * ctx.ntt_fwd(b[None], t)[0]) % q
    got = ctx.ntt_inv(prod.astype(np.uint32)[None], t)[0]
    want = [0] * n
    for i in range(n):
        for j in range(n):
            k, s = (i + j) % n, -1 if i + j >= n else 1
            want[k] = (want[k] + s * int(a[i]) * int(b[j])) % q
    assert [int(v) for v in got] == want
    assert np.array_equal(ctx.ntt_inv(ctx.ntt_fwd(a[None], t), t)[0], a)


@SETTINGS
@given(log_n=st.integers(3, 8), gi=st.integers(0, 10**6), hi=st.integers(0, 10**6), seed=st.integers(0, 2**31))
def test_automorphisms_compose(oracle_mod, log_n, gi, hi, seed):
    ctx = _ctx(oracle_mod, log_n, 2, 1)
    m = 2 * ctx.n
    g, h = 2 * (gi % ctx.n) + 1, 2 * (hi % ctx.n) + 1
    a = _rand(ctx, 0, seed)[None]
    assert np.array_equal(ctx.automorph_eval(ctx.automorph_eval(a, g), h), ctx.automorph_eval(a, (g * h) % m))


@SETTINGS
@given(n_q=st.integers(2, 7), n_p=st.integers(1, 4), dnum=st.integers(1, 7), lv=st.integers(0, 6),
       seed=st.integers(0, 2**31))
def test_modup_lifts_within_the_centred_bound(oracle_mod, n_q, n_p, dnum, lv, seed):
    ctx = _ctx(oracle_mod, 4, n_q, n_p)
    level = lv % n_q
    alpha = -(-n_q // min(dnum, n_q))
    na = level + 1
    c = np.stack([_rand(ctx, i, seed + i) for i in range(na)])
    dt = ctx.modup(c, level, alpha)
    x = ctx.ntt_inv(c, 0)
    ext = ctx.ext_limbs(level)
    for j, (lo, hi) in enumerate(ctx.digits(level, alpha)):
        D = 1
        for i in range(lo, hi):
            D *= ctx.mod[i]
        for u in range(len(ext)):
            if lo <= u < hi:
                assert np.array_equal(dt[j, u], c[u])
                continue
            t = ext[u]
            coef = ctx.ntt_inv(dt[j, u][None], t)[0]
            for k in (0, ctx.n // 2, ctx.n - 1):
                # the centred conversion of the digit's residues at coefficient k, with Python integers
                s = 0
                for i in range(lo, hi):
                    qi = ctx.mod[i]
                    di = D // qi
                    y = int(x[i, k]) * pow(di % qi, -1, qi) % qi
                    if y > (qi - 1) // 2:
                        y -= qi
                    s += y * di
                assert int(coef[k]) == s % ctx.mod[t]
                X = s  # a lift of every residue x_i, within alpha/2 multiples of D of the centred CRT value
                assert all(X % ctx.mod[i] == int(x[i, k]) for i in range(lo, hi))
                assert abs(X) <= (hi - lo) * D // 2 + D // 2


@SETTINGS
@given(n_q=st.integers(2, 6), lv=st.integers(1, 5), seed=st.integers(0, 2**31))
def test_rescale_is_exact_division(oracle_mod, n_q, lv, seed):
    ctx = _ctx(oracle_mod, 4, n_q, 1)
    level = 1 + (lv - 1) % (n_q - 1)
    na = level + 1
    ct = np.stack([np.stack([_rand(ctx, i, seed + 7 * comp + i) for i in range(na)]) for comp in range(2)])
    out = ctx.rescale(ct, level)
    ql = ctx.mod[level]
    for comp in range(2):
        coef = ctx.ntt_inv(ct[comp], 0)
        got = ctx.ntt_inv(out[comp], 0)
        for k in (0, 3, ctx.n - 1):
            C = ctx.crt_centered(coef[:, k:k + 1], range(na))[0]
            r = C % ql
            if r > (ql - 1) // 2:
                r -= ql
            want = (C - r) // ql
            for i in range(level):
                assert int(got[i, k]) == want % ctx.mod[i]
