"""Pins for ModUp and ModDown (fast base conversion).

Property checks: the ModUp output of digit j is, coefficient by coefficient, an integer V
(recovered by CRT over the target limbs) that is a lift of the digit's residues
(V = x_i mod q_i) with V = X + u*D_j, X the centred CRT lift and |u| <= alpha/2; digit limbs
pass through unchanged.  ModDown of P*c + e with small e returns c - u with |u| <= k/2.
An exact Python-integer evaluation of the centred conversion is checked as well.
"""
import numpy as np
import pytest


def _centered(v, m):
    v %= m
    return v - m if v > m // 2 else v


def _crt(residues, mods):
    M = 1
    for m in mods:
        M *= m
    x = 0
    for r, m in zip(residues, mods):
        mi = M // m
        x += r * mi * pow(mi % m, -1, m)
    return _centered(x, M), M


@pytest.mark.parametrize("log_n,n_q,n_p,alpha,level", [
    (5, 6, 4, 2, 5), (5, 6, 4, 2, 4), (5, 7, 5, 3, 6), (5, 7, 5, 3, 4), (6, 4, 5, 4, 3),
    (5, 5, 6, 1, 4)])
def test_modup_properties(oracle_mod, log_n, n_q, n_p, alpha, level):
    ctx = oracle_mod.Ctx(log_n, n_q, n_p)
    n = ctx.n
    na = level + 1
    rng = np.random.default_rng(level * 31 + alpha)
    c = np.stack([rng.integers(0, ctx.mod[t], n, dtype=np.uint64) for t in range(na)]).astype(np.uint32)
    dt = ctx.modup(c, level, alpha)
    ext = ctx.ext_limbs(level)
    assert dt.shape == (-(-na // alpha), len(ext), n)
    x = ctx.ntt_inv(c, 0)                       # digit residues in the coefficient domain
    us = []
    for j, (lo, hi) in enumerate(ctx.digits(level, alpha)):
        D = 1
        for i in range(lo, hi):
            D *= ctx.mod[i]
        tgt = [u for u in range(len(ext)) if not (lo <= u < hi)]
        for u in range(lo, hi):
            assert np.array_equal(dt[j, u], c[u])
        coef = {u: ctx.ntt_inv(dt[j, u], ext[u]) for u in tgt}
        tmods = [ctx.mod[ext[u]] for u in tgt]
        for k in range(n):
            V, M = _crt([int(coef[u][k]) for u in tgt], tmods)
            assert M > 2 * (hi - lo + 1) * D      # targets determine V
            for i in range(lo, hi):
                assert V % ctx.mod[i] == int(x[i, k])
            X, _ = _crt([int(x[i, k]) for i in range(lo, hi)], [ctx.mod[i] for i in range(lo, hi)])
            assert (V - X) % D == 0
            u_ = (V - X) // D
            assert abs(u_) <= (hi - lo) / 2
            us.append(u_)
            # exact centred conversion in Python integers
            W = 0
            for i in range(lo, hi):
                qi = ctx.mod[i]
                Di = D // qi
                W += _centered(int(x[i, k]) * pow(Di % qi, -1, qi), qi) * Di
            assert W == V
    if alpha >= 3:
        assert abs(np.mean(us)) < 0.5


@pytest.mark.parametrize("log_n,n_q,n_p,level", [(5, 4, 3, 3), (5, 6, 4, 2), (6, 3, 1, 2)])
def test_moddown_divides_by_p(oracle_mod, log_n, n_q, n_p, level):
    ctx = oracle_mod.Ctx(log_n, n_q, n_p)
    n, na = ctx.n, level + 1
    rng = np.random.default_rng(n_p)
    P = 1
    for p in ctx.p:
        P *= p
    ext = ctx.ext_limbs(level)
    c_coef = np.stack([rng.integers(0, ctx.mod[t], n, dtype=np.uint64) for t in range(na)])
    e = rng.integers(-1000, 1000, n)
    acc = np.empty((len(ext), n), dtype=np.uint32)
    for u, t in enumerate(ext):
        m = ctx.mod[t]
        cu = [int(v) for v in c_coef[u]] if u < na else [0] * n
        acc[u] = np.array([(P * cu[k] + int(e[k])) % m for k in range(n)], dtype=np.uint32)
    acc_eval = np.stack([ctx.ntt_fwd(acc[u], ext[u]) for u in range(len(ext))])
    out = ctx.moddown(acc_eval, level)
    out_coef = ctx.ntt_inv(out, 0)
    diffs = np.stack([(out_coef[i].astype(np.int64) - c_coef[i].astype(np.int64)) % ctx.mod[i]
                      for i in range(na)])
    for k in range(n):
        d = [_centered(int(diffs[i, k]), ctx.mod[i]) for i in range(na)]
        assert len(set(d)) == 1 and abs(d[0]) <= n_p / 2
