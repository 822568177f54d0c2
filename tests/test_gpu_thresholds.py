"""Centred-lift thresholds on the GPU.

Fast base conversion (ModUp, ModDown) and the rescale lift each coefficient y in [0, q) to the
centred representative: y itself when y <= (q-1)/2, y - q when y > (q-1)/2.  Uniform inputs land
on the boundary with probability about 2^-30 per value, so these tests plant it: the inputs are
built so that, after the inverse NTT and the constant factor the step applies, the lifted values
are exactly (q-1)/2, (q+1)/2, 0 and q-1, mixed across the limbs of a digit.  The GPU result
must equal the oracle bit for bit.

Planted values (per coefficient n < N/2, limb i of the group, pattern k = (n + i) mod 4):
  k = 0: (q-1)/2, the largest value kept positive;   k = 1: (q+1)/2, the smallest made negative;
  k = 2: 0;                                           k = 3: q-1, which lifts to -1.
Coefficients n >= N/2 are uniform.
"""
import numpy as np
import pytest

import workloads as W

torch = pytest.importorskip("torch")


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint32)).cuda()


def _host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


def _planted(q: int, i: int, n: int, gen) -> np.ndarray:
    """Coefficient-domain values of one limb with the threshold pattern in the first half."""
    v = gen.integers(0, q, size=n, dtype=np.uint64)
    idx = np.arange(n // 2)
    pat = np.array([(q - 1) // 2, (q + 1) // 2, 0, q - 1], dtype=np.uint64)
    v[: n // 2] = pat[(idx + i) % 4]
    return v


def _prod_mod(ms, m) -> int:
    r = 1
    for x in ms:
        r = (r * x) % m
    return r


def _setup(ks, oracle_mod, key, mode):
    cfg = W.CONFIGS[key]
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    octx = oracle_mod.Ctx(cfg.log_n, cfg.n_q, cfg.n_p)
    assert octx.q == q and octx.p == p
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    ks.ckks_set_bconv_mode(ctx, ks.CKKS_BCONV_TENSOR if mode == "tensor" else ks.CKKS_BCONV_CUDA_CORES)
    return cfg, octx, ctx


CASES = [("n12-dnum2", 3), ("n14-hoisted8", 11), ("n14-hoisted8", 6), ("n16-full", 35)]
MODES = ["cuda_cores", "tensor"]       # the base-conversion engine (same bits either way)


@pytest.mark.gpu
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("key,level", CASES)
def test_modup_threshold(ks_lib, oracle_mod, key, level, mode):
    """ModUp: y_i = iNTT(c_i) (D_j/q_i)^-1 lands on the thresholds, so c_i = NTT(y_i (D_j/q_i))."""
    ks = ks_lib
    cfg, octx, ctx = _setup(ks, oracle_mod, key, mode)
    n, na, alpha = cfg.n, level + 1, cfg.alpha
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 5150 + level)
    coef = np.empty((na, n), dtype=np.uint32)
    for i in range(na):
        qi = octx.q[i]
        lo = (i // alpha) * alpha
        others = [octx.q[t] for t in range(lo, min(lo + alpha, na)) if t != i]
        d = _prod_mod(others, qi)
        coef[i] = ((_planted(qi, i, n, gen) * np.uint64(d)) % np.uint64(qi)).astype(np.uint32)
    c = octx.ntt_fwd(coef, 0)
    beta = -(-na // alpha)
    dt = torch.empty((beta, na + cfg.n_p, n), dtype=torch.uint32, device="cuda")
    ks.ckks_modup(ctx, _dev(c), level, dt, ctx.workspace(level))
    assert np.array_equal(_host(dt), octx.modup(c, level, alpha))


@pytest.mark.gpu
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("key,level", CASES)
def test_moddown_threshold(ks_lib, oracle_mod, key, level, mode):
    """ModDown: the special limbs' y_i = iNTT(acc_{p_i}) (P/p_i)^-1 land on the thresholds."""
    ks = ks_lib
    cfg, octx, ctx = _setup(ks, oracle_mod, key, mode)
    n, na, k = cfg.n, level + 1, cfg.n_p
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 6150 + level)
    acc = W.uniform_residues(octx.q[:na] + octx.p, n, gen)
    coef = np.empty((k, n), dtype=np.uint32)
    for i in range(k):
        pi = octx.p[i]
        d = _prod_mod([octx.p[t] for t in range(k) if t != i], pi)
        coef[i] = ((_planted(pi, i, n, gen) * np.uint64(d)) % np.uint64(pi)).astype(np.uint32)
    acc[na:] = octx.ntt_fwd(coef, cfg.n_q)
    out = torch.empty((na, n), dtype=torch.uint32, device="cuda")
    ks.ckks_moddown(ctx, _dev(acc), level, out, ctx.workspace(level))
    assert np.array_equal(_host(out), octx.moddown(acc, level))


@pytest.mark.gpu
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("key,level", CASES)
def test_rescale_threshold(ks_lib, oracle_mod, key, level, mode):
    """Rescale: limb l of both components holds (q_l -+ 1)/2, 0 and q_l - 1 as coefficients."""
    ks = ks_lib
    cfg, octx, ctx = _setup(ks, oracle_mod, key, mode)
    n, na = cfg.n, level + 1
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 7150 + level)
    ct = W.uniform_residues(octx.q[:na] * 2, n, gen).reshape(2, na, n)
    ql = octx.q[level]
    for comp in range(2):
        ct[comp, level] = octx.ntt_fwd(_planted(ql, comp, n, gen).astype(np.uint32)[None], level)[0]
    out = torch.empty((2, level, n), dtype=torch.uint32, device="cuda")
    ks.ckks_rescale(ctx, _dev(ct), level, out, ctx.workspace(level))
    assert np.array_equal(_host(out), octx.rescale(ct, level))


def test_planted_values_lift_as_stated(oracle_mod):
    """The construction itself (CPU): the oracle's inverse NTT of a planted limb, times the
    conversion factor's inverse, gives back the four threshold values."""
    cfg = W.CONFIGS["n14-hoisted8"]
    octx = oracle_mod.Ctx(cfg.log_n, cfg.n_q, cfg.n_p)
    n, q0 = cfg.n, octx.q[0]
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 1)
    d = _prod_mod(octx.q[1:cfg.alpha], q0)
    v = _planted(q0, 0, n, gen)
    c = octx.ntt_fwd(((v * np.uint64(d)) % np.uint64(q0)).astype(np.uint32)[None], 0)
    back = octx.ntt_inv(c, 0)[0].astype(np.uint64) * np.uint64(pow(d, -1, q0)) % np.uint64(q0)
    assert np.array_equal(back, v)
    assert list(back[:4]) == [(q0 - 1) // 2, (q0 + 1) // 2, 0, q0 - 1]
