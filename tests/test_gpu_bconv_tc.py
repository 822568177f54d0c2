"""Base conversion on the tensor cores (CKKS_BCONV_TENSOR) against the oracle, bit for bit.

The tensor-core engine computes the same residues as the CUDA-core one through an exact 8-bit
contraction, so every entry point must give the oracle's bits in either mode.  Covered: ModUp and
ModDown alone (full and partial last digits, groups of 1 to 12 primes), the key switch, rotation
and relinearisation, a batch of items with several target chunks, hoisted rotations, the
centred-lift thresholds, and groups wider than 15 primes (which fall back to the CUDA cores)."""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint32)).cuda()


def _host(t):
    torch.cuda.synchronize()
    return t.cpu().numpy()


def _ctx(ks, oracle_mod, log_n, n_q, n_p, dnum):
    q, p = ks.ckks_gen_primes(log_n, n_q, n_p)
    octx = oracle_mod.Ctx(log_n, n_q, n_p)
    assert octx.q == q and octx.p == p
    ctx = ks.Context(log_n, q, p, dnum)
    ks.ckks_set_bconv_mode(ctx, ks.CKKS_BCONV_TENSOR)
    return q, p, octx, ctx


@pytest.mark.parametrize("key,level", [("n12-dnum2", 3), ("n12-dnum4", 2), ("n14-hoisted8", 11),
                                       ("n14-hoisted8", 6), ("n16-full", 35), ("n16-stream64", 20),
                                       ("n16-full", 0)])
def test_tc_modup_moddown(ks_lib, oracle_mod, key, level):
    ks = ks_lib
    cfg = W.CONFIGS[key]
    q, p, octx, ctx = _ctx(ks, oracle_mod, cfg.log_n, cfg.n_q, cfg.n_p, cfg.dnum)
    n, na = cfg.n, level + 1
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 8100 + level)
    c = W.uniform_residues(q[:na], n, gen)
    beta = -(-na // cfg.alpha)
    ext = na + cfg.n_p
    dt = torch.empty((beta, ext, n), dtype=torch.uint32, device="cuda")
    ks.ckks_modup(ctx, _dev(c), level, dt, ctx.workspace(level))
    assert np.array_equal(_host(dt), octx.modup(c, level, cfg.alpha))
    acc = W.uniform_residues(q[:na] + p, n, gen)
    out = torch.empty((na, n), dtype=torch.uint32, device="cuda")
    ks.ckks_moddown(ctx, _dev(acc), level, out, ctx.workspace(level))
    assert np.array_equal(_host(out), octx.moddown(acc, level))


@pytest.mark.parametrize("log_n,level", [(13, 5), (13, 2), (15, 5), (15, 4)])
def test_tc_modup_moddown_every_ring(ks_lib, oracle_mod, log_n, level):
    """N = 2^13 and 2^15, 6 + 2 primes, dnum 3, full and partial last digits: ModUp and ModDown
    equal the oracle."""
    ks = ks_lib
    q, p, octx, ctx = _ctx(ks, oracle_mod, log_n, 6, 2, 3)
    n, na, alpha = 1 << log_n, level + 1, 2
    gen = W.rng(3, W.TAG_SYNTH, 8400 + 16 * log_n + level)
    c = W.uniform_residues(q[:na], n, gen)
    beta, ext = -(-na // alpha), na + 2
    dt = torch.empty((beta, ext, n), dtype=torch.uint32, device="cuda")
    ks.ckks_modup(ctx, _dev(c), level, dt, ctx.workspace(level))
    assert np.array_equal(_host(dt), octx.modup(c, level, alpha))
    acc = W.uniform_residues(q[:na] + p, n, gen)
    out = torch.empty((na, n), dtype=torch.uint32, device="cuda")
    ks.ckks_moddown(ctx, _dev(acc), level, out, ctx.workspace(level))
    assert np.array_equal(_host(out), octx.moddown(acc, level))


@pytest.mark.parametrize("key", ["n12-dnum2", "n14-hoisted8", "n16-full"])
def test_tc_rotate_relin_and_modes_agree(ks_lib, oracle_mod, key):
    """Rotation and relinearisation with oracle-built keys; every other mode gives the same bits."""
    from oracle.scenario import Scenario
    ks = ks_lib
    cfg = W.CONFIGS[key]
    sc = Scenario(cfg)
    q, p, octx, ctx = _ctx(ks, oracle_mod, cfg.log_n, cfg.n_q, cfg.n_p, cfg.dnum)
    lvl = cfg.level
    _, x = sc.ciphertext(0)
    _, y = sc.ciphertext(1)
    g = sc.galois(cfg.rot_steps[0])
    bg, b0 = sc.key(g), sc.key(0)
    evk_g = ks.make_evk(_dev(bg), cfg.chacha_seed, g)
    evk_0 = ks.make_evk(_dev(b0), cfg.chacha_seed, 0)
    ws = ctx.workspace(lvl)
    out = torch.empty((2, lvl + 1, cfg.n), dtype=torch.uint32, device="cuda")
    ks.ckks_rotate(ctx, _dev(x), lvl, g, evk_g, out, ws)
    want_rot = octx.rotate(x, lvl, cfg.alpha, g, bg, cfg.chacha_seed, g)
    assert np.array_equal(_host(out), want_rot)
    d = torch.empty((3, lvl + 1, cfg.n), dtype=torch.uint32, device="cuda")
    ks.ckks_tensor(ctx, _dev(x), _dev(y), lvl, d)
    ks.ckks_relin(ctx, d, lvl, evk_0, out, ws)
    want_rel = octx.relin(octx.tensor(x, y, lvl), lvl, cfg.alpha, b0, cfg.chacha_seed, 0)
    assert np.array_equal(_host(out), want_rel)
    for other in (ks.CKKS_BCONV_CUDA_CORES, ks.CKKS_BCONV_AUTO):
        ks.ckks_set_bconv_mode(ctx, other)
        ks.ckks_rotate(ctx, _dev(x), lvl, g, evk_g, out, ws)
        assert np.array_equal(_host(out), want_rot), other


def test_tc_batch_and_hoisted(ks_lib, oracle_mod):
    """A 5-item key-switch batch (several items per launch and two target chunks per group) and
    4 hoisted rotations at N=2^14; every item equals the oracle."""
    ks = ks_lib
    cfg = W.CONFIGS["n14-hoisted8"]
    q, p, octx, ctx = _ctx(ks, oracle_mod, cfg.log_n, cfg.n_q, cfg.n_p, cfg.dnum)
    lvl, n = cfg.level, cfg.n
    na, items = lvl + 1, 5
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 8200)
    nd = -(-cfg.n_q // cfg.alpha)
    keys = [W.uniform_residues((q + p) * nd, n, gen).reshape(nd, len(q) + len(p), n) for _ in range(items)]
    seed = bytes(range(32))
    evks = [ks.make_evk(_dev(k), seed, 2 * i + 3) for i, k in enumerate(keys)]
    c = W.uniform_residues(q[:na] * items, n, gen).reshape(items, na, n)
    out = torch.empty((items, 2, na, n), dtype=torch.uint32, device="cuda")
    ks.ckks_keyswitch_batch(ctx, _dev(c), lvl, evks, out, ctx.workspace(lvl, items))
    got = _host(out)
    for i in range(items):
        assert np.array_equal(got[i], octx.keyswitch(c[i], lvl, cfg.alpha, keys[i], seed, 2 * i + 3)), i
    ct = W.uniform_residues(q[:na] * 2, n, gen).reshape(2, na, n)
    gs = [ks.galois_element(cfg.log_n, r) for r in (1, -2, 4, -8)]
    hk = [ks.make_evk(_dev(keys[i]), seed, gs[i]) for i in range(4)]
    rot = torch.empty((4, 2, na, n), dtype=torch.uint32, device="cuda")
    ks.ckks_rotate_hoisted(ctx, _dev(ct), lvl, gs, hk, rot, ctx.workspace(lvl, 4))
    want = octx.rotate_hoisted(ct, lvl, cfg.alpha, gs, keys[:4], [seed] * 4, gs)
    assert np.array_equal(_host(rot), want)


def test_tc_wide_groups_fall_back(ks_lib, oracle_mod):
    """dnum 1 at N=2^12 (a digit of 36 primes, 24 special primes): both conversions are wider
    than the tensor-core tile and run on the CUDA cores; the output is the oracle's."""
    ks = ks_lib
    q, p, octx, ctx = _ctx(ks, oracle_mod, 12, 36, 24, 1)
    n, lvl = 1 << 12, 35
    gen = W.rng(1, W.TAG_SYNTH, 8300)
    c = W.uniform_residues(q, n, gen)
    key = W.uniform_residues(q + p, n, gen).reshape(1, 60, n)
    seed = bytes(range(32))
    out = torch.empty((2, 36, n), dtype=torch.uint32, device="cuda")
    ks.ckks_keyswitch(ctx, _dev(c), lvl, ks.make_evk(_dev(key), seed, 5), out, ctx.workspace(lvl))
    assert np.array_equal(_host(out), octx.keyswitch(c, lvl, 36, key, seed, 5))


def test_tc_mode_errors(ks_lib):
    ks = ks_lib
    q, p = ks.ckks_gen_primes(12, 4, 1)
    ctx = ks.Context(12, q, p, 2)
    with pytest.raises(ks.CkksError) as e:
        ks.ckks_set_bconv_mode(ctx, 7)
    assert e.value.code == ks.CKKS_ERR_ARG
