"""The linear parts of bootstrapping on the GPU against the oracle, bit for bit.

ModRaise (ckks_modraise) and the DFT levels of CoeffToSlot and SlotToCoeff, each level one
baby-step giant-step transform (ckks_bsgs, double hoisting) with the level's slot diagonals
encoded by the oracle at scale q_level, followed by one rescale (ckks_rescale).  Every level's
output equals the oracle's; the last one also decodes to the numpy map (the oracle's own pin in
tests/test_oracle_dft.py)."""
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


@pytest.mark.parametrize("key,level", [("n12-dnum4", 3), ("n14-hoisted8", 11), ("n16-full", 35)])
def test_modraise_parity(ks_lib, oracle_mod, key, level):
    from oracle import bootstrap as bt
    ks = ks_lib
    cfg = W.CONFIGS[key]
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    octx = oracle_mod.Ctx(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    ct = W.uniform_residues([q[0]] * 2, cfg.n, W.rng(cfg.seed, W.TAG_SYNTH, 9100)).reshape(2, 1, cfg.n)
    out = torch.empty((2, level + 1, cfg.n), dtype=torch.uint32, device="cuda")
    ws = torch.empty(2 * cfg.n, dtype=torch.uint32, device="cuda")
    ks.ckks_modraise(ctx, _dev(ct), level, out, ws)
    assert np.array_equal(_host(out), bt.modraise(octx, ct, level))


@pytest.mark.parametrize("direction", ["coeff_to_slot", "slot_to_coeff"])
@pytest.mark.parametrize("key,levels,n1", [("n12-dnum4", 3, 4), ("n14-hoisted8", 3, 8)])
def test_dft_levels_parity(ks_lib, oracle_mod, key, levels, n1, direction):
    _dft_levels(ks_lib, key, levels, n1, direction)


@pytest.mark.slow
def test_dft_levels_parity_n16(ks_lib, oracle_mod):
    """CoeffToSlot on the N=2^16 chain (level 24, dnum 4): 15 stages in 3 levels of 5, 63
    diagonals per level in 8 baby x 8 giant steps."""
    _dft_levels(ks_lib, "n16-bsgs32", 3, 8, "coeff_to_slot")


def _dft_levels(ks_lib, key, levels, n1, direction):
    from oracle import bootstrap as bt
    from oracle.scenario import Scenario
    ks = ks_lib
    cfg = W.CONFIGS[key]
    sc = Scenario(cfg)
    octx, log_n, ns = sc.ctx, cfg.log_n, cfg.n // 2
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    inverse = direction == "coeff_to_slot"
    z, ct = sc.ciphertext(0)
    if not inverse:
        z = z / 4.0
        ct = sc.encrypt_slots(z, 0)
    lvl = cfg.level
    keys, evks = {}, {}
    g_ct = _dev(ct)
    for lens in bt.split_levels(log_n, levels, inverse):
        babies, giants, pt = bt.bsgs_plan(bt.level_diagonals(log_n, lens, inverse), ns, n1)
        for s in babies + giants:
            g = bt.galois_of_shift(octx, s)
            if g != 1 and g not in keys:
                keys[g] = sc.key(g)
                evks[g] = ks.make_evk(_dev(keys[g]), cfg.chacha_seed, g)
        enc = bt.encode_plan(octx, pt, lvl, float(octx.q[lvl]))
        want = bt.linear_level(octx, ct, lvl, cfg.alpha, babies, giants, enc, keys, cfg.chacha_seed)
        bg = [bt.galois_of_shift(octx, s) for s in babies]
        gg = [bt.galois_of_shift(octx, s) for s in giants]
        na = lvl + 1
        mid = torch.empty((2, na, cfg.n), dtype=torch.uint32, device="cuda")
        ws = ks.ckks_bsgs_workspace(ctx, lvl, len(bg), len(gg))
        ks.ckks_bsgs(ctx, g_ct, lvl, bg, [evks.get(g) for g in bg], gg, [evks.get(g) for g in gg], _dev(enc),
                     mid, ws)
        g_next = torch.empty((2, lvl, cfg.n), dtype=torch.uint32, device="cuda")
        ks.ckks_rescale(ctx, mid, lvl, g_next, ctx.workspace(lvl))
        assert ks.ckks_sync_status(ctx, None, 10000) == ks.CKKS_OK
        assert np.array_equal(_host(g_next), want), (direction, lvl)
        ct, g_ct, lvl = want, g_next, lvl - 1
    got = sc.decrypt_slots(_host(g_ct), lvl)
    ref = bt.coeff_to_slot(z, log_n, levels) if inverse else bt.slot_to_coeff(z, log_n, levels)
    err = np.max(np.abs(got - ref))
    assert err < (2.0 ** -8 if inverse else 2.0 ** -9 * np.max(np.abs(ref))), err


def test_constant_ops_parity(ks_lib, oracle_mod):
    """ckks_mul_const, ckks_add_const and ckks_add against the oracle's restatement, bit for bit,
    with negative constants and constants above the primes."""
    from oracle import bootstrap as bt
    ks = ks_lib
    cfg = W.CONFIGS["n14-hoisted8"]
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    octx = oracle_mod.Ctx(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    lvl, n = cfg.level, cfg.n
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 9300)
    x = W.uniform_residues(q[: lvl + 1] * 2, n, gen).reshape(2, lvl + 1, n)
    y = W.uniform_residues(q[: lvl + 1] * 2, n, gen).reshape(2, lvl + 1, n)
    out = torch.empty((2, lvl + 1, n), dtype=torch.uint32, device="cuda")
    for v in (-3, 2, 5 * (1 << 40) + 7, -(1 << 45) - 1):
        ks.ckks_mul_const(ctx, _dev(x), 2, lvl, v, out)
        assert np.array_equal(_host(out), bt.mul_const(octx, x, lvl, v)), v
        ks.ckks_add_const(ctx, _dev(x), lvl, v, out)
        assert np.array_equal(_host(out), bt.add_const(octx, x, lvl, v)), v
    ks.ckks_add(ctx, _dev(x), _dev(y), 2, lvl, out)
    mods = np.array(q[: lvl + 1], dtype=np.uint64)[:, None]
    assert np.array_equal(_host(out), ((x.astype(np.uint64) + y) % mods).astype(np.uint32))


def _evalmod_case(ks, oracle_mod, key, level, r, d, check_decode):
    from oracle import bootstrap as bt
    from oracle.scenario import Scenario
    cfg = W.CONFIGS[key]
    sc = Scenario(cfg)
    octx = sc.ctx
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    S = float(octx.q[level])
    x = np.random.default_rng(5).uniform(-2, 2, cfg.n // 2)
    m = oracle_mod.encode(x.astype(complex), cfg.n, S)
    e = W.gaussian_error(cfg.n, cfg.sigma, W.rng(cfg.seed, W.TAG_ENC_ERR, 77))[0]
    a = W.uniform_residues(octx.q[: level + 1], cfg.n, W.rng(cfg.seed, W.TAG_ENC_A, 77))
    ct = octx.encrypt(sc.s, m, e, a, level)
    b0 = sc.key(0)
    want, lv, so = bt.evalmod(octx, ct, level, S, r, d, cfg.alpha, b0, cfg.chacha_seed)
    evk = ks.make_evk(_dev(b0), cfg.chacha_seed, 0)
    out = torch.empty((2, level + 1, cfg.n), dtype=torch.uint32, device="cuda")
    g_lv, g_so = ks.ckks_evalmod(ctx, _dev(ct), level, S, r, d, evk, out, ks.ckks_evalmod_workspace(ctx, level))
    assert (g_lv, g_so) == (lv, so)
    got = _host(out).reshape(-1)[: 2 * (lv + 1) * cfg.n].reshape(2, lv + 1, cfg.n)
    assert np.array_equal(got, want)
    if check_decode:
        err = np.abs(sc.decrypt_slots(got, lv, so).real - np.sin(2 * np.pi * x) / (2 * np.pi))
        assert err.max() < 2.0 ** -9


def test_evalmod_parity_n14(ks_lib, oracle_mod):
    """EvalMod (degree 8 in theta, two double angles) at N=2^14 from level 11, bit for bit (this
    chain's key-switching noise is too large for the decoded values to mean much)."""
    _evalmod_case(ks_lib, oracle_mod, "n14-hoisted8", 11, 2, 4, False)


def test_evalmod_batch_equals_single_calls(ks_lib, oracle_mod):
    """ckks_evalmod_batch on 3 ciphertexts at N=2^14 (level 11, degree 8, two double angles): each
    item equals ckks_evalmod on it alone, bit for bit (and that call equals the oracle, above)."""
    ks = ks_lib
    cfg = W.CONFIGS["n14-hoisted8"]
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    lvl, n, nb = 11, cfg.n, 3
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 9400)
    ct = W.uniform_residues(q[: lvl + 1] * 2 * nb, n, gen).reshape(nb, 2, lvl + 1, n)
    nd = -(-cfg.n_q // cfg.alpha)
    b0 = W.uniform_residues((q + p) * nd, n, gen).reshape(nd, len(q) + len(p), n)
    evk = ks.make_evk(_dev(b0), cfg.chacha_seed, 0)
    S = float(q[lvl])
    out = torch.empty((nb, 2, lvl + 1, n), dtype=torch.uint32, device="cuda")
    lv, so = ks.ckks_evalmod_batch(ctx, _dev(ct), lvl, S, 2, 4, evk, out, ks.ckks_evalmod_batch_workspace(ctx, lvl, nb))
    got = _host(out).reshape(-1)[: nb * 2 * (lv + 1) * n].reshape(nb, 2, lv + 1, n)
    one = torch.empty((2, lvl + 1, n), dtype=torch.uint32, device="cuda")
    ws1 = ks.ckks_evalmod_workspace(ctx, lvl)
    for i in range(nb):
        assert ks.ckks_evalmod(ctx, _dev(ct[i]), lvl, S, 2, 4, evk, one, ws1) == (lv, so)
        assert np.array_equal(_host(one).reshape(-1)[: 2 * (lv + 1) * n].reshape(2, lv + 1, n), got[i]), i
    assert ks.ckks_sync_status(ctx, None, 10000) == ks.CKKS_OK


@pytest.mark.slow
def test_evalmod_parity_n16(ks_lib, oracle_mod):
    """EvalMod (degree 12, three double angles) at N=2^16, dnum 4, from level 35: bit for bit with
    the oracle, and decoding to sin(2 pi x) / (2 pi) within 2^-9."""
    _evalmod_case(ks_lib, oracle_mod, "n16-stream64", 35, 3, 6, True)


def test_mul_i_parity(ks_lib, oracle_mod):
    """ckks_mul_i (X^(N/2) in the evaluation domain: w or -w per half) against the oracle's
    coefficient-domain negacyclic shift, bit for bit, on 3 components at level 7 of n12-boot."""
    from oracle import bootstrap as bt
    ks = ks_lib
    cfg = W.CONFIGS["n12-boot"]
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    octx = oracle_mod.Ctx(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    lvl = 7
    x = W.uniform_residues(q[: lvl + 1] * 3, cfg.n, W.rng(cfg.seed, W.TAG_SYNTH, 9500)).reshape(3, lvl + 1, cfg.n)
    out = torch.empty((3, lvl + 1, cfg.n), dtype=torch.uint32, device="cuda")
    ks.ckks_mul_i(ctx, _dev(x), 3, lvl, out)
    assert np.array_equal(_host(out), bt.mul_monomial_half(octx, x, lvl))


def test_bootstrap_parity_n12(ks_lib, oracle_mod):
    """ckks_bootstrap on the n12-boot chain (level 0 -> 23 -> 5: CoeffToSlot and SlotToCoeff in 3
    levels of 8 baby steps, EvalMod of degree 12 with three double angles) equals the oracle's
    bootstrap bit for bit, twice in a row on one workspace; the output decodes to the input slots
    (the oracle's own pin, tests/test_oracle_bootstrap.py)."""
    _bootstrap_case(ks_lib, "n12-boot", (0, 1))


@pytest.mark.slow
def test_bootstrap_parity_n16(ks_lib, oracle_mod):
    """The benchmark's bootstrap shape at full size: N=2^16, 36+12 primes, dnum 4, level 0 -> 35 ->
    17 (CoeffToSlot and SlotToCoeff in 3 levels of 8 baby x 8 giant steps, EvalMod of degree 12 with
    three double angles), bit for bit with the oracle, and decoding to the input slots (measured
    2^-8.7 at most with the oracle; the oracle takes minutes here)."""
    _bootstrap_case(ks_lib, "n16-boot", (0,))


def _bootstrap_case(ks_lib, key, indices):
    from oracle import bootstrap as bt
    from oracle.scenario import Scenario
    ks = ks_lib
    cfg = W.CONFIGS[key]
    sc = Scenario(cfg)
    octx = sc.ctx
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    r, d, levels, n1 = 3, 6, 3, 8
    c2s_p, s2c_p = bt.bootstrap_plans(cfg.log_n, levels, n1)
    lc, ls, lout = bt.bootstrap_levels(cfg.level, levels, levels, r, d)
    c2s, g1 = bt.encoded_plans(octx, c2s_p, lc)
    s2c, g2 = bt.encoded_plans(octx, s2c_p, ls)
    keys = {g: sc.key(g) for g in sorted(set(g1) | set(g2))}
    evks = {g: ks.make_evk(_dev(b), cfg.chacha_seed, g) for g, b in keys.items()}
    g_conj = 2 * cfg.n - 1
    conj_b, relin_b = sc.key(g_conj), sc.key(0)

    def gpu_levels(plans):
        out = []
        for babies, giants, enc in plans:
            bg = [bt.galois_of_shift(octx, s) for s in babies]
            gg = [bt.galois_of_shift(octx, s) for s in giants]
            out.append((bg, [evks.get(g) for g in bg], gg, [evks.get(g) for g in gg], _dev(enc)))
        return out

    plan = ks.BootstrapPlan(cfg.level, gpu_levels(c2s), gpu_levels(s2c),
                            ks.make_evk(_dev(conj_b), cfg.chacha_seed, g_conj),
                            ks.make_evk(_dev(relin_b), cfg.chacha_seed, 0), r, d)
    assert plan.out_level == lout
    ws = ks.ckks_bootstrap_workspace(ctx, plan)
    out = torch.empty((2, lout + 1, cfg.n), dtype=torch.uint32, device="cuda")
    for index in indices:
        z, ct = sc.ciphertext(index, level=0)
        want, lv, ratio = bt.bootstrap(octx, ct, cfg.level, cfg.alpha, c2s, s2c, keys, conj_b, relin_b,
                                       cfg.chacha_seed, r, d)
        g_lv, g_ratio = ks.ckks_bootstrap(ctx, _dev(ct.reshape(2, 1, cfg.n)), plan, out, ws)
        assert ks.ckks_sync_status(ctx, None, 10000) == ks.CKKS_OK
        assert (g_lv, g_ratio) == (lv, ratio)
        got = _host(out)
        assert np.array_equal(got, want), index
        assert np.max(np.abs(sc.decrypt_slots(got, lv, sc.scale * ratio) - z)) < 2.0 ** -6


def test_bootstrap_rejects_bad_plans(ks_lib):
    """ckks_bootstrap's argument checks: a plan that consumes more levels than the top level has
    (CKKS_ERR_UNSUPPORTED), level counts outside 1..16 and an output overlapping the input
    (CKKS_ERR_ARG), a short workspace (CKKS_ERR_WORKSPACE); nothing runs on the GPU for any of them."""
    ks = ks_lib
    cfg = W.CONFIGS["n12-boot"]
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    n, nd = cfg.n, -(-cfg.n_q // cfg.alpha)
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 9600)
    mods = q + p
    evk = ks.make_evk(_dev(W.uniform_residues(mods * nd, n, gen).reshape(nd, len(mods), n)), cfg.chacha_seed, 0)
    conj = ks.make_evk(_dev(W.uniform_residues(mods * nd, n, gen).reshape(nd, len(mods), n)), cfg.chacha_seed,
                       2 * n - 1)

    def level(lv):
        pt = _dev(W.uniform_residues(q[: lv + 1] + p, n, gen)).reshape(1, 1, lv + 1 + cfg.n_p, n)
        return ([1], [None], [1], [None], pt)

    ct = _dev(W.uniform_residues([q[0]] * 2, n, gen)).reshape(2, 1, n)

    def call(plan, out=None, ws_bytes=None):
        lv, ratio = ks._ci(), ks.ctypes.c_double()
        need = ks._L.ckks_bootstrap_workspace_bytes(ctx.handle, ks.ctypes.byref(plan.plan))
        ws = torch.empty(max(need, 1 << 20) // 4 + 64, dtype=torch.uint32, device="cuda")
        o = out if out is not None else torch.empty((2, 24, n), dtype=torch.uint32, device="cuda")
        nb = ws.numel() * 4 if ws_bytes is None else ws_bytes
        return need, ks._L.ckks_bootstrap(ctx.handle, ks._ptr(ct), ks.ctypes.byref(plan.plan), ks._ptr(o),
                                          ks.ctypes.byref(lv), ks.ctypes.byref(ratio), ks._ptr(ws), nb, None)

    # 1 + (1 + 0 + 3) + 1 = 6 levels from top level 5
    need, rc = call(ks.BootstrapPlan(5, [level(5)], [level(0)], conj, evk, 0, 1))
    assert need == 0 and rc == ks.CKKS_ERR_UNSUPPORTED
    ok = ks.BootstrapPlan(23, [level(23)], [level(18)], conj, evk, 0, 1)
    need, rc = call(ok, ws_bytes=1024)
    assert need > 0 and rc == ks.CKKS_ERR_WORKSPACE
    empty = ks.BootstrapPlan(23, [], [level(18)], conj, evk, 0, 1)
    assert call(empty)[1] == ks.CKKS_ERR_ARG
    assert call(ok, out=ct.view(-1)[: 2 * n].view(2, 1, n))[1] == ks.CKKS_ERR_ARG
    assert ks.ckks_sync_status(ctx, None, 10000) == ks.CKKS_OK
