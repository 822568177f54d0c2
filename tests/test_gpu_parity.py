"""GPU parity: every step and composite call of the CUDA library, through the C ABI, against the
CPU oracle, element by element.  All of it is integer RNS arithmetic, so the bar is bit
equality.  Inputs are seeded (workloads.py) or oracle-built (keys, ciphertexts)."""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _dev(a: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint32)).cuda()


def _host(t) -> np.ndarray:
    torch.cuda.synchronize()
    return t.cpu().numpy()


def _rand_limbs(mods, n, seed):
    return W.uniform_residues(mods, n, W.rng(seed, W.TAG_SYNTH))


class Setup:
    """Oracle scenario plus the matching GPU context for one configuration."""

    def __init__(self, ks, cfg):
        from oracle.scenario import Scenario
        self.ks, self.cfg = ks, cfg
        self.sc = Scenario(cfg)
        q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
        assert q == self.sc.ctx.q and p == self.sc.ctx.p
        self.ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
        self._keys = {}

    def key(self, key_id, stored_a=False):
        if (key_id, stored_a) not in self._keys:
            if stored_a:
                b, a = self.sc.key(key_id, want_a=True)
                kb, ka = _dev(b), _dev(a)
            else:
                b = self.sc.key(key_id)
                kb, ka = _dev(b), None
            evk = self.ks.make_evk(kb, self.cfg.chacha_seed, key_id, a=ka)
            self._keys[(key_id, stored_a)] = (b, kb, ka, evk)
        return self._keys[(key_id, stored_a)]


_SETUPS = {}


def setup_for(ks, key):
    if key not in _SETUPS:
        _SETUPS[key] = Setup(ks, W.CONFIGS[key])
    return _SETUPS[key]


# ----------------------------------------------------------------------------- NTT

@pytest.mark.parametrize("log_n", [12, 13, 14, 15, 16])
def test_ntt_parity(ks_lib, oracle_mod, log_n):
    ks = ks_lib
    q, p = ks.ckks_gen_primes(log_n, 3, 2)
    ctx = ks.Context(log_n, q, p, 3)
    octx = oracle_mod.Ctx(log_n, 3, 2)
    n = 1 << log_n
    mods = q + p
    a = _rand_limbs(mods, n, 100 + log_n)
    t = _dev(a)
    ks.ckks_ntt_fwd(ctx, t, 0, 5)
    f = _host(t)
    assert np.array_equal(f, octx.ntt_fwd(a, 0))
    ks.ckks_ntt_inv(ctx, t, 0, 5)
    assert np.array_equal(_host(t), a)
    # a sub-range starting at a special prime
    b = _rand_limbs(mods[3:], n, 7)
    t = _dev(b)
    ks.ckks_ntt_inv(ctx, t, 3, 2)
    assert np.array_equal(_host(t), octx.ntt_inv(b, 3))
    # edge inputs: all zero, all q-1
    z = np.zeros((5, n), dtype=np.uint32)
    t = _dev(z)
    ks.ckks_ntt_fwd(ctx, t, 0, 5)
    assert not _host(t).any()
    m1 = np.stack([np.full(n, m - 1, dtype=np.uint32) for m in mods])
    t = _dev(m1)
    ks.ckks_ntt_fwd(ctx, t, 0, 5)
    assert np.array_equal(_host(t), octx.ntt_fwd(m1, 0))


def test_automorph_parity(ks_lib, oracle_mod):
    ks = ks_lib
    s = setup_for(ks, "n14-hoisted8")
    n = s.cfg.n
    a = _rand_limbs(s.sc.ctx.q[:3], n, 3)
    out = torch.empty_like(_dev(a))
    for g in [5, ks.galois_element(14, -1), 2 * n - 1, 3]:
        ks.ckks_automorph(s.ctx, _dev(a), out, 3, g)
        assert np.array_equal(_host(out), s.sc.ctx.automorph_eval(a, g))


def test_chacha_expand_parity(ks_lib):
    ks = ks_lib
    s = setup_for(ks, "n16-full")
    out = torch.empty(s.cfg.n, dtype=torch.uint32, device="cuda")
    for (kid, j, t) in [(0, 0, 0), (5, 2, 47), (2**32 - 1, 1, 36)]:
        ks.ckks_chacha_expand(s.ctx, s.cfg.chacha_seed, kid, j, t, out)
        assert np.array_equal(_host(out), s.sc.ctx.chacha_expand(s.cfg.chacha_seed, kid, j, t))


# ----------------------------------------------------------------------------- steps

@pytest.mark.parametrize("key,level", [("n12-dnum2", 3), ("n12-dnum2", 0), ("n12-dnum4", 2), ("n14-hoisted8", 11), ("n14-hoisted8", 6), ("n16-full", 35), ("n16-bsgs32", 24), ("n16-stream64", 20)])
def test_modup_parity(ks_lib, key, level):
    ks = ks_lib
    s = setup_for(ks, key)
    n, na = s.cfg.n, level + 1
    c = _rand_limbs(s.sc.ctx.q[:na], n, 11 + level)
    beta = -(-na // s.cfg.alpha)
    ext = na + s.cfg.n_p
    dt = torch.empty((beta, ext, n), dtype=torch.uint32, device="cuda")
    ws = s.ctx.workspace(level)
    ks.ckks_modup(s.ctx, _dev(c), level, dt, ws)
    assert np.array_equal(_host(dt), s.sc.ctx.modup(c, level, s.cfg.alpha))


@pytest.mark.parametrize("key,level", [("n12-dnum2", 3), ("n14-hoisted8", 11), ("n14-hoisted8", 4), ("n16-full", 35), ("n16-stream64", 20)])
def test_inner_product_parity(ks_lib, key, level):
    ks = ks_lib
    s = setup_for(ks, key)
    n, na = s.cfg.n, level + 1
    beta = -(-na // s.cfg.alpha)
    ext = na + s.cfg.n_p
    ext_mods = [s.sc.ctx.mod[t] for t in s.sc.ctx.ext_limbs(level)]
    dt = np.stack([_rand_limbs(ext_mods, n, 40 + j) for j in range(beta)])
    g = s.sc.galois(1)
    for stored in (False, True):
        b, kb, ka, evk = s.key(g, stored_a=stored)
        acc = torch.empty((2, ext, n), dtype=torch.uint32, device="cuda")
        ks.ckks_inner_product(s.ctx, _dev(dt), level, evk, acc)
        a0, a1 = s.sc.ctx.inner_product(dt, level, s.cfg.alpha, b, s.cfg.chacha_seed, g)
        got = _host(acc)
        assert np.array_equal(got[0], a0) and np.array_equal(got[1], a1)


@pytest.mark.parametrize("key,level", [("n12-dnum2", 3), ("n14-hoisted8", 11), ("n16-full", 35), ("n16-full", 0), ("n16-stream64", 20)])
def test_moddown_parity(ks_lib, key, level):
    ks = ks_lib
    s = setup_for(ks, key)
    n, na = s.cfg.n, level + 1
    ext_mods = [s.sc.ctx.mod[t] for t in s.sc.ctx.ext_limbs(level)]
    acc = _rand_limbs(ext_mods, n, 77)
    out = torch.empty((na, n), dtype=torch.uint32, device="cuda")
    ws = s.ctx.workspace(level)
    ks.ckks_moddown(s.ctx, _dev(acc), level, out, ws)
    assert np.array_equal(_host(out), s.sc.ctx.moddown(acc, level))


def test_tensor_parity(ks_lib):
    ks = ks_lib
    s = setup_for(ks, "n14-hoisted8")
    _, x = s.sc.ciphertext(0)
    _, y = s.sc.ciphertext(1)
    d = torch.empty((3,) + x.shape[1:], dtype=torch.uint32, device="cuda")
    ks.ckks_tensor(s.ctx, _dev(x), _dev(y), s.cfg.level, d)
    assert np.array_equal(_host(d), s.sc.ctx.tensor(x, y, s.cfg.level))


# ----------------------------------------------------------------------------- composites

@pytest.mark.parametrize("key", ["n12-dnum2", "n12-dnum4", "n14-hoisted8", "n16-full"])
def test_rotate_relin_parity(ks_lib, key):
    ks = ks_lib
    s = setup_for(ks, key)
    cfg, lvl = s.cfg, s.cfg.level
    z, ct = s.sc.ciphertext(0)
    ws = s.ctx.workspace(lvl)
    out = torch.empty((2, lvl + 1, cfg.n), dtype=torch.uint32, device="cuda")
    r = cfg.rot_steps[0]
    g = s.sc.galois(r)
    b, kb, _, evk = s.key(g)
    ks.ckks_rotate(s.ctx, _dev(ct), lvl, g, evk, out, ws)
    assert np.array_equal(_host(out), s.sc.ctx.rotate(ct, lvl, cfg.alpha, g, b, cfg.chacha_seed, g))
    # relinearisation of a tensor product
    _, y = s.sc.ciphertext(1)
    d = s.sc.ctx.tensor(ct, y, lvl)
    b0, kb0, _, evk0 = s.key(0)
    ks.ckks_relin(s.ctx, _dev(d), lvl, evk0, out, ws)
    assert np.array_equal(_host(out), s.sc.ctx.relin(d, lvl, cfg.alpha, b0, cfg.chacha_seed, 0))
    # bare key switch of c1
    ks.ckks_keyswitch(s.ctx, _dev(ct[1]), lvl, evk0, out, ws)
    assert np.array_equal(_host(out), s.sc.ctx.keyswitch(ct[1], lvl, cfg.alpha, b0, cfg.chacha_seed, 0))


def test_stored_a_ablation_parity(ks_lib):
    ks = ks_lib
    s = setup_for(ks, "n14-hoisted8")
    lvl = s.cfg.level
    _, ct = s.sc.ciphertext(0)
    g = s.sc.galois(1)
    b, kb, ka, evk = s.key(g, stored_a=True)
    out = torch.empty((2, lvl + 1, s.cfg.n), dtype=torch.uint32, device="cuda")
    ks.ckks_rotate(s.ctx, _dev(ct), lvl, g, evk, out, s.ctx.workspace(lvl))
    assert np.array_equal(_host(out), s.sc.ctx.rotate(ct, lvl, s.cfg.alpha, g, b, s.cfg.chacha_seed, g))


@pytest.mark.parametrize("key,steps", [("n12-dnum2", (1, -1, 2)), ("n12-dnum4", (1, -1, 3)), ("n14-hoisted8", W.CONFIGS["n14-hoisted8"].rot_steps)])
def test_hoisted_parity(ks_lib, key, steps):
    ks = ks_lib
    s = setup_for(ks, key)
    cfg, lvl = s.cfg, s.cfg.level
    _, ct = s.sc.ciphertext(0)
    gs = [s.sc.galois(r) for r in steps]
    keys = [s.key(g) for g in gs]
    out = torch.empty((len(gs), 2, lvl + 1, cfg.n), dtype=torch.uint32, device="cuda")
    ks.ckks_rotate_hoisted(s.ctx, _dev(ct), lvl, gs, [k[3] for k in keys], out, s.ctx.workspace(lvl, len(gs)))
    want = s.sc.ctx.rotate_hoisted(ct, lvl, cfg.alpha, gs, [k[0] for k in keys], [cfg.chacha_seed] * len(gs), gs)
    assert np.array_equal(_host(out), want)


def test_n16_bsgs32_hoisted_sampled(ks_lib):
    """n16-bsgs32 (32 hoisted rotations at level 24, dnum 4): the GPU runs the full batch of 32;
    the oracle recomputes a sample of 3 rotations (each output depends only on its own key)."""
    ks = ks_lib
    s = setup_for(ks, "n16-bsgs32")
    cfg, lvl = s.cfg, s.cfg.level
    _, ct = s.sc.ciphertext(0)
    gs = [s.sc.galois(r) for r in cfg.rot_steps]
    keys = [s.key(g) for g in gs]
    out = torch.empty((len(gs), 2, lvl + 1, cfg.n), dtype=torch.uint32, device="cuda")
    ks.ckks_rotate_hoisted(s.ctx, _dev(ct), lvl, gs, [k[3] for k in keys], out, s.ctx.workspace(lvl, len(gs)))
    got = _host(out)
    for i in (0, 15, 31):
        want = s.sc.ctx.rotate(ct, lvl, cfg.alpha, gs[i], keys[i][0], cfg.chacha_seed, gs[i])
        assert np.array_equal(got[i], want)


def test_n16_stream64_pipeline_sampled(ks_lib):
    """n16-stream64 (tensor + relin + rotate by 2^(i mod 15) at level 20, dnum 4) on a sample of
    pairs; every pair is independent."""
    ks = ks_lib
    s = setup_for(ks, "n16-stream64")
    cfg, lvl = s.cfg, s.cfg.level
    ws = s.ctx.workspace(lvl)
    na = lvl + 1
    b0, _, _, evk0 = s.key(0)
    for i in (0, 14):
        _, x = s.sc.ciphertext(2 * i)
        _, y = s.sc.ciphertext(2 * i + 1)
        g = s.sc.galois(cfg.rot_steps[i])
        b, _, _, evk = s.key(g)
        d = torch.empty((3, na, cfg.n), dtype=torch.uint32, device="cuda")
        r1 = torch.empty((2, na, cfg.n), dtype=torch.uint32, device="cuda")
        r2 = torch.empty_like(r1)
        ks.ckks_tensor(s.ctx, _dev(x), _dev(y), lvl, d)
        ks.ckks_relin(s.ctx, d, lvl, evk0, r1, ws)
        ks.ckks_rotate(s.ctx, r1, lvl, g, evk, r2, ws)
        od = s.sc.ctx.tensor(x, y, lvl)
        o1 = s.sc.ctx.relin(od, lvl, cfg.alpha, b0, cfg.chacha_seed, 0)
        o2 = s.sc.ctx.rotate(o1, lvl, cfg.alpha, g, b, cfg.chacha_seed, g)
        assert np.array_equal(_host(r2), o2)


@pytest.mark.parametrize("dnum", [1, 36])
def test_extreme_dnum(ks_lib, oracle_mod, dnum):
    """dnum = 1 (one digit of 36 primes) and dnum = L+1 (one prime per digit) at N=2^12."""
    ks = ks_lib
    log_n, n_q, n_p = 12, 36, 12 if dnum == 36 else 24
    q, p = ks.ckks_gen_primes(log_n, n_q, n_p)
    octx = oracle_mod.Ctx(log_n, n_q, n_p)
    alpha = -(-n_q // dnum)
    ctx = ks.Context(log_n, q, p, dnum)
    n = 1 << log_n
    for level in (35, 17):
        c = _rand_limbs(q[: level + 1], n, 5 + level)
        beta = -(-(level + 1) // alpha)
        ext = level + 1 + n_p
        dt = torch.empty((beta, ext, n), dtype=torch.uint32, device="cuda")
        ks.ckks_modup(ctx, _dev(c), level, dt, ctx.workspace(level))
        assert np.array_equal(_host(dt), octx.modup(c, level, alpha))
        acc = _rand_limbs([octx.mod[t] for t in octx.ext_limbs(level)], n, 9)
        out = torch.empty((level + 1, n), dtype=torch.uint32, device="cuda")
        ks.ckks_moddown(ctx, _dev(acc), level, out, ctx.workspace(level))
        assert np.array_equal(_host(out), octx.moddown(acc, level))


def test_extreme_dnum_batch(ks_lib, oracle_mod):
    """dnum = 1: both base conversions use the generic kernel (digit of 36 primes, 24 special
    primes).  A batch of 3 key switches with distinct keys equals the single calls, and item 0
    equals the oracle."""
    ks = ks_lib
    log_n, n_q, n_p, dnum = 12, 36, 24, 1
    q, p = ks.ckks_gen_primes(log_n, n_q, n_p)
    octx = oracle_mod.Ctx(log_n, n_q, n_p)
    ctx = ks.Context(log_n, q, p, dnum)
    n, items = 1 << log_n, 3
    seed = bytes(range(32))
    for level in (35, 17):
        keys = [_rand_limbs(q + p, n, 40 + 3 * level + i).reshape(1, n_q + n_p, n) for i in range(items)]
        evks = [ks.make_evk(_dev(k), seed, 3 + 2 * i) for i, k in enumerate(keys)]
        c = np.stack([_rand_limbs(q[: level + 1], n, 60 + 3 * level + i) for i in range(items)])
        out = torch.empty((items, 2, level + 1, n), dtype=torch.uint32, device="cuda")
        ks.ckks_keyswitch_batch(ctx, _dev(c), level, evks, out, ctx.workspace(level, items))
        got = _host(out)
        one = torch.empty((2, level + 1, n), dtype=torch.uint32, device="cuda")
        for i in range(items):
            ks.ckks_keyswitch(ctx, _dev(c[i]), level, evks[i], one, ctx.workspace(level))
            assert np.array_equal(_host(one), got[i]), (level, i)
        assert np.array_equal(got[0], octx.keyswitch(c[0], level, n_q, keys[0], seed, 3))


def test_error_codes(ks_lib):
    ks = ks_lib
    s = setup_for(ks, "n12-dnum2")
    lvl, n = s.cfg.level, s.cfg.n
    ct = torch.zeros((2, lvl + 1, n), dtype=torch.uint32, device="cuda")
    out = torch.empty_like(ct)
    ws = s.ctx.workspace(lvl)
    _, _, _, evk = s.key(0)
    with pytest.raises(ks.CkksError) as e:
        ks.ckks_relin(s.ctx, ct, lvl, evk, out, ws[: ws.numel() // 2])
    assert e.value.code == ks.CKKS_ERR_WORKSPACE
    with pytest.raises(ks.CkksError) as e:
        ks.ckks_keyswitch(s.ctx, ct.view(-1)[1:], lvl, evk, out, ws)
    assert e.value.code == ks.CKKS_ERR_ALIGN
    with pytest.raises(ks.CkksError) as e:
        ks.ckks_keyswitch(s.ctx, ct, lvl + 1, evk, out, ws)
    assert e.value.code == ks.CKKS_ERR_UNSUPPORTED
    with pytest.raises(ks.CkksError) as e:
        ks.ckks_rotate(s.ctx, ct, lvl, 4, evk, out, ws)
    assert e.value.code == ks.CKKS_ERR_ARG
    assert ks.ckks_sync_status(s.ctx, None, 5000) == ks.CKKS_OK
