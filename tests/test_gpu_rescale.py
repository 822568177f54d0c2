"""GPU parity for rescale (ckks_rescale, ckks_rescale_batch) and conjugation (ckks_rotate with
g = 2N - 1), through the C ABI, against the CPU oracle, bit for bit."""
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


class Setup:
    def __init__(self, ks, key):
        from oracle.scenario import Scenario
        self.ks, self.cfg = ks, W.CONFIGS[key]
        self.sc = Scenario(self.cfg)
        q, p = ks.ckks_gen_primes(self.cfg.log_n, self.cfg.n_q, self.cfg.n_p)
        assert q == self.sc.ctx.q and p == self.sc.ctx.p
        self.ctx = ks.Context(self.cfg.log_n, q, p, self.cfg.dnum)

    def rand_ct(self, level, seed, n_items=None):
        shape = (2,) if n_items is None else (n_items, 2)
        count = int(np.prod(shape))
        a = W.uniform_residues(self.sc.ctx.q[: level + 1] * count, self.cfg.n, W.rng(seed, W.TAG_SYNTH, level))
        return a.reshape(*shape, level + 1, self.cfg.n)

    def evk(self, key_id):
        b = self.sc.key(key_id)
        kb = _dev(b)
        return b, kb, self.ks.make_evk(kb, self.cfg.chacha_seed, key_id)


_S = {}


def setup_for(ks, key):
    if key not in _S:
        _S[key] = Setup(ks, key)
    return _S[key]


@pytest.mark.parametrize("key,level", [("n12-dnum2", 3), ("n12-dnum2", 1), ("n14-hoisted8", 11), ("n14-hoisted8", 5), ("n16-full", 35), ("n16-full", 1), ("n16-stream64", 20)])
def test_rescale_parity(ks_lib, key, level):
    ks = ks_lib
    s = setup_for(ks, key)
    ct = s.rand_ct(level, 500 + level)
    out = torch.empty((2, level, s.cfg.n), dtype=torch.uint32, device="cuda")
    ws = s.ctx.workspace(level)
    ks.ckks_rescale(s.ctx, _dev(ct), level, out, ws)
    assert np.array_equal(_host(out), s.sc.ctx.rescale(ct, level))


@pytest.mark.parametrize("key,level,n", [("n14-hoisted8", 11, 3), ("n12-dnum2", 2, 66)])
def test_rescale_batch_parity(ks_lib, key, level, n):
    """Every item equals the oracle; 66 items cross the 64-item launch chunk."""
    ks = ks_lib
    s = setup_for(ks, key)
    ct = s.rand_ct(level, 900 + n, n_items=n)
    out = torch.empty((n, 2, level, s.cfg.n), dtype=torch.uint32, device="cuda")
    ws = s.ctx.workspace(level, n)
    ks.ckks_rescale_batch(s.ctx, n, _dev(ct), level, out, ws)
    got = _host(out)
    for z in range(n):
        assert np.array_equal(got[z], s.sc.ctx.rescale(ct[z], level)), z


@pytest.mark.parametrize("key", ["n12-dnum4", "n14-hoisted8"])
def test_mul_relin_rescale_chain(ks_lib, key):
    """tensor -> relin -> rescale on the GPU equals the oracle chain and decodes to z1*z2."""
    ks = ks_lib
    s = setup_for(ks, key)
    lvl, n = s.cfg.level, s.cfg.n
    z1, x = s.sc.ciphertext(0)
    z2, y = s.sc.ciphertext(1)
    d = torch.empty((3, lvl + 1, n), dtype=torch.uint32, device="cuda")
    r = torch.empty((2, lvl + 1, n), dtype=torch.uint32, device="cuda")
    out = torch.empty((2, lvl, n), dtype=torch.uint32, device="cuda")
    ws = s.ctx.workspace(lvl)
    b0, _, evk0 = s.evk(0)
    ks.ckks_tensor(s.ctx, _dev(x), _dev(y), lvl, d)
    ks.ckks_relin(s.ctx, d, lvl, evk0, r, ws)
    ks.ckks_rescale(s.ctx, r, lvl, out, ws)
    oc = s.sc.ctx
    want = oc.rescale(oc.relin(oc.tensor(x, y, lvl), lvl, s.cfg.alpha, b0, s.cfg.chacha_seed, 0), lvl)
    got = _host(out)
    assert np.array_equal(got, want)
    scale = s.sc.scale ** 2 / oc.mod[lvl]
    assert np.abs(s.sc.decrypt_slots(got, level=lvl - 1, scale=scale) - z1 * z2).max() < 2.0 ** -9


@pytest.mark.parametrize("key", ["n12-dnum4", "n14-hoisted8", "n16-full"])
def test_conjugation_parity(ks_lib, key):
    ks = ks_lib
    s = setup_for(ks, key)
    lvl, n = s.cfg.level, s.cfg.n
    g = ks.conjugation_element(s.cfg.log_n)
    assert g == 2 * n - 1
    z, ct = s.sc.ciphertext(0)
    b, _, evk = s.evk(g)
    out = torch.empty((2, lvl + 1, n), dtype=torch.uint32, device="cuda")
    ks.ckks_rotate(s.ctx, _dev(ct), lvl, g, evk, out, s.ctx.workspace(lvl))
    got = _host(out)
    assert np.array_equal(got, s.sc.ctx.rotate(ct, lvl, s.cfg.alpha, g, b, s.cfg.chacha_seed, g))
    if key != "n16-full":
        assert np.abs(s.sc.decrypt_slots(got) - np.conj(z)).max() < 2.0 ** -9.5


def test_conjugation_in_hoisted_batch(ks_lib):
    """Conjugation hoisted together with rotations equals the single calls."""
    ks = ks_lib
    s = setup_for(ks, "n14-hoisted8")
    lvl, n = s.cfg.level, s.cfg.n
    gs = [s.sc.galois(1), ks.conjugation_element(s.cfg.log_n), s.sc.galois(-2)]
    keys = [s.evk(g) for g in gs]
    _, ct = s.sc.ciphertext(0)
    dct = _dev(ct)
    out = torch.empty((3, 2, lvl + 1, n), dtype=torch.uint32, device="cuda")
    ws = s.ctx.workspace(lvl, 3)
    ks.ckks_rotate_hoisted(s.ctx, dct, lvl, gs, [k[2] for k in keys], out, ws)
    got = _host(out)
    for i, g in enumerate(gs):
        assert np.array_equal(got[i], s.sc.ctx.rotate(ct, lvl, s.cfg.alpha, g, keys[i][0], s.cfg.chacha_seed, g))


def test_rescale_errors(ks_lib):
    ks = ks_lib
    s = setup_for(ks, "n12-dnum2")
    lvl, n = s.cfg.level, s.cfg.n
    ct = torch.zeros((2, lvl + 1, n), dtype=torch.uint32, device="cuda")
    out = torch.empty((2, lvl, n), dtype=torch.uint32, device="cuda")
    ws = s.ctx.workspace(lvl)
    with pytest.raises(ks.CkksError) as e:
        ks.ckks_rescale(s.ctx, ct, 0, out, ws)
    assert e.value.code == ks.CKKS_ERR_ARG
    with pytest.raises(ks.CkksError) as e:
        ks.ckks_rescale(s.ctx, ct, lvl, ct, ws)                       # output overlaps input
    assert e.value.code == ks.CKKS_ERR_ARG
    with pytest.raises(ks.CkksError) as e:
        ks.ckks_rescale(s.ctx, ct, lvl, out, ws[:16])
    assert e.value.code == ks.CKKS_ERR_WORKSPACE
    with pytest.raises(ks.CkksError) as e:
        ks.ckks_rescale(s.ctx, ct, lvl + 1, out, ws)
    assert e.value.code == ks.CKKS_ERR_UNSUPPORTED
    with pytest.raises(ks.CkksError) as e:
        ks.ckks_rescale(s.ctx, ct.view(-1)[1:], lvl, out, ws)
    assert e.value.code == ks.CKKS_ERR_ALIGN
    assert ks.ckks_sync_status(s.ctx, None, 5000) == ks.CKKS_OK
