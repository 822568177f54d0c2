"""GPU parity for the baby-step giant-step linear transform with double hoisting (ckks_bsgs),
through the C ABI, against the CPU oracle, bit for bit."""
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
        self.keys = {}

    def key(self, g):
        if g == 1:
            return None, None
        if g not in self.keys:
            b = self.sc.key(g)
            kb = _dev(b)
            self.keys[g] = (b, kb, self.ks.make_evk(kb, self.cfg.chacha_seed, g))
        b, _, evk = self.keys[g]
        return (b, g), evk

    def rand_pt(self, level, n_giant, n_baby, seed):
        ctx = self.sc.ctx
        mods = ctx.q[: level + 1] + ctx.p
        ext = len(mods)
        return np.stack([W.uniform_residues(mods, self.cfg.n, W.rng(seed, W.TAG_SYNTH, j, k))
                         for j in range(n_giant) for k in range(n_baby)]).reshape(n_giant, n_baby, ext, self.cfg.n)

    def run(self, baby, giant, pt, ct, level):
        ks = self.ks
        ob = [self.key(g) for g in baby]
        og = [self.key(g) for g in giant]
        out = torch.empty((2, level + 1, self.cfg.n), dtype=torch.uint32, device="cuda")
        ws = ks.ckks_bsgs_workspace(self.ctx, level, len(baby), len(giant))
        ks.ckks_bsgs(self.ctx, _dev(ct), level, baby, [e for _, e in ob], giant, [e for _, e in og], _dev(pt),
                     out, ws)
        got = _host(out)
        want = self.sc.ctx.bsgs(ct, level, self.cfg.alpha, baby, [k for k, _ in ob], giant, [k for k, _ in og],
                                pt, self.cfg.chacha_seed)
        return got, want


_S = {}


def setup_for(ks, key):
    if key not in _S:
        _S[key] = Setup(ks, key)
    return _S[key]


def test_bsgs_parity_small(ks_lib):
    s = setup_for(ks_lib, "n12-dnum4")
    lvl = s.cfg.level
    baby = [1] + [s.sc.galois(k) for k in (1, 2, 3)]
    giant = [1, s.sc.galois(4), s.sc.galois(8)]
    _, ct = s.sc.ciphertext(0)
    got, want = s.run(baby, giant, s.rand_pt(lvl, 3, 4, 11), ct, lvl)
    assert np.array_equal(got, want)


def test_bsgs_parity_two_primes_per_digit(ks_lib):
    """n12-dnum2: dnum 2 (two primes per digit) and a single special prime."""
    s = setup_for(ks_lib, "n12-dnum2")
    lvl = s.cfg.level
    baby = [1, s.sc.galois(1)]
    giant = [1, s.sc.galois(2)]
    _, ct = s.sc.ciphertext(0)
    got, want = s.run(baby, giant, s.rand_pt(lvl, 2, 2, 15), ct, lvl)
    assert np.array_equal(got, want)


def test_evk_keeps_its_tensors_alive(ks_lib):
    """A key record made from a temporary tensor keeps that device memory allocated."""
    import gc
    ks = ks_lib
    s = setup_for(ks_lib, "n12-dnum2")
    lvl, g = s.cfg.level, s.sc.galois(1)
    b = s.sc.key(g)
    evk = ks.make_evk(_dev(b), s.cfg.chacha_seed, g)      # no other reference to the tensor
    gc.collect()
    junk = [torch.full((b.size,), 7, dtype=torch.int32, device="cuda") for _ in range(4)]
    _, ct = s.sc.ciphertext(0)
    out = torch.empty((2, lvl + 1, s.cfg.n), dtype=torch.uint32, device="cuda")
    ks.ckks_rotate(s.ctx, _dev(ct), lvl, g, evk, out, s.ctx.workspace(lvl))
    assert np.array_equal(_host(out), s.sc.ctx.rotate(ct, lvl, s.cfg.alpha, g, b, s.cfg.chacha_seed, g))
    del junk


def test_bsgs_parity_identity_in_the_middle(ks_lib):
    """Identity steps at any position (the giant rotations then run as two batches)."""
    s = setup_for(ks_lib, "n14-hoisted8")
    lvl = s.cfg.level
    baby = [s.sc.galois(1), s.sc.galois(2), 1, s.sc.galois(3)]
    giant = [s.sc.galois(4), 1, s.sc.galois(8)]
    _, ct = s.sc.ciphertext(0)
    got, want = s.run(baby, giant, s.rand_pt(lvl, 3, 4, 12), ct, lvl)
    assert np.array_equal(got, want)


def test_bsgs_parity_more_than_16_babies(ks_lib):
    """20 baby steps: the plaintext sums run in two launches, carrying partial sums."""
    s = setup_for(ks_lib, "n12-dnum4")
    lvl = s.cfg.level
    baby = [1] + [s.sc.galois(k) for k in range(1, 20)]
    giant = [1, s.sc.galois(20)]
    _, ct = s.sc.ciphertext(1)
    got, want = s.run(baby, giant, s.rand_pt(lvl, 2, 20, 13), ct, lvl)
    assert np.array_equal(got, want)


def test_bsgs_decode(ks_lib):
    """Encoded diagonals: the GPU result decodes to sum_i d_i * rot_i(z)."""
    from oracle import encode
    s = setup_for(ks_lib, "n14-hoisted8")
    sc, ctx, lvl, n = s.sc, s.sc.ctx, s.cfg.level, s.cfg.n
    z, ct = sc.ciphertext(0)
    n1, n2 = 4, 3
    baby = [sc.galois(k) if k else 1 for k in range(n1)]
    giant = [sc.galois(n1 * j) if j else 1 for j in range(n2)]
    rng = np.random.default_rng(7)
    d = rng.uniform(-1, 1, (n1 * n2, n // 2)) + 1j * rng.uniform(-1, 1, (n1 * n2, n // 2))
    limbs = list(range(lvl + 1)) + list(range(ctx.n_q, ctx.n_q + ctx.n_p))
    pt = np.stack([ctx.signed_to_eval(encode(np.roll(d[n1 * j + k], n1 * j), n, 2.0 ** 20), limbs)
                   for j in range(n2) for k in range(n1)]).reshape(n2, n1, len(limbs), n)
    got, want = s.run(baby, giant, pt, ct, lvl)
    assert np.array_equal(got, want)
    ref = sum(d[i] * np.roll(z, -i) for i in range(n1 * n2))
    assert np.abs(sc.decrypt_slots(got, scale=sc.scale * 2.0 ** 20) - ref).max() < 2.0 ** -7.5


@pytest.mark.slow
def test_bsgs_parity_n16_bsgs32_full(ks_lib):
    """n16-bsgs32's 32 rotation keys as one transform: baby steps 0..15, giant steps 16 j for
    j = 0..17 (288 diagonals), level 24, random plaintexts over the extended basis."""
    s = setup_for(ks_lib, "n16-bsgs32")
    lvl = s.cfg.level
    baby = [1] + [s.sc.galois(k) for k in range(1, 16)]
    giant = [1] + [s.sc.galois(16 * j) for j in range(1, 18)]
    _, ct = s.sc.ciphertext(0)
    got, want = s.run(baby, giant, s.rand_pt(lvl, 18, 16, 14), ct, lvl)
    assert np.array_equal(got, want)


def test_bsgs_errors(ks_lib):
    ks = ks_lib
    s = setup_for(ks, "n12-dnum2")
    lvl, n = s.cfg.level, s.cfg.n
    ct = torch.zeros((2, lvl + 1, n), dtype=torch.uint32, device="cuda")
    out = torch.empty_like(ct)
    pt = torch.zeros((1, 2, lvl + 1 + s.cfg.n_p, n), dtype=torch.uint32, device="cuda")
    g = s.sc.galois(1)
    _, evk = s.key(g)
    ws = ks.ckks_bsgs_workspace(s.ctx, lvl, 2, 1)
    with pytest.raises(ks.CkksError) as e:
        ks.ckks_bsgs(s.ctx, ct, lvl, [1, 4], [None, evk], [1], [None], pt, out, ws)     # even element
    assert e.value.code == ks.CKKS_ERR_ARG
    with pytest.raises(ks.CkksError) as e:
        ks.ckks_bsgs(s.ctx, ct, lvl, [1, g], [None, evk], [1], [None], pt, ct, ws)      # output = input
    assert e.value.code == ks.CKKS_ERR_ARG
    with pytest.raises(ks.CkksError) as e:
        ks.ckks_bsgs(s.ctx, ct, lvl, [1, g], [None, evk], [1], [None], pt, out, ws[:64])
    assert e.value.code == ks.CKKS_ERR_WORKSPACE
    with pytest.raises(ks.CkksError) as e:
        ks.ckks_bsgs(s.ctx, ct, lvl, [1, g], [None, evk], [1], [None], pt, out, ws[1:])
    assert e.value.code in (ks.CKKS_ERR_ALIGN, ks.CKKS_ERR_WORKSPACE)
    assert ks.ckks_sync_status(s.ctx, None, 5000) == ks.CKKS_OK
