"""Degenerate and empty cases of the C ABI on the GPU, against exact expectations."""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _dev(a: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint32)).cuda()


@pytest.fixture(scope="module")
def setup(ks_lib):
    from oracle.scenario import Scenario
    ks = ks_lib
    cfg = W.CONFIGS["n12-dnum2"]
    sc = Scenario(cfg)
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    return ks, cfg, sc, ks.Context(cfg.log_n, q, p, cfg.dnum)


def test_empty_batches_do_nothing(setup):
    ks, cfg, sc, ctx = setup
    lvl, n = cfg.level, cfg.n
    buf = torch.full((2, lvl + 1, n), 7, dtype=torch.uint32, device="cuda")
    out = torch.full((2, lvl + 1, n), 9, dtype=torch.uint32, device="cuda")
    ws = ctx.workspace(lvl)
    ks.ckks_keyswitch_batch(ctx, buf, lvl, [], out, ws)
    ks.ckks_rotate_batch(ctx, buf, lvl, [], [], out, ws)
    ks.ckks_relin_batch(ctx, buf, lvl, [], out, ws)
    ks.ckks_tensor_batch(ctx, 0, buf, buf, lvl, out)
    ks.ckks_rescale_batch(ctx, 0, buf, lvl, out, ws)
    ks.ckks_rotate_hoisted(ctx, buf, lvl, [], [], out, ws)
    assert ks.ckks_sync_status(ctx, None, 5000) == ks.CKKS_OK
    assert bool((out == 9).all())


def test_rotation_by_the_identity(setup):
    """g = 1: kappa_1 is the identity, so the rotation is the key switch of c1 plus c0."""
    ks, cfg, sc, ctx = setup
    lvl = cfg.level
    _, ct = sc.ciphertext(0)
    b = sc.key(0)                                          # any key: the identity uses key_id 1 here
    kb = _dev(b)
    evk = ks.make_evk(kb, cfg.chacha_seed, 1)
    out = torch.empty((2, lvl + 1, cfg.n), dtype=torch.uint32, device="cuda")
    ks_out = torch.empty_like(out)
    ws = ctx.workspace(lvl)
    ks.ckks_rotate(ctx, _dev(ct), lvl, 1, evk, out, ws)
    ks.ckks_keyswitch(ctx, _dev(ct[1]), lvl, evk, ks_out, ws)
    torch.cuda.synchronize()
    mods = np.array(sc.ctx.q[: lvl + 1], dtype=np.uint64)[:, None]
    want = ks_out.cpu().numpy().astype(np.uint64)
    want[0] = (want[0] + ct[0].astype(np.uint64)) % mods
    assert np.array_equal(out.cpu().numpy(), want.astype(np.uint32))
    assert np.array_equal(out.cpu().numpy(), sc.ctx.rotate(ct, lvl, cfg.alpha, 1, b, cfg.chacha_seed, 1))


def test_bsgs_identity_returns_the_input(setup):
    """One identity baby, one identity giant, plaintext 1: ModDown(P c) = c exactly."""
    ks, cfg, sc, ctx = setup
    lvl = cfg.level
    _, ct = sc.ciphertext(1)
    ext = lvl + 1 + cfg.n_p
    pt = torch.ones((1, 1, ext, cfg.n), dtype=torch.uint32, device="cuda")
    out = torch.empty((2, lvl + 1, cfg.n), dtype=torch.uint32, device="cuda")
    ws = ks.ckks_bsgs_workspace(ctx, lvl, 1, 1)
    ks.ckks_bsgs(ctx, _dev(ct), lvl, [1], [None], [1], [None], pt, out, ws)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), ct)
