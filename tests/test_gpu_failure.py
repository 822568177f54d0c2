"""Failure path of bounded device waits: a wait that expires is reported by ckks_sync_status as
CKKS_ERR_TIMEOUT, the error is cleared, and the context keeps producing correct results.
The expiry is provoked by an mbarrier that never completes (a self-test kernel of the library);
nothing faults, traps or hangs."""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def test_wait_expiry_is_reported_and_context_survives(ks_lib):
    from oracle.scenario import Scenario
    ks = ks_lib
    cfg = W.CONFIGS["n12-dnum2"]
    sc = Scenario(cfg)
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    assert ks.ckks_sync_status(ctx, None, 5000) == ks.CKKS_OK
    ks.ckks_selftest_wait_expiry(ctx)
    assert ks.ckks_sync_status(ctx, None, 20000) == ks.CKKS_ERR_TIMEOUT
    assert ks.ckks_sync_status(ctx, None, 5000) == ks.CKKS_OK          # cleared
    # the context still computes bit-exact results
    lvl = cfg.level
    g = sc.galois(1)
    b = sc.key(g)
    kb = torch.from_numpy(b).cuda()
    evk = ks.make_evk(kb, cfg.chacha_seed, g)
    _, ct = sc.ciphertext(0)
    out = torch.empty((2, lvl + 1, cfg.n), dtype=torch.uint32, device="cuda")
    ks.ckks_rotate(ctx, torch.from_numpy(ct).cuda(), lvl, g, evk, out, ctx.workspace(lvl))
    assert ks.ckks_sync_status(ctx, None, 5000) == ks.CKKS_OK
    assert np.array_equal(out.cpu().numpy(), sc.ctx.rotate(ct, lvl, cfg.alpha, g, b, cfg.chacha_seed, g))
