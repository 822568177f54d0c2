"""Failure paths, each made without faulting the GPU, after which the context keeps producing
correct results:
- a bounded device wait that expires (an mbarrier that never completes, a self-test kernel of
  the library) is reported by ckks_sync_status as CKKS_ERR_TIMEOUT and cleared;
- a launch the CUDA runtime rejects on the host (an invalid block size) is reported as
  CKKS_ERR_CUDA with the runtime's message, and leaves no sticky error behind."""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _rotation_still_exact(ks, ctx, cfg, sc):
    lvl = cfg.level
    g = sc.galois(1)
    b = sc.key(g)
    evk = ks.make_evk(torch.from_numpy(b).cuda(), cfg.chacha_seed, g)
    _, ct = sc.ciphertext(0)
    out = torch.empty((2, lvl + 1, cfg.n), dtype=torch.uint32, device="cuda")
    ks.ckks_rotate(ctx, torch.from_numpy(ct).cuda(), lvl, g, evk, out, ctx.workspace(lvl))
    assert ks.ckks_sync_status(ctx, None, 5000) == ks.CKKS_OK
    assert np.array_equal(out.cpu().numpy(), sc.ctx.rotate(ct, lvl, cfg.alpha, g, b, cfg.chacha_seed, g))


def test_launch_error_is_reported_and_context_survives(ks_lib):
    from oracle.scenario import Scenario
    ks = ks_lib
    cfg = W.CONFIGS["n12-dnum2"]
    sc = Scenario(cfg)
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    assert ks.ckks_selftest_launch_error(ctx) == ks.CKKS_ERR_CUDA
    assert "ckks_selftest_launch_error" in ks.ckks_last_error()
    assert ks.ckks_sync_status(ctx, None, 5000) == ks.CKKS_OK           # not sticky
    _rotation_still_exact(ks, ctx, cfg, sc)


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
