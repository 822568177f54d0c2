"""Allocation-free key switching: ckks_keyswitch_noalloc against ckks_keyswitch.

Some callers of this library cannot allocate device memory themselves: their host framework
owns every device allocation (a serving runtime with its own memory pool), or the call sits in
a latency-critical loop where a cudaMalloc, which may synchronise the device, is not allowed.
For them the library has one key-switch entry point that keeps its workspace in a fixed array
of the library's own device memory instead of a caller buffer.  These tests call it through
the C ABI twice in a row and require the same bits as the ordinary entry point and as the CPU
oracle each time (integer RNS arithmetic: the tolerance is exact equality), check that a call
leaves the device's allocated and free memory unchanged, and check that a parameter set whose
workspace does not fit is refused with a clear error.
"""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _residues(moduli, n, gen):
    return torch.from_numpy(W.uniform_residues(moduli, n, gen)).cuda()


@pytest.mark.parametrize("key", ["n12-dnum2", "n14-hoisted8"])
def test_noalloc_matches_keyswitch_twice(ks_lib, oracle_mod, key):
    ks = ks_lib
    cfg = W.CONFIGS[key]
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    lvl = cfg.level
    assert ctx.workspace_bytes(lvl) <= ks.NOALLOC_SCRATCH_BYTES
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 4242)
    n_digits = -(-cfg.n_q // cfg.alpha)
    b = _residues((q + p) * n_digits, cfg.n, gen)          # a key's stored half (synthetic)
    evk = ks.make_evk(b, cfg.chacha_seed, ks.galois_element(cfg.log_n, 1))
    ws = ctx.workspace(lvl)
    octx = oracle_mod.Ctx(cfg.log_n, cfg.n_q, cfg.n_p)
    g = ks.galois_element(cfg.log_n, 1)
    for _ in range(2):
        c = _residues(q[: lvl + 1], cfg.n, gen)
        want = torch.empty((2, lvl + 1, cfg.n), dtype=torch.uint32, device="cuda")
        got = torch.full_like(want, 0xFFFFFFFF)
        ks.ckks_keyswitch(ctx, c, lvl, evk, want, ws)
        ks.ckks_keyswitch_noalloc(ctx, c, lvl, evk, got)
        torch.cuda.synchronize()
        assert np.array_equal(got.cpu().numpy(), want.cpu().numpy())
        oracle = octx.keyswitch(c.cpu().numpy(), lvl, cfg.alpha, b.cpu().numpy(), cfg.chacha_seed, g)
        assert np.array_equal(got.cpu().numpy(), oracle)


def test_noalloc_allocates_nothing(ks_lib):
    """After a first call (which loads the kernels it uses), a second call on a non-default stream
    changes neither PyTorch's allocated bytes nor the device's free memory."""
    ks = ks_lib
    cfg = W.CONFIGS["n14-hoisted8"]
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    lvl = cfg.level
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 4343)
    n_digits = -(-cfg.n_q // cfg.alpha)
    b = _residues((q + p) * n_digits, cfg.n, gen)
    evk = ks.make_evk(b, cfg.chacha_seed, 0)
    c = _residues(q[: lvl + 1], cfg.n, gen)
    out = torch.empty((2, lvl + 1, cfg.n), dtype=torch.uint32, device="cuda")
    side = torch.cuda.Stream()
    ks.ckks_keyswitch_noalloc(ctx, c, lvl, evk, out, side)
    torch.cuda.synchronize()
    alloc0, free0 = torch.cuda.memory_allocated(), torch.cuda.mem_get_info()[0]
    ks.ckks_keyswitch_noalloc(ctx, c, lvl, evk, out, side)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == alloc0
    assert torch.cuda.mem_get_info()[0] == free0


def test_noalloc_rejects_oversized(ks_lib):
    ks = ks_lib
    cfg = W.CONFIGS["n16-full"]
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    assert ctx.workspace_bytes(cfg.level) > ks.NOALLOC_SCRATCH_BYTES
    c = torch.zeros((cfg.level + 1, cfg.n), dtype=torch.uint32, device="cuda")
    out = torch.empty((2, cfg.level + 1, cfg.n), dtype=torch.uint32, device="cuda")
    b = torch.zeros((3, cfg.n_q + cfg.n_p, cfg.n), dtype=torch.uint32, device="cuda")
    evk = ks.make_evk(b, cfg.chacha_seed, 0)
    with pytest.raises(ks.CkksError) as e:
        ks.ckks_keyswitch_noalloc(ctx, c, cfg.level, evk, out)
    assert e.value.code == ks.CKKS_ERR_WORKSPACE
    assert "fixed" in str(e.value)
