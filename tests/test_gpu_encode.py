"""The library's encoder (ckks_encode) against the oracle's.

Both round the scaled inverse slot DFT half away from zero in double precision, through different
transforms, so a coefficient whose scaled value lies within rounding error of a half-integer may
differ by one; every other coefficient must be equal.  Checked in the coefficient domain (the
oracle's inverse NTT of every limb) on random slots at N=2^12, 2^14 and 2^16, over the ciphertext
basis and over the extended basis; and the encoded plaintext decodes to the slots."""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.mark.parametrize("key,level,special", [("n12-dnum2", 3, False), ("n14-hoisted8", 11, True),
                                               ("n16-full", 35, False), ("n16-bsgs32", 24, True)])
def test_encode_matches_oracle(ks_lib, oracle_mod, key, level, special):
    ks = ks_lib
    cfg = W.CONFIGS[key]
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    octx = oracle_mod.Ctx(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    n = cfg.n
    z = W.slots(cfg, W.rng(cfg.seed, W.TAG_SLOTS, 77))
    scale = float(2 ** cfg.log_scale)
    limbs = list(range(level + 1)) + ([cfg.n_q + i for i in range(cfg.n_p)] if special else [])
    out = torch.empty((len(limbs), n), dtype=torch.uint32, device="cuda")
    ws = torch.empty(n, dtype=torch.int64, device="cuda")
    ks.ckks_encode(ctx, list(z), scale, level, out, ws, with_special=special)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    m = oracle_mod.encode(z, n, scale)
    diffs = 0
    for r, t in enumerate(limbs):
        coef = octx.ntt_inv(got[r][None], t)[0].astype(np.int64)
        want = np.mod(m, octx.mod[t])
        d = np.mod(coef - want, octx.mod[t])
        assert np.all((d == 0) | (d == 1) | (d == octx.mod[t] - 1)), (t, int(np.max(np.minimum(d, octx.mod[t] - d))))
        diffs = max(diffs, int(np.count_nonzero(d)))
    assert diffs <= 4, diffs
    dec = oracle_mod.decode(octx.crt_centered(np.stack([octx.ntt_inv(got[r][None], t)[0]
                                                        for r, t in enumerate(limbs[:2])]), limbs[:2]), n, scale)
    assert np.max(np.abs(dec - z)) < 2.0 ** -15


def test_encode_errors(ks_lib):
    ks = ks_lib
    q, p = ks.ckks_gen_primes(12, 4, 1)
    ctx = ks.Context(12, q, p, 2)
    out = torch.empty((4, 4096), dtype=torch.uint32, device="cuda")
    ws = torch.empty(4096, dtype=torch.int64, device="cuda")
    with pytest.raises(ValueError):
        ks.ckks_encode(ctx, [0j] * 100, 2.0 ** 20, 3, out, ws)
    with pytest.raises(ks.CkksError) as e:
        ks.ckks_encode(ctx, [0j] * 2048, -1.0, 3, out, ws)
    assert e.value.code == ks.CKKS_ERR_ARG
    with pytest.raises(ks.CkksError) as e:
        ks.ckks_encode(ctx, [0j] * 2048, 2.0 ** 20, 3, out, ws[:100])
    assert e.value.code == ks.CKKS_ERR_WORKSPACE
