"""Seeded sweep of small parameter sets on the GPU against the oracle, bit for bit.

Chains at N=2^12 (6 + 2 primes), N=2^13 (5 + 3 primes) and N=2^15 (4 + 2 primes; the column
passes of 128 rows, which the N = 2^14 and 2^16 configurations do not reach); every dnum from 1 to L+1, so digit
widths from the whole chain down to one prime; for each, two levels drawn from a seeded
generator, one of them chosen so that the last digit is partial whenever the digit width allows
it.  At each point: a key switch, two hoisted rotations (steps 1 and -3) and a rescale (level >= 1),
each with its own synthetic key halves (uniform residues; the bits do not depend on the key being
well formed) and compared element by element with the oracle."""
import numpy as np
import pytest

import workloads as W

torch = pytest.importorskip("torch")

CHAINS = [(12, 6, 2), (13, 5, 3), (15, 4, 2)]


def _grid():
    pts = []
    for log_n, n_q, n_p in CHAINS:
        gen = W.rng(4000 + log_n, W.TAG_SYNTH)
        for dnum in range(1, n_q + 1):
            alpha = -(-n_q // dnum)
            levels = {int(gen.integers(0, n_q))}
            partial = [lv for lv in range(n_q) if (lv + 1) % alpha]
            levels.add(int(gen.choice(partial)) if partial else n_q - 1)
            for lv in sorted(levels):
                pts.append((log_n, n_q, n_p, dnum, lv))
    return pts


GRID = _grid()


def test_grid_covers_every_digit_width_and_partial_digits():
    for log_n, n_q, n_p in CHAINS:
        pts = [p for p in GRID if p[0] == log_n]
        assert sorted({p[3] for p in pts}) == list(range(1, n_q + 1))
        assert any((lv + 1) % -(-n_q // d) for _, _, _, d, lv in pts)
    assert len(GRID) <= 2 * sum(c[1] for c in CHAINS)


@pytest.mark.gpu
@pytest.mark.parametrize("log_n,n_q,n_p,dnum,level", GRID)
def test_sweep_point(ks_lib, oracle_mod, log_n, n_q, n_p, dnum, level):
    ks = ks_lib
    q, p = ks.ckks_gen_primes(log_n, n_q, n_p)
    octx = oracle_mod.Ctx(log_n, n_q, n_p)
    assert octx.q == q and octx.p == p
    ctx = ks.Context(log_n, q, p, dnum)
    n, na = 1 << log_n, level + 1
    alpha = -(-n_q // dnum)
    nd = -(-n_q // alpha)
    gen = W.rng(5000 + log_n, W.TAG_SYNTH, dnum, level)
    seed = W.random_bytes(32, gen)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint32)).cuda()
    keys = [W.uniform_residues(q + p, n, gen) for _ in range(3 * nd)]
    keys = [np.stack(keys[i * nd:(i + 1) * nd]) for i in range(3)]
    ws = ctx.workspace(level, 2)
    # key switch
    c = W.uniform_residues(q[:na], n, gen)
    kid = int(gen.integers(0, 2**32, dtype=np.uint64))
    out = torch.empty((2, na, n), dtype=torch.uint32, device="cuda")
    ks.ckks_keyswitch(ctx, dev(c), level, ks.make_evk(dev(keys[0]), seed, kid), out, ws)
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy(), octx.keyswitch(c, level, alpha, keys[0], seed, kid))
    # two hoisted rotations
    ct = W.uniform_residues(q[:na] * 2, n, gen).reshape(2, na, n)
    gs = [ks.galois_element(log_n, 1), ks.galois_element(log_n, -3)]
    evks = [ks.make_evk(dev(keys[1 + i]), seed, gs[i]) for i in range(2)]
    rot = torch.empty((2, 2, na, n), dtype=torch.uint32, device="cuda")
    ks.ckks_rotate_hoisted(ctx, dev(ct), level, gs, evks, rot, ws)
    torch.cuda.synchronize()
    want = octx.rotate_hoisted(ct, level, alpha, gs, keys[1:3], [seed, seed], gs)
    assert np.array_equal(rot.cpu().numpy(), want)
    # rescale
    if level >= 1:
        rs = torch.empty((2, level, n), dtype=torch.uint32, device="cuda")
        ks.ckks_rescale(ctx, dev(ct), level, rs, ws)
        torch.cuda.synchronize()
        assert np.array_equal(rs.cpu().numpy(), octx.rescale(ct, level))
