"""Batched entry points: every item of a batch equals the single call (and so the oracle) bit for
bit, including batches longer than one launch chunk and hoisted rotations spanning chunks."""
import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


def _res(moduli, n, gen):
    return torch.from_numpy(W.uniform_residues(moduli, n, gen)).cuda()


def _setup(ks, key):
    cfg = W.CONFIGS[key]
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    return cfg, q, p, ks.Context(cfg.log_n, q, p, cfg.dnum)


@pytest.mark.parametrize("key,n", [("n12-dnum2", 5), ("n14-hoisted8", 3), ("n16-full", 2)])
def test_batches_equal_single_calls(ks_lib, key, n):
    ks = ks_lib
    cfg, q, p, ctx = _setup(ks, key)
    lvl, N = cfg.level, cfg.n
    na = lvl + 1
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 900 + n)
    nd = -(-cfg.n_q // cfg.alpha)
    keys_t = [_res((q + p) * nd, N, gen).view(nd, len(q) + len(p), N) for _ in range(n)]
    gs = [ks.galois_element(cfg.log_n, r) for r in (1, -1, 2, 3, -5, 7)[:n]]
    evks = [ks.make_evk(keys_t[i], cfg.chacha_seed, gs[i]) for i in range(n)]
    x = _res(q[:na] * 2 * n, N, gen).view(n, 2, na, N)
    y = _res(q[:na] * 2 * n, N, gen).view(n, 2, na, N)
    ws_b = ctx.workspace(lvl, n)
    ws_1 = ctx.workspace(lvl)
    # tensor
    d = torch.empty((n, 3, na, N), dtype=torch.uint32, device="cuda")
    ks.ckks_tensor_batch(ctx, n, x, y, lvl, d)
    for i in range(n):
        di = torch.empty((3, na, N), dtype=torch.uint32, device="cuda")
        ks.ckks_tensor(ctx, x[i], y[i], lvl, di)
        assert torch.equal(di, d[i])
    # relin (items share one key), rotate, keyswitch
    out = torch.empty((n, 2, na, N), dtype=torch.uint32, device="cuda")
    one = torch.empty((2, na, N), dtype=torch.uint32, device="cuda")
    ks.ckks_relin_batch(ctx, d, lvl, [evks[0]] * n, out, ws_b)
    for i in range(n):
        ks.ckks_relin(ctx, d[i], lvl, evks[0], one, ws_1)
        assert torch.equal(one, out[i])
    ks.ckks_rotate_batch(ctx, x, lvl, gs, evks, out, ws_b)
    for i in range(n):
        ks.ckks_rotate(ctx, x[i], lvl, gs[i], evks[i], one, ws_1)
        assert torch.equal(one, out[i])
    c = x[:, 1].contiguous()
    ks.ckks_keyswitch_batch(ctx, c, lvl, evks, out, ws_b)
    for i in range(n):
        ks.ckks_keyswitch(ctx, c[i], lvl, evks[i], one, ws_1)
        assert torch.equal(one, out[i])


def test_rotate_batch_longer_than_a_chunk(ks_lib):
    """70 rotations at N=2^12 (two launch chunks of at most 64 items)."""
    ks = ks_lib
    cfg, q, p, ctx = _setup(ks, "n12-dnum4")
    lvl, N, na, n = cfg.level, cfg.n, cfg.level + 1, 70
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 77)
    nd = -(-cfg.n_q // cfg.alpha)
    kt = _res((q + p) * nd, N, gen).view(nd, len(q) + len(p), N)
    gs = [ks.galois_element(cfg.log_n, r) for r in range(1, n + 1)]
    evks = [ks.make_evk(kt, cfg.chacha_seed, g) for g in gs]
    ct = _res(q[:na] * 2 * n, N, gen).view(n, 2, na, N)
    out = torch.empty((n, 2, na, N), dtype=torch.uint32, device="cuda")
    ks.ckks_rotate_batch(ctx, ct, lvl, gs, evks, out, ctx.workspace(lvl, n))
    one = torch.empty((2, na, N), dtype=torch.uint32, device="cuda")
    ws1 = ctx.workspace(lvl)
    for i in (0, 63, 64, 69):
        ks.ckks_rotate(ctx, ct[i], lvl, gs[i], evks[i], one, ws1)
        assert torch.equal(one, out[i])


def test_hoisted_across_chunks_matches_oracle(ks_lib, oracle_mod):
    """Hoisted rotations spanning two chunks equal the oracle (sampled rotations)."""
    from oracle.scenario import Scenario
    ks = ks_lib
    cfg = W.CONFIGS["n12-dnum4"]
    sc = Scenario(cfg)
    q, p = ks.ckks_gen_primes(cfg.log_n, cfg.n_q, cfg.n_p)
    ctx = ks.Context(cfg.log_n, q, p, cfg.dnum)
    lvl, n = cfg.level, 66
    _, ct = sc.ciphertext(0)
    steps = list(range(1, n + 1))
    gs = [sc.galois(r) for r in steps]
    keys_np = {g: sc.key(g) for g in gs}
    keys_t = {g: torch.from_numpy(keys_np[g]).cuda() for g in gs}
    evks = [ks.make_evk(keys_t[g], cfg.chacha_seed, g) for g in gs]
    out = torch.empty((n, 2, lvl + 1, cfg.n), dtype=torch.uint32, device="cuda")
    ks.ckks_rotate_hoisted(ctx, torch.from_numpy(ct).cuda(), lvl, gs, evks, out, ctx.workspace(lvl, n))
    got = out.cpu().numpy()
    for i in (0, 40, 64, 65):
        want = sc.ctx.rotate(ct, lvl, cfg.alpha, gs[i], keys_np[gs[i]], cfg.chacha_seed, gs[i])
        assert np.array_equal(got[i], want)


def test_shared_key_groups(ks_lib):
    """Items whose a half is the same (same seed and key id) share one regenerated keystream in
    groups of up to 8; items with another seed, or a stored a half, do not.  Every item equals
    the single call (which regenerates the keystream in registers)."""
    ks = ks_lib
    cfg, q, p, ctx = _setup(ks, "n14-hoisted8")
    lvl, N = cfg.level, cfg.n
    na = lvl + 1
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 4242)
    nd = -(-cfg.n_q // cfg.alpha)
    shape = (nd, len(q) + len(p), N)
    b1, b2, b3, b4, a4 = (_res((q + p) * nd, N, gen).view(*shape) for _ in range(5))
    s1, s2 = bytes(range(32)), bytes(range(1, 33))
    kid = 77
    A = ks.make_evk(b1, s1, kid)            # shares its a half with A2 (same seed and key id)
    A2 = ks.make_evk(b2, s1, kid)
    Bk = ks.make_evk(b3, s2, kid)
    S = ks.make_evk(b4, s1, kid, a=a4)      # stored a half: never grouped
    n = 21
    evks = [[A, A2, Bk][i % 3] for i in range(n - 1)] + [S]
    c = _res(q[:na] * n, N, gen).view(n, na, N)
    out = torch.empty((n, 2, na, N), dtype=torch.uint32, device="cuda")
    one = torch.empty((2, na, N), dtype=torch.uint32, device="cuda")
    ks.ckks_keyswitch_batch(ctx, c, lvl, evks, out, ctx.workspace(lvl, n))
    ws_1 = ctx.workspace(lvl)
    for i in range(n):
        ks.ckks_keyswitch(ctx, c[i], lvl, evks[i], one, ws_1)
        assert torch.equal(one, out[i]), i


@pytest.mark.slow
def test_bench_launch_configuration(ks_lib, oracle_mod):
    """The launch configuration the benchmark times: n16-full, 4 units per batched call, every
    unit with its own seed and b half; tensor -> relin -> rotate(1).  Every item equals the
    single calls; items 0 and 3 equal the oracle (sampled: the oracle takes seconds per unit)."""
    import hashlib
    ks = ks_lib
    cfg, q, p, ctx = _setup(ks, "n16-full")
    lvl, N = cfg.level, cfg.n
    na, B = lvl + 1, 4
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 777)
    nd = -(-cfg.n_q // cfg.alpha)
    g = ks.galois_element(cfg.log_n, 1)
    b_rel = [_res((q + p) * nd, N, gen).view(nd, len(q) + len(p), N) for _ in range(B)]
    b_rot = [_res((q + p) * nd, N, gen).view(nd, len(q) + len(p), N) for _ in range(B)]
    seeds = [hashlib.sha256(cfg.chacha_seed + bytes([0, i])).digest() for i in range(B)]
    k_rel = [ks.make_evk(b_rel[i], seeds[i], 0) for i in range(B)]
    k_rot = [ks.make_evk(b_rot[i], seeds[i], g) for i in range(B)]
    x = _res(q[:na] * 2 * B, N, gen).view(B, 2, na, N)
    y = _res(q[:na] * 2 * B, N, gen).view(B, 2, na, N)
    d = torch.empty((B, 3, na, N), dtype=torch.uint32, device="cuda")
    r = torch.empty((B, 2, na, N), dtype=torch.uint32, device="cuda")
    out = torch.empty((B, 2, na, N), dtype=torch.uint32, device="cuda")
    ws = ctx.workspace(lvl, B)
    ks.ckks_tensor_batch(ctx, B, x, y, lvl, d)
    ks.ckks_relin_batch(ctx, d, lvl, k_rel, r, ws)
    ks.ckks_rotate_batch(ctx, r, lvl, [g] * B, k_rot, out, ws)
    torch.cuda.synchronize()
    one_d = torch.empty((3, na, N), dtype=torch.uint32, device="cuda")
    one_r = torch.empty((2, na, N), dtype=torch.uint32, device="cuda")
    one_o = torch.empty((2, na, N), dtype=torch.uint32, device="cuda")
    ws1 = ctx.workspace(lvl)
    for i in range(B):
        ks.ckks_tensor(ctx, x[i], y[i], lvl, one_d)
        ks.ckks_relin(ctx, one_d, lvl, k_rel[i], one_r, ws1)
        ks.ckks_rotate(ctx, one_r, lvl, g, k_rot[i], one_o, ws1)
        assert torch.equal(one_o, out[i]), i
    octx = oracle_mod.Ctx(cfg.log_n, cfg.n_q, cfg.n_p)
    for i in (0, B - 1):
        xi, yi = x[i].cpu().numpy(), y[i].cpu().numpy()
        rel = octx.relin(octx.tensor(xi, yi, lvl), lvl, cfg.alpha, b_rel[i].cpu().numpy(), seeds[i], 0)
        want = octx.rotate(rel, lvl, cfg.alpha, g, b_rot[i].cpu().numpy(), seeds[i], g)
        assert np.array_equal(out[i].cpu().numpy(), want), i


def test_two_streams_share_a_context(ks_lib):
    """The benchmark's concurrency: one context, two streams with a workspace each, each stream
    running tensor -> relin -> rotate on its own 2 units of n16-full while the other runs.  Both
    results equal the same calls made one after the other on the default stream."""
    import hashlib
    ks = ks_lib
    cfg, q, p, ctx = _setup(ks, "n16-full")
    lvl, N = cfg.level, cfg.n
    na, B, S = lvl + 1, 4, 2
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 779)
    nd = -(-cfg.n_q // cfg.alpha)
    g = ks.galois_element(cfg.log_n, 1)
    seeds = [hashlib.sha256(cfg.chacha_seed + bytes([1, i])).digest() for i in range(B)]
    k_rel = [ks.make_evk(_res((q + p) * nd, N, gen).view(nd, len(q) + len(p), N), seeds[i], 0) for i in range(B)]
    k_rot = [ks.make_evk(_res((q + p) * nd, N, gen).view(nd, len(q) + len(p), N), seeds[i], g) for i in range(B)]
    x = _res(q[:na] * 2 * B, N, gen).view(B, 2, na, N)
    y = _res(q[:na] * 2 * B, N, gen).view(B, 2, na, N)

    def run(streams):
        d = torch.empty((B, 3, na, N), dtype=torch.uint32, device="cuda")
        r = torch.empty((B, 2, na, N), dtype=torch.uint32, device="cuda")
        out = torch.empty((B, 2, na, N), dtype=torch.uint32, device="cuda")
        per = B // len(streams)
        wss = [ctx.workspace(lvl, per) for _ in streams]
        torch.cuda.synchronize()
        for si, st in enumerate(streams):
            z = slice(si * per, (si + 1) * per)
            with torch.cuda.stream(st):
                ks.ckks_tensor_batch(ctx, per, x[z], y[z], lvl, d[z], st)
                ks.ckks_relin_batch(ctx, d[z], lvl, k_rel[z], r[z], wss[si], st)
                ks.ckks_rotate_batch(ctx, r[z], lvl, [g] * per, k_rot[z], out[z], wss[si], st)
        torch.cuda.synchronize()
        for st in streams:
            assert ks.ckks_sync_status(ctx, st, 10000) == ks.CKKS_OK
        return out

    want = run([torch.cuda.default_stream()])
    got = run([torch.cuda.Stream() for _ in range(S)])
    assert torch.equal(got, want)


@pytest.mark.slow
def test_n16_stream64_shared_keystream_batches(ks_lib, oracle_mod):
    """The n16-stream64 line's launch configuration (N=2^16, level 20, dnum 4, so beta = 3):
    ckks_relin_batch over 64 items with one relinearisation key, whose items form 8 groups of 8
    that share one regenerated a half, and ckks_rotate_batch over 64 items with the 15 keys of
    steps 2^(i mod 15), groups of 4 or 5 items.  Sampled items (the first and last of the batch,
    and items inside a group) equal the oracle bit for bit."""
    ks = ks_lib
    cfg, q, p, ctx = _setup(ks, "n16-stream64")
    lvl, N = cfg.level, cfg.n
    na, P = lvl + 1, cfg.n_pairs
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 6464)
    nd = -(-cfg.n_q // cfg.alpha)
    shape = (nd, len(q) + len(p), N)
    b_rel = W.uniform_residues((q + p) * nd, N, gen).reshape(shape)
    steps = sorted(set(cfg.rot_steps), key=cfg.rot_steps.index)
    gal = {r: ks.galois_element(cfg.log_n, r) for r in steps}
    b_rot = {r: W.uniform_residues((q + p) * nd, N, gen).reshape(shape) for r in steps}
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    k_rel = ks.make_evk(dev(b_rel), cfg.chacha_seed, 0)
    k_rot = {r: ks.make_evk(dev(b_rot[r]), cfg.chacha_seed, gal[r]) for r in steps}
    d = W.uniform_residues(q[:na] * 3 * P, N, gen).reshape(P, 3, na, N)
    ws = ctx.workspace(lvl, P)
    r1 = torch.empty((P, 2, na, N), dtype=torch.uint32, device="cuda")
    out = torch.empty_like(r1)
    ks.ckks_relin_batch(ctx, dev(d), lvl, [k_rel] * P, r1, ws)
    ks.ckks_rotate_batch(ctx, r1, lvl, [gal[r] for r in cfg.rot_steps], [k_rot[r] for r in cfg.rot_steps],
                         out, ws)
    torch.cuda.synchronize()
    got_r, got_o = r1.cpu().numpy(), out.cpu().numpy()
    octx = oracle_mod.Ctx(cfg.log_n, cfg.n_q, cfg.n_p)
    for i in (0, 13, 63):           # 13: inside the relinearisation group of items 8..15
        want = octx.relin(d[i], lvl, cfg.alpha, b_rel, cfg.chacha_seed, 0)
        assert np.array_equal(got_r[i], want), ("relin", i)
    for i in (0, 17, 63):           # 17: step 4's group is items 2, 17, 32, 47, 62
        r = cfg.rot_steps[i]
        want = octx.rotate(got_r[i], lvl, cfg.alpha, gal[r], b_rot[r], cfg.chacha_seed, gal[r])
        assert np.array_equal(got_o[i], want), ("rotate", i)


@pytest.mark.parametrize("key,n_ct,steps", [("n14-hoisted8", 8, (1, -1, 2, -2, 4, -4, 8, -8)),
                                            ("n12-dnum4", 9, (1, -1, 2, -2, 4, -4, 8, -8)),
                                            ("n14-hoisted8", 3, (5,))])
def test_hoisted_batch_equals_per_ciphertext(ks_lib, key, n_ct, steps):
    """ckks_rotate_hoisted_batch: output (u, r) equals ckks_rotate_hoisted of ciphertext u alone
    (pinned to the oracle in test_gpu_parity), bit for bit; 9 x 8 pairs span two launches of 64 and
    8, and one rotation per ciphertext takes the fused row pass."""
    ks = ks_lib
    cfg, q, p, ctx = _setup(ks, key)
    lvl, N = cfg.level, cfg.n
    na = lvl + 1
    gen = W.rng(cfg.seed, W.TAG_SYNTH, 9700 + n_ct)
    nd = -(-cfg.n_q // cfg.alpha)
    gs = [ks.galois_element(cfg.log_n, r) for r in steps]
    evks = [ks.make_evk(_res((q + p) * nd, N, gen).view(nd, len(q) + len(p), N), cfg.chacha_seed, g) for g in gs]
    R = len(gs)
    x = _res(q[:na] * 2 * n_ct, N, gen).view(n_ct, 2, na, N)
    out = torch.empty((n_ct, R, 2, na, N), dtype=torch.uint32, device="cuda")
    ws = ctx.workspace(lvl, min(n_ct, 64 // R) * R)
    ks.ckks_rotate_hoisted_batch(ctx, x, lvl, gs, evks, out, ws)
    one = torch.empty((R, 2, na, N), dtype=torch.uint32, device="cuda")
    ws_1 = ctx.workspace(lvl, R)
    for u in range(n_ct):
        ks.ckks_rotate_hoisted(ctx, x[u], lvl, gs, evks, one, ws_1)
        assert torch.equal(one, out[u]), u
    assert ks.ckks_sync_status(ctx, None, 10000) == ks.CKKS_OK


def test_hoisted_batch_sampled_oracle(ks_lib, oracle_mod):
    """ckks_rotate_hoisted_batch at n14-hoisted8 with the oracle's keys: ciphertexts 0 and 5 of 8,
    all 8 rotations, equal the oracle's hoisted rotations bit for bit."""
    from oracle.scenario import Scenario
    ks = ks_lib
    cfg, q, p, ctx = _setup(ks, "n14-hoisted8")
    sc = Scenario(cfg)
    lvl, N = cfg.level, cfg.n
    gs = [sc.galois(r) for r in cfg.rot_steps]
    keys = [sc.key(g) for g in gs]
    evks = [ks.make_evk(torch.from_numpy(k).cuda(), cfg.chacha_seed, g) for k, g in zip(keys, gs)]
    cts = [sc.ciphertext(u)[1] for u in range(8)]
    x = torch.from_numpy(np.stack(cts)).cuda()
    out = torch.empty((8, len(gs), 2, lvl + 1, N), dtype=torch.uint32, device="cuda")
    ks.ckks_rotate_hoisted_batch(ctx, x, lvl, gs, evks, out, ctx.workspace(lvl, 8 * len(gs)))
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    for u in (0, 5):
        want = sc.ctx.rotate_hoisted(cts[u], lvl, cfg.alpha, gs, keys, [cfg.chacha_seed] * len(gs), gs)
        assert np.array_equal(got[u], want), u
