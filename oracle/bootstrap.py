"""Oracle for the linear parts of CKKS bootstrapping: the slot DFT ("special FFT") factored into
radix-2 stages, its levels as sums of slot diagonals, their baby-step giant-step plan, and ModRaise.

TEST INFRASTRUCTURE ONLY (tests, smoke check).  Shares no code with the CUDA library.

Bootstrapping (Cheon, Han, Kim, Kim, Song, Eurocrypt 2018; the linear maps in the form of Chen,
Chillotti, Song, Eurocrypt 2019) moves a ciphertext's coefficients into its slots (CoeffToSlot),
reduces them modulo q_0 slot-wise (EvalMod), and moves them back (SlotToCoeff).  The Perseus
write-up (ai4snews, Interpretation) puts bootstrap placement at the centre of its stack, and the
summary of EncryptedLLM (lpnh.cn page, Results) quotes 22-27 ms per bootstrap; no page gives the
construction, which is restated here from its definition:

  Decoding evaluates the plaintext m (degree < N, real coefficients) at the slot roots
  w_j = zeta^(5^j mod 2N), zeta = exp(i pi / N), j < n = N/2.  Since w_j^n = i, with
  t_k = m_k + i m_(k+n) (k < n):  z_j = sum_k t_k w_j^k,  i.e.  z = V t,  V[j][k] = w_j^k.
  SlotToCoeff multiplies the slot vector by V, CoeffToSlot by V^-1.

V factors like a radix-2 decimation-in-time FFT whose inputs are in bit-reversed order: for
butterfly length L = 2, 4, ..., n and the block-local index j < L/2 the twiddle is
w_(L,j) = zeta^((5^j mod 4L) n / L), and (x_a, x_b) -> (x_a + w x_b, x_a - w x_b) on the pair
(a, b) = (i + j, i + j + L/2).  (For the two halves of a size-L block the 5^j exponents differ by
5^(L/2) = 1 + 2L mod 4L, which turns w into -w: the butterfly's minus sign.)  Each stage is a
sum of three slot diagonals, with shifts 0, +L/2 and -L/2 (rot_r(x)[p] = x[(p + r) mod n], the
slot rotation by r); a run of consecutive stages multiplies into one level whose shifts are the
signed sums of the stages' half-lengths.
"""
from __future__ import annotations

import math

import numpy as np


def slot_root_exponents(log_n: int) -> np.ndarray:
    """5^j mod 2N for j < N/2."""
    n_slots, m = 1 << (log_n - 1), 2 << log_n
    e = np.empty(n_slots, dtype=np.int64)
    v = 1
    for j in range(n_slots):
        e[j] = v
        v = (v * 5) % m
    return e


def dft_matrix(log_n: int) -> np.ndarray:
    """V[j][k] = zeta^((5^j k) mod 2N), j, k < N/2 (O(n^2): small N only)."""
    n_slots, m = 1 << (log_n - 1), 2 << log_n
    e = slot_root_exponents(log_n)
    k = np.arange(n_slots)
    return np.exp(2j * np.pi * ((e[:, None] * k[None, :]) % m) / m)


def bitrev(x: np.ndarray) -> np.ndarray:
    n = x.shape[-1]
    bits = n.bit_length() - 1
    idx = np.array([int(format(i, f"0{bits}b")[::-1], 2) if bits else 0 for i in range(n)])
    return x[..., idx]


def stage_twiddles(log_n: int, length: int) -> np.ndarray:
    """w_(L, j) for j < L/2: zeta^((5^j mod 4L) n / L)."""
    n_slots, m = 1 << (log_n - 1), 2 << log_n
    e = slot_root_exponents(log_n)[: length // 2] % (4 * length)
    return np.exp(2j * np.pi * (e * (n_slots // length)) / m)


def rot(x: np.ndarray, r: int) -> np.ndarray:
    """Slot rotation: rot(x, r)[p] = x[(p + r) mod n]."""
    return np.roll(x, -r, axis=-1)


def stage_diagonals(log_n: int, length: int, inverse: bool = False) -> dict:
    """One butterfly stage as {shift: diagonal}: x' = sum_r d_r * rot(x, r).
    Forward: top p (block-local j < L/2) gets x_p + w x_(p+L/2); bottom p gets x_(p-L/2) - w x_p.
    Inverse (the exact inverse of the forward stage): top gets (x_p + x_(p+L/2)) / 2, bottom gets
    (x_(p-L/2) - x_p) conj(w) / 2."""
    n_slots = 1 << (log_n - 1)
    h = length // 2
    w = stage_twiddles(log_n, length)
    p = np.arange(n_slots)
    jj = p % length
    top = jj < h
    wj = np.where(top, w[np.minimum(jj, h - 1)], w[np.maximum(jj - h, 0)])
    d0 = np.zeros(n_slots, dtype=complex)
    dp = np.zeros(n_slots, dtype=complex)
    dm = np.zeros(n_slots, dtype=complex)
    if not inverse:
        d0[top], dp[top] = 1.0, wj[top]
        dm[~top], d0[~top] = 1.0, -wj[~top]
    else:
        d0[top], dp[top] = 0.5, 0.5
        dm[~top], d0[~top] = 0.5 * np.conj(wj[~top]), -0.5 * np.conj(wj[~top])
    out = {}
    for s, v in ((0, d0), (h % n_slots, dp), ((-h) % n_slots, dm)):   # +-n/2 coincide for L = n
        if np.any(v):
            out[s] = out.get(s, 0) + v
    return out


def apply_diagonals(x: np.ndarray, diags: dict) -> np.ndarray:
    out = np.zeros_like(x, dtype=complex)
    for r, d in diags.items():
        out = out + d * rot(x, r)
    return out


def compose(first: dict, then: dict, n_slots: int) -> dict:
    """Diagonals of `then` applied after `first`: shifts add (mod n)."""
    out = {}
    for s, b in then.items():
        for r, a in first.items():
            k = (s + r) % n_slots
            out[k] = out.get(k, 0) + b * rot(a, s)
    return out


def stage_lengths(log_n: int) -> list:
    """Butterfly lengths 2, 4, ..., n in the forward (SlotToCoeff) order."""
    return [1 << s for s in range(1, log_n)]


def level_diagonals(log_n: int, lengths, inverse: bool) -> dict:
    """One level made of consecutive stages (in the order they are applied)."""
    n_slots = 1 << (log_n - 1)
    acc = None
    for length in lengths:
        d = stage_diagonals(log_n, length, inverse)
        acc = d if acc is None else compose(acc, d, n_slots)
    return acc


def split_levels(log_n: int, n_levels: int, inverse: bool) -> list:
    """The stage lengths of each level: SlotToCoeff applies L = 2, 4, ..., n; CoeffToSlot applies
    the inverse stages in reverse order (L = n, ..., 2).  Levels take consecutive stages, the
    first levels one stage more when they do not divide evenly."""
    lens = stage_lengths(log_n)
    if inverse:
        lens = lens[::-1]
    q, r = divmod(len(lens), n_levels)
    out, i = [], 0
    for lv in range(n_levels):
        c = q + (1 if lv < r else 0)
        out.append(lens[i:i + c])
        i += c
    return out


def slot_to_coeff(x_brv: np.ndarray, log_n: int, n_levels: int) -> np.ndarray:
    """V applied to t given in bit-reversed order, level by level."""
    for lens in split_levels(log_n, n_levels, False):
        x_brv = apply_diagonals(x_brv, level_diagonals(log_n, lens, False))
    return x_brv


def coeff_to_slot(z: np.ndarray, log_n: int, n_levels: int) -> np.ndarray:
    """V^-1 z, returned in bit-reversed order, level by level."""
    for lens in split_levels(log_n, n_levels, True):
        z = apply_diagonals(z, level_diagonals(log_n, lens, True))
    return z


def bsgs_plan(diags: dict, n_slots: int, n1: int):
    """Baby-step giant-step plan of a level: its shifts are multiples of a step s (the smallest
    half-length); with d = (g n1 + k) s, k < n1:
        L(x) = sum_g rot(sum_k rot(D_d, -g n1 s) * rot(x, k s), g n1 s).
    Returns (baby shifts [k s], giant shifts [g n1 s], pt[giant][baby] complex diagonals, zero
    where no diagonal exists).  Shifts are taken in (-n/2, n/2]."""
    centred = {((r + n_slots // 2) % n_slots) - n_slots // 2 if r else 0: v for r, v in diags.items()}
    nz = [abs(r) for r in centred if r]
    step = min(nz) if nz else 1
    for r in centred:
        assert r % step == 0
    ms = sorted(r // step for r in centred)
    g_lo, g_hi = ms[0] // n1, ms[-1] // n1
    giants = list(range(g_lo, g_hi + 1))
    babies = list(range(n1))
    pt = np.zeros((len(giants), n1, n_slots), dtype=complex)
    for r, v in centred.items():
        m = r // step
        g, k = m // n1, m % n1
        pt[giants.index(g), k] = rot(v, -g * n1 * step)
    return [k * step for k in babies], [g * n1 * step for g in giants], pt


def apply_bsgs(x: np.ndarray, babies, giants, pt) -> np.ndarray:
    out = np.zeros_like(x, dtype=complex)
    for gi, gs in enumerate(giants):
        inner = np.zeros_like(x, dtype=complex)
        for bi, bs in enumerate(babies):
            inner = inner + pt[gi, bi] * rot(x, bs)
        out = out + rot(inner, gs)
    return out


def modraise(ctx, ct: np.ndarray, level: int) -> np.ndarray:
    """ModRaise: a ciphertext at level 0 ([2][1][N] or [2][N], evaluation domain mod q_0) read as
    integer polynomials with centred coefficients in (-q_0/2, q_0/2] and reduced into q_0..q_level:
    per component, inverse NTT mod q_0, centred lift, then each limb's NTT.  Returns
    [2][level+1][N].  It decrypts to m + q_0 I for a small integer polynomial I."""
    ct = np.ascontiguousarray(ct, dtype=np.uint32).reshape(2, ctx.n)
    q0 = ctx.q[0]
    out = np.empty((2, level + 1, ctx.n), dtype=np.uint32)
    for comp in range(2):
        coef = ctx.ntt_inv(ct[comp][None], 0)[0].astype(np.int64)
        v = np.where(coef > (q0 - 1) // 2, coef - q0, coef)
        out[comp] = ctx.signed_to_eval(v, range(level + 1))
    return out


def encode_plan(ctx, pt: np.ndarray, level: int, scale: float) -> np.ndarray:
    """The plan's complex diagonals [n_giant][n_baby][n_slots] encoded at `scale` and put in the
    evaluation domain over the extended basis q_0..q_level, p_0..p_(k-1):
    uint32 [n_giant][n_baby][ext][N] (an all-zero diagonal encodes to zero)."""
    from . import encode
    limbs = ctx.ext_limbs(level)
    ng, nb = pt.shape[:2]
    out = np.zeros((ng, nb, len(limbs), ctx.n), dtype=np.uint32)
    for g in range(ng):
        for b in range(nb):
            if np.any(pt[g, b]):
                out[g, b] = ctx.signed_to_eval(encode(pt[g, b], ctx.n, scale), limbs)
    return out


def galois_of_shift(ctx, shift: int) -> int:
    """Galois element of the slot rotation by `shift` (1 for no rotation)."""
    return 1 if shift % (ctx.n // 2) == 0 else ctx.galois(shift)


def linear_level(ctx, ct, level: int, alpha: int, babies, giants, pt_enc, keys: dict, seed: bytes):
    """One level: the baby-step giant-step transform (Ctx.bsgs, double hoisting) then the rescale by
    q_level.  keys: Galois element -> b half of its rotation key."""
    bg = [galois_of_shift(ctx, s) for s in babies]
    gg = [galois_of_shift(ctx, s) for s in giants]
    bk = [None if g == 1 else (keys[g], g) for g in bg]
    gk = [None if g == 1 else (keys[g], g) for g in gg]
    out = ctx.bsgs(ct, level, alpha, bg, bk, gg, gk, pt_enc, seed)
    return ctx.rescale(out, level)


# ----------------------------------------------------------------------------- EvalMod
# The modular reduction of bootstrapping: slots x (real, near the integers) -> x - round(x),
# approximated by sin(2 pi x) / (2 pi) = cos(2 pi (x - 1/4)) / (2 pi), the cosine evaluated as an
# even Taylor polynomial of theta = 2 pi (x - 1/4) / 2^r followed by r double angles
# cos(2t) = 2 cos(t)^2 - 1 (the scaled-sine approach of Cheon, Han, Kim, Kim, Song, Eurocrypt
# 2018, with the double-angle step of Han and Ki, CT-RSA 2020).  Every constant is an integer:
# the IEEE double product rounded half away from zero (C's llround), so that the library's
# evaluation of the same sequence is comparable bit for bit.

def llround(x: float) -> int:
    """Round half away from zero, exactly as C's llround for doubles below 2^52 in magnitude."""
    f = math.floor(x)
    d = x - f                       # exact
    if d > 0.5:
        return int(f) + 1
    if d < 0.5:
        return int(f)
    return int(f) + 1 if x > 0 else int(f)


def mul_const(ctx, ct: np.ndarray, level: int, v: int) -> np.ndarray:
    """Every component times the integer v, limb by limb modulo q_i."""
    q = np.array(ctx.q[: level + 1], dtype=np.uint64)[:, None]
    w = np.array([v % int(qi) for qi in ctx.q[: level + 1]], dtype=np.uint64)[:, None]
    return ((np.asarray(ct, dtype=np.uint64) * w) % q).astype(np.uint32)


def add_const(ctx, ct: np.ndarray, level: int, v: int) -> np.ndarray:
    """The constant polynomial v (every evaluation slot) added to component 0."""
    q = np.array(ctx.q[: level + 1], dtype=np.uint64)[:, None]
    w = np.array([v % int(qi) for qi in ctx.q[: level + 1]], dtype=np.uint64)[:, None]
    out = np.array(ct, dtype=np.uint32, copy=True)
    out[0] = ((out[0].astype(np.uint64) + w) % q).astype(np.uint32)
    return out


def evalmod(ctx, ct: np.ndarray, level: int, scale: float, r: int, d: int, alpha: int,
            relin_b: np.ndarray, seed: bytes):
    """Returns (ciphertext [2][level_out+1][N], level_out, scale_out); consumes d + r + 3 levels."""
    a = []
    fact = 1.0
    for k in range(d + 1):
        a.append((-1.0 if k & 1 else 1.0) / fact)
        fact *= float(2 * k + 1) * float(2 * k + 2)
    c1 = 2.0 * math.pi / float(1 << r)
    q = lambda lv: float(ctx.q[lv])

    def mult(x, y, lv):
        return ctx.rescale(ctx.relin(ctx.tensor(x, y, lv), lv, alpha, relin_b, seed, 0), lv)

    lv, S = level, scale
    t = ctx.rescale(mul_const(ctx, ct, lv, llround(c1 * q(lv))), lv)
    lv -= 1
    t = add_const(ctx, t, lv, llround(-(c1 / 4.0) * S))
    u = mult(t, t, lv)
    Su = S * S / q(lv)
    lv -= 1
    lu = lv
    p = ctx.rescale(mul_const(ctx, u, lv, llround(a[d] * q(lv))), lv)
    lv -= 1
    Sp = Su
    p = add_const(ctx, p, lv, llround(a[d - 1] * Sp))
    for k in range(d - 2, -1, -1):
        ua = np.ascontiguousarray(u[:, : lv + 1])
        p = mult(p, ua, lv)
        Sp = Sp * Su / q(lv)
        lv -= 1
        p = add_const(ctx, p, lv, llround(a[k] * Sp))
    for _ in range(r):
        p = mult(p, p, lv)
        Sp = Sp * Sp / q(lv)
        lv -= 1
        p = mul_const(ctx, p, lv, 2)
        p = add_const(ctx, p, lv, llround(-1.0 * Sp))
    out = ctx.rescale(mul_const(ctx, p, lv, llround(1.0 / (2.0 * math.pi) * q(lv))), lv)
    lv -= 1
    assert lu >= lv
    return out, lv, Sp


# ----------------------------------------------------------------------------- the whole bootstrap
# ModRaise, CoeffToSlot, the split into real and imaginary halves, EvalMod on each half, their
# recombination and SlotToCoeff (Cheon, Han, Kim, Kim, Song, Eurocrypt 2018, Sec. 4, with the
# linear maps of Chen, Chillotti, Song, Eurocrypt 2019).  After CoeffToSlot the slots hold
# t_k / q_0 = M_k / q_0 + i M_(k+n) / q_0 (bit-reversed order) for the raised plaintext
# M = m + q_0 I.  The real half (z + conj z) / 2 and the imaginary half (z - conj z) / (2 i) are
# formed with one conjugation; the 1/2 is folded into the last CoeffToSlot level's diagonals and the
# division by i is a product with the monomial X^(N/2), which multiplies every slot by i.

def mul_monomial_half(ctx, ct: np.ndarray, level: int) -> np.ndarray:
    """X^(N/2) times every component of ct [n_comp][level+1][N] (evaluation domain).  Done in the
    coefficient domain as the plain negacyclic product: coefficient a_k moves to k + N/2, and the
    upper half wraps round to the bottom with a minus sign (X^N = -1).  Each slot root
    w_j = zeta^(5^j) has w_j^(N/2) = exp(i pi 5^j / 2) = i (5^j = 1 mod 4), so the slots are
    multiplied by i."""
    ct = np.ascontiguousarray(ct, dtype=np.uint32)
    h = ctx.n // 2
    q = np.array(ctx.q[: level + 1], dtype=np.int64)[:, None]
    out = np.empty_like(ct)
    for comp in range(ct.shape[0]):
        coef = ctx.ntt_inv(ct[comp], 0).astype(np.int64)
        sh = np.empty_like(coef)
        sh[:, h:] = coef[:, :h]
        sh[:, :h] = (q - coef[:, h:]) % q
        out[comp] = ctx.ntt_fwd(sh.astype(np.uint32), 0)
    return out


def _add(ctx, x, y, level):
    q = np.array(ctx.q[: level + 1], dtype=np.uint64)[:, None]
    return ((np.asarray(x, dtype=np.uint64) + np.asarray(y, dtype=np.uint64)) % q).astype(np.uint32)


def _sub(ctx, x, y, level):
    q = np.array(ctx.q[: level + 1], dtype=np.uint64)[:, None]
    return ((np.asarray(x, dtype=np.uint64) + q - np.asarray(y, dtype=np.uint64)) % q).astype(np.uint32)


def bootstrap_plans(log_n: int, levels: int, n1: int):
    """The complex baby-step giant-step plans of CoeffToSlot and SlotToCoeff, `levels` levels each:
    lists of (baby shifts, giant shifts, pt[giant][baby][n_slots]).  The last CoeffToSlot level
    carries the factor 1/2 of the split into real and imaginary halves."""
    ns = 1 << (log_n - 1)
    c2s = []
    for i, lens in enumerate(split_levels(log_n, levels, True)):
        diags = level_diagonals(log_n, lens, True)
        if i == levels - 1:
            diags = {r: 0.5 * v for r, v in diags.items()}
        c2s.append(bsgs_plan(diags, ns, n1))
    s2c = [bsgs_plan(level_diagonals(log_n, lens, False), ns, n1) for lens in split_levels(log_n, levels, False)]
    return c2s, s2c


def bootstrap_levels(top: int, n_c2s: int, n_s2c: int, r: int, d: int):
    """Levels at which the CoeffToSlot and SlotToCoeff transforms run, and the output level."""
    c2s = [top - i for i in range(n_c2s)]
    lz = top - n_c2s - (d + r + 3)
    s2c = [lz - i for i in range(n_s2c)]
    return c2s, s2c, lz - n_s2c


def bootstrap(ctx, ct0: np.ndarray, top: int, alpha: int, c2s, s2c, keys: dict, conj_b, relin_b,
              seed: bytes, r: int, d: int):
    """Bootstraps ct0 ([2][1][N] or [2][N] at level 0).  c2s, s2c: per level (baby shifts, giant
    shifts, plaintexts encoded at scale q_level over the extended basis, uint32
    [giant][baby][ext][N]), at the levels of bootstrap_levels.  keys: Galois element -> b half of
    the rotation key; conj_b: the key of g = 2N - 1; relin_b: the key of s^2 (key_id 0).
    Returns (ciphertext [2][level_out+1][N], level_out, ratio): the output decodes at scale
    ratio * Delta to the input's slots, Delta being the input's scale (its plaintext m becomes
    sin(2 pi m / q_0) q_0 / (2 pi) ~ m, times ratio)."""
    g_conj = 2 * ctx.n - 1
    lv = top
    ct = modraise(ctx, ct0, top)
    for babies, giants, enc in c2s:
        ct = linear_level(ctx, ct, lv, alpha, babies, giants, enc, keys, seed)
        lv -= 1
    cj = ctx.rotate(ct, lv, alpha, g_conj, conj_b, seed, g_conj)
    re = _add(ctx, ct, cj, lv)
    im = mul_monomial_half(ctx, _sub(ctx, cj, ct, lv), lv)
    s_in = float(ctx.q[0])
    re, lo, sp = evalmod(ctx, re, lv, s_in, r, d, alpha, relin_b, seed)
    im, lo2, sp2 = evalmod(ctx, im, lv, s_in, r, d, alpha, relin_b, seed)
    assert (lo, sp) == (lo2, sp2)
    lv = lo
    ct = _add(ctx, re, mul_monomial_half(ctx, im, lv), lv)
    for babies, giants, enc in s2c:
        ct = linear_level(ctx, ct, lv, alpha, babies, giants, enc, keys, seed)
        lv -= 1
    return ct, lv, sp / s_in


def encoded_plans(ctx, plans, lvls):
    """Encodes each complex plan at its level (scale q_level, extended basis).  Returns the list of
    (baby shifts, giant shifts, encoded plaintexts) and the sorted Galois elements the plans rotate
    by (1 excluded)."""
    out, gal = [], set()
    for (babies, giants, pt), lv in zip(plans, lvls):
        gal.update(galois_of_shift(ctx, s) for s in babies + giants)
        out.append((babies, giants, encode_plan(ctx, pt, lv, float(ctx.q[lv]))))
    gal.discard(1)
    return out, sorted(gal)
