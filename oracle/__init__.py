"""CPU oracle for RNS-CKKS hybrid key switching with ChaCha12 key regeneration.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg (and its ``--impl reference`` arm) may import this package.  It shares no code
with the CUDA library; the integer core is plain C (``ckks_oracle.c``), the encoding and CRT
steps below are numpy and Python integers.

Method: the Perseus write-up (ai4snews, Interpretation, 2nd paragraph) regenerates the
uniform half of each key-switching key with counter-mode ChaCha12 inside the kernels that use
the key, over a 32-bit RNS CKKS chain; the arithmetic follows full-RNS CKKS (Cheon-Han-Kim-
Kim-Song, SAC 2018) and hybrid key switching (Han-Ki, CT-RSA 2020).

Parity status: every function here is pinned by ``tests/test_oracle_*.py`` against brute force,
closed forms, Python big-integer restatements, an independent ChaCha20 (OpenSSL through
``cryptography``) and the RFC 8439 block vector, and by decryption identities.  The 12-round
count is pinned by the published reduced-round test vectors (ChaCha12 and ChaCha8 with an
all-zero key and IV, ``tests/golden/chacha_vectors.txt``), beside the 20-round RFC vectors.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build_oracle

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = build_oracle.build()
        L = ctypes.CDLL(path)
        u32p = ctypes.POINTER(ctypes.c_uint32)
        i64p = ctypes.POINTER(ctypes.c_int64)
        u8p = ctypes.POINTER(ctypes.c_uint8)
        vp = ctypes.c_void_p
        ci, cu = ctypes.c_int, ctypes.c_uint32
        sig = {
            "or_is_prime": (ci, [ctypes.c_uint64]),
            "or_gen_primes": (ci, [ci, ci, u32p]),
            "or_find_psi": (cu, [cu, ci]),
            "or_ctx_create": (vp, [ci, ci, ci, u32p, u32p]),
            "or_ctx_destroy": (None, [vp]),
            "or_ctx_psi": (cu, [vp, ci]),
            "or_ntt_fwd": (None, [vp, u32p, ci, ci]),
            "or_ntt_inv": (None, [vp, u32p, ci, ci]),
            "or_automorph_coef": (None, [vp, ci, u32p, u32p, cu]),
            "or_automorph_eval": (None, [vp, u32p, u32p, ci, cu]),
            "or_galois_elt": (cu, [ci, ci]),
            "or_chacha_block": (None, [u32p, cu, u32p, ci, u32p]),
            "or_chacha_expand": (None, [vp, u8p, cu, cu, ci, u32p]),
            "or_modup": (None, [vp, u32p, ci, ci, u32p]),
            "or_inner_product": (None, [vp, u32p, ci, ci, u32p, u32p, u8p, cu, u32p, u32p]),
            "or_moddown": (None, [vp, u32p, ci, u32p]),
            "or_keyswitch": (None, [vp, u32p, ci, ci, u32p, u32p, u8p, cu, u32p]),
            "or_rotate": (None, [vp, u32p, ci, ci, cu, u32p, u32p, u8p, cu, u32p]),
            "or_rotate_hoisted": (None, [vp, u32p, ci, ci, ci, u32p, ctypes.POINTER(u32p),
                                         ctypes.POINTER(u32p), u8p, u32p, u32p]),
            "or_relin": (None, [vp, u32p, ci, ci, u32p, u32p, u8p, cu, u32p]),
            "or_tensor": (None, [vp, u32p, u32p, ci, u32p]),
            "or_rescale": (None, [vp, u32p, ci, ci, u32p]),
            "or_signed_to_eval": (None, [vp, i64p, ci, u32p]),
            "or_keygen": (None, [vp, ci, i64p, u32p, i64p, u8p, cu, u32p, u32p]),
            "or_encrypt": (None, [vp, i64p, i64p, i64p, u32p, ci, u32p]),
            "or_decrypt": (None, [vp, u32p, ci, ci, u32p, u32p]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _u32(a: np.ndarray):
    assert a.dtype == np.uint32 and a.flags["C_CONTIGUOUS"], (a.dtype, a.flags)
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint32))


def _i64(a: np.ndarray):
    assert a.dtype == np.int64 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))


def _u8(b: bytes):
    arr = (ctypes.c_uint8 * len(b)).from_buffer_copy(b)
    return ctypes.cast(arr, ctypes.POINTER(ctypes.c_uint8)), arr


# ----------------------------------------------------------------------------- scalars

def is_prime(x: int) -> bool:
    return bool(lib().or_is_prime(x))


def gen_primes(log_n: int, count: int) -> list:
    out = np.zeros(count, dtype=np.uint32)
    got = lib().or_gen_primes(log_n, count, _u32(out))
    if got != count:
        raise ValueError(f"only {got} primes below 2^30 for log_n={log_n}")
    return [int(x) for x in out]


def find_psi(q: int, log_n: int) -> int:
    return int(lib().or_find_psi(q, log_n))


def galois_elt(log_n: int, r: int) -> int:
    return int(lib().or_galois_elt(log_n, r))


def chain(log_n: int, n_q: int, n_p: int):
    """(q list, p list): the first n_p primes found are special, the next n_q ciphertext."""
    pr = gen_primes(log_n, n_p + n_q)
    return pr[n_p:], pr[:n_p]


def chacha_block(key: bytes, counter: int, nonce: bytes, rounds: int) -> bytes:
    """One ChaCha block (RFC 8439 state layout), `rounds` rounds, 64 output bytes."""
    k = np.frombuffer(key, dtype="<u4").astype(np.uint32).copy()
    nn = np.frombuffer(nonce, dtype="<u4").astype(np.uint32).copy()
    out = np.zeros(16, dtype=np.uint32)
    lib().or_chacha_block(_u32(k), counter, _u32(nn), rounds, _u32(out))
    return out.astype("<u4").tobytes()


# ----------------------------------------------------------------------------- context

class Ctx:
    """Oracle context over one prime chain: q_0..q_{n_q-1} then p_0..p_{n_p-1}."""

    def __init__(self, log_n: int, n_q: int, n_p: int, alpha: int | None = None,
                 q=None, p=None):
        if q is None:
            q, p = chain(log_n, n_q, n_p)
        self.log_n, self.n, self.n_q, self.n_p = log_n, 1 << log_n, n_q, n_p
        self.q, self.p = list(q), list(p)
        self.mod = self.q + self.p
        self.alpha = alpha
        qa = np.array(self.q, dtype=np.uint32)
        pa = np.array(self.p if self.p else [0], dtype=np.uint32)
        self._h = lib().or_ctx_create(log_n, n_q, n_p, _u32(qa), _u32(pa))

    def __del__(self):
        if getattr(self, "_h", None) and _lib is not None:
            _lib.or_ctx_destroy(self._h)
            self._h = None

    # --- helpers
    def digits(self, level: int, alpha: int):
        na = level + 1
        return [(lo, min(lo + alpha, na)) for lo in range(0, na, alpha)]

    def ext_limbs(self, level: int):
        """global limb indices of the extended basis at `level`: q_0..q_l, p_0..p_{k-1}."""
        return list(range(level + 1)) + [self.n_q + i for i in range(self.n_p)]

    def psi(self, t: int) -> int:
        return int(lib().or_ctx_psi(self._h, t))

    # --- NTT
    def ntt_fwd(self, poly: np.ndarray, first_limb: int = 0) -> np.ndarray:
        a = np.ascontiguousarray(poly, dtype=np.uint32).copy()
        nl = a.size // self.n
        lib().or_ntt_fwd(self._h, _u32(a), first_limb, nl)
        return a

    def ntt_inv(self, poly: np.ndarray, first_limb: int = 0) -> np.ndarray:
        a = np.ascontiguousarray(poly, dtype=np.uint32).copy()
        nl = a.size // self.n
        lib().or_ntt_inv(self._h, _u32(a), first_limb, nl)
        return a

    def automorph_eval(self, poly: np.ndarray, g: int) -> np.ndarray:
        a = np.ascontiguousarray(poly, dtype=np.uint32)
        out = np.empty_like(a)
        lib().or_automorph_eval(self._h, _u32(a), _u32(out), a.size // self.n, g)
        return out

    def automorph_coef(self, limb: np.ndarray, t: int, g: int) -> np.ndarray:
        a = np.ascontiguousarray(limb, dtype=np.uint32)
        out = np.empty_like(a)
        lib().or_automorph_coef(self._h, t, _u32(a), _u32(out), g)
        return out

    def galois(self, r: int) -> int:
        return galois_elt(self.log_n, r)

    def chacha_expand(self, seed: bytes, key_id: int, digit: int, t: int) -> np.ndarray:
        out = np.empty(self.n, dtype=np.uint32)
        sp, _keep = _u8(seed)
        lib().or_chacha_expand(self._h, sp, key_id, digit, t, _u32(out))
        return out

    # --- key switching steps
    def modup(self, c: np.ndarray, level: int, alpha: int) -> np.ndarray:
        na = level + 1
        ext = na + self.n_p
        beta = -(-na // alpha)
        c = np.ascontiguousarray(c, dtype=np.uint32).reshape(na, self.n)
        dt = np.empty((beta, ext, self.n), dtype=np.uint32)
        lib().or_modup(self._h, _u32(c), level, alpha, _u32(dt))
        return dt

    def inner_product(self, dt, level, alpha, b, seed, key_id, a_stored=None):
        ext = level + 1 + self.n_p
        dt = np.ascontiguousarray(dt, dtype=np.uint32)
        b = np.ascontiguousarray(b, dtype=np.uint32)
        acc0 = np.empty((ext, self.n), dtype=np.uint32)
        acc1 = np.empty((ext, self.n), dtype=np.uint32)
        sp, _keep = _u8(seed)
        ap = _u32(np.ascontiguousarray(a_stored, dtype=np.uint32)) if a_stored is not None else None
        lib().or_inner_product(self._h, _u32(dt), level, alpha, _u32(b), ap, sp, key_id,
                               _u32(acc0), _u32(acc1))
        return acc0, acc1

    def moddown(self, acc: np.ndarray, level: int) -> np.ndarray:
        acc = np.ascontiguousarray(acc, dtype=np.uint32)
        out = np.empty((level + 1, self.n), dtype=np.uint32)
        lib().or_moddown(self._h, _u32(acc), level, _u32(out))
        return out

    def keyswitch(self, c, level, alpha, b, seed, key_id, a_stored=None):
        c = np.ascontiguousarray(c, dtype=np.uint32)
        b = np.ascontiguousarray(b, dtype=np.uint32)
        out = np.empty((2, level + 1, self.n), dtype=np.uint32)
        sp, _keep = _u8(seed)
        ap = _u32(np.ascontiguousarray(a_stored, dtype=np.uint32)) if a_stored is not None else None
        lib().or_keyswitch(self._h, _u32(c), level, alpha, _u32(b), ap, sp, key_id, _u32(out))
        return out

    def rotate(self, ct, level, alpha, g, b, seed, key_id, a_stored=None):
        ct = np.ascontiguousarray(ct, dtype=np.uint32)
        b = np.ascontiguousarray(b, dtype=np.uint32)
        out = np.empty((2, level + 1, self.n), dtype=np.uint32)
        sp, _keep = _u8(seed)
        ap = _u32(np.ascontiguousarray(a_stored, dtype=np.uint32)) if a_stored is not None else None
        lib().or_rotate(self._h, _u32(ct), level, alpha, g, _u32(b), ap, sp, key_id, _u32(out))
        return out

    def rotate_hoisted(self, ct, level, alpha, gs, keys_b, seeds, key_ids, keys_a=None):
        ct = np.ascontiguousarray(ct, dtype=np.uint32)
        nr = len(gs)
        kb = [np.ascontiguousarray(b, dtype=np.uint32) for b in keys_b]
        bptrs = (ctypes.POINTER(ctypes.c_uint32) * nr)(*[_u32(b) for b in kb])
        aptrs = None
        if keys_a is not None:
            ka = [np.ascontiguousarray(a, dtype=np.uint32) for a in keys_a]
            aptrs = (ctypes.POINTER(ctypes.c_uint32) * nr)(*[_u32(a) for a in ka])
        garr = np.array(gs, dtype=np.uint32)
        ids = np.array(key_ids, dtype=np.uint32)
        sp, _keep = _u8(b"".join(seeds))
        out = np.empty((nr, 2, level + 1, self.n), dtype=np.uint32)
        lib().or_rotate_hoisted(self._h, _u32(ct), level, alpha, nr, _u32(garr), bptrs, aptrs,
                                sp, _u32(ids), _u32(out))
        return out

    def relin(self, d, level, alpha, b, seed, key_id, a_stored=None):
        d = np.ascontiguousarray(d, dtype=np.uint32)
        b = np.ascontiguousarray(b, dtype=np.uint32)
        out = np.empty((2, level + 1, self.n), dtype=np.uint32)
        sp, _keep = _u8(seed)
        ap = _u32(np.ascontiguousarray(a_stored, dtype=np.uint32)) if a_stored is not None else None
        lib().or_relin(self._h, _u32(d), level, alpha, _u32(b), ap, sp, key_id, _u32(out))
        return out

    def rescale(self, ct, level):
        """Rescale by q_level: [n_comp][level+1][N] -> [n_comp][level][N] (evaluation domain)."""
        ct = np.ascontiguousarray(ct, dtype=np.uint32)
        if ct.ndim == 2:
            ct = ct[None]
        assert level >= 1 and ct.shape[1:] == (level + 1, self.n)
        out = np.empty((ct.shape[0], level, self.n), dtype=np.uint32)
        lib().or_rescale(self._h, _u32(ct), ct.shape[0], level, _u32(out))
        return out

    def bsgs(self, ct, level, alpha, baby_g, baby_keys, giant_g, giant_keys, pt, seed):
        """Baby-step giant-step linear transform with double hoisting.

        Computes sum_j rot_{G_j}( sum_k pt[j][k] * rot_{B_k}(ct) ) where the baby rotations are
        hoisted (one ModUp of c1) and kept in the extended basis PQ, the plaintext products are
        summed there, and one ModDown per giant step follows (double hoisting: Bossuat, Mouchet,
        Troncoso-Pastoriza, Hubaux, "Efficient Bootstrapping for Approximate Homomorphic
        Encryption with Non-Sparse Keys", Eurocrypt 2021, Sec. 6; the BSGS split is Halevi and
        Shoup's).  Then each giant partial is rotated (a full single rotation; identity for
        G_j = 1) and the partials are added.  In PQ the baby term for B_k is
            X_k = (acc0_k + P kappa_{B_k}(c0), acc1_k),  acc_k = IP(kappa_{B_k}(ModUp(c1)), key_k),
        with P c0 zero on the special limbs; for B_k = 1 (no rotation) X_k = (P c0, P c1).
        baby_keys[k], giant_keys[j]: (b, key_id), ignored where the Galois element is 1.
        pt: [n_giant][n_baby][ext][N] canonical evaluation-domain plaintexts over q_0..q_l, p_*.
        Returns [2][l+1][N]."""
        na, n, npr = level + 1, self.n, self.n_p
        ext = na + npr
        ct = np.ascontiguousarray(ct, dtype=np.uint32).reshape(2, na, n)
        pt = np.asarray(pt)
        assert pt.shape == (len(giant_g), len(baby_g), ext, n)
        mods = np.array(self.q[:na] + self.p, dtype=np.uint64)[:, None]
        P = 1
        for p in self.p:
            P *= p
        p_mod_q = np.array([P % q for q in self.q[:na]], dtype=np.uint64)[:, None]
        dt = None
        X = []
        for k, g in enumerate(baby_g):
            x = np.zeros((2, ext, n), dtype=np.uint64)
            if g == 1:
                for comp in range(2):
                    x[comp, :na] = (ct[comp].astype(np.uint64) * p_mod_q) % mods[:na]
            else:
                if dt is None:
                    dt = self.modup(ct[1], level, alpha)
                b, key_id = baby_keys[k]
                acc0, acc1 = self.inner_product(self.automorph_eval(dt, g), level, alpha, b, seed, key_id)
                rc0 = self.automorph_eval(ct[0], g).astype(np.uint64)
                x[0] = acc0
                x[0, :na] = (x[0, :na] + rc0 * p_mod_q) % mods[:na]
                x[1] = acc1
            X.append(x)
        out = np.zeros((2, na, n), dtype=np.uint64)
        for j, g in enumerate(giant_g):
            v = np.zeros((2, ext, n), dtype=np.uint64)
            for k in range(len(baby_g)):
                pk = pt[j, k].astype(np.uint64)
                for comp in range(2):
                    v[comp] = (v[comp] + (pk * X[k][comp]) % mods) % mods
            part = np.stack([self.moddown(v[comp].astype(np.uint32), level) for comp in range(2)])
            if g != 1:
                b, key_id = giant_keys[j]
                part = self.rotate(part, level, alpha, g, b, seed, key_id)
            out = (out + part) % mods[:na]
        return out.astype(np.uint32)

    def tensor(self, x, y, level):
        x = np.ascontiguousarray(x, dtype=np.uint32)
        y = np.ascontiguousarray(y, dtype=np.uint32)
        d = np.empty((3, level + 1, self.n), dtype=np.uint32)
        lib().or_tensor(self._h, _u32(x), _u32(y), level, _u32(d))
        return d

    # --- keys and encryption
    def signed_to_eval(self, v: np.ndarray, limbs) -> np.ndarray:
        v = np.ascontiguousarray(v, dtype=np.int64)
        out = np.empty((len(limbs), self.n), dtype=np.uint32)
        for i, t in enumerate(limbs):
            lib().or_signed_to_eval(self._h, _i64(v), t, _u32(out[i]))
        return out

    def secret_eval(self, s: np.ndarray) -> np.ndarray:
        """s in the evaluation domain over the whole chain [n_q+n_p][N]."""
        return self.signed_to_eval(s, range(self.n_q + self.n_p))

    def keygen(self, alpha: int, s: np.ndarray, s2_eval: np.ndarray, e: np.ndarray,
               seed: bytes, key_id: int, want_a: bool = False):
        nt = self.n_q + self.n_p
        nd = -(-self.n_q // alpha)
        s = np.ascontiguousarray(s, dtype=np.int64)
        e = np.ascontiguousarray(e, dtype=np.int64).reshape(nd, self.n)
        s2 = np.ascontiguousarray(s2_eval, dtype=np.uint32)
        b = np.empty((nd, nt, self.n), dtype=np.uint32)
        a = np.empty((nd, nt, self.n), dtype=np.uint32) if want_a else None
        sp, _keep = _u8(seed)
        lib().or_keygen(self._h, alpha, _i64(s), _u32(s2), _i64(e), sp, key_id, _u32(b),
                        _u32(a) if want_a else None)
        return (b, a) if want_a else b

    def encrypt(self, s, m, e, a, level):
        na = level + 1
        a = np.ascontiguousarray(a, dtype=np.uint32).reshape(na, self.n)
        ct = np.empty((2, na, self.n), dtype=np.uint32)
        lib().or_encrypt(self._h, _i64(np.ascontiguousarray(s, dtype=np.int64)),
                         _i64(np.ascontiguousarray(m, dtype=np.int64)),
                         _i64(np.ascontiguousarray(e, dtype=np.int64)), _u32(a), level, _u32(ct))
        return ct

    def decrypt_residues(self, ct, level, s_eval):
        ct = np.ascontiguousarray(ct, dtype=np.uint32)
        n_comp = ct.shape[0]
        out = np.empty((level + 1, self.n), dtype=np.uint32)
        lib().or_decrypt(self._h, _u32(ct), n_comp, level, _u32(np.ascontiguousarray(s_eval)),
                         _u32(out))
        return out

    def crt_centered(self, res: np.ndarray, limbs) -> list:
        """Centred CRT lift (Python integers) of residues [len(limbs)][N]."""
        mods = [self.mod[t] for t in limbs]
        Q = 1
        for m in mods:
            Q *= m
        acc = [0] * self.n
        for i, m in enumerate(mods):
            qi = Q // m
            ci = qi * pow(qi % m, -1, m)
            row = res[i].tolist()
            acc = [(a + r * ci) for a, r in zip(acc, row)]
        half = Q // 2
        out = []
        for a in acc:
            a %= Q
            out.append(a - Q if a > half else a)
        return out

    def decrypt(self, ct, level, s_eval) -> list:
        res = self.decrypt_residues(ct, level, s_eval)
        return self.crt_centered(res, range(level + 1))


# ----------------------------------------------------------------------------- encoding

def _slot_exponents(n: int) -> np.ndarray:
    """e_j = 5^j mod 2N for j < N/2 (the slot j evaluation point is zeta^(e_j))."""
    e = np.empty(n // 2, dtype=np.int64)
    v = 1
    for j in range(n // 2):
        e[j] = v
        v = (v * 5) % (2 * n)
    return e


def encode(z: np.ndarray, n: int, scale: float) -> np.ndarray:
    """CKKS encoding m = round(scale * tau^-1(z)), tau evaluating at zeta^(5^j) and at the
    conjugate points zeta^(-5^j), zeta = exp(i*pi/N).  Coefficients:
    m_n = (scale/N) * sum_{odd e} w_e * zeta^(-e*n) with w_(5^j) = z_j, w_(-5^j) = conj(z_j),
    evaluated with one length-N FFT (e = 2k+1).  Rounded half away from zero."""
    ej = _slot_exponents(n)
    W = np.zeros(n, dtype=np.complex128)
    W[(ej - 1) // 2] = z
    W[((2 * n - ej) - 1) // 2] = np.conj(z)
    k = np.arange(n)
    zeta_neg = np.exp(-1j * np.pi * k / n)
    m = (scale / n) * zeta_neg * np.fft.fft(W)
    r = m.real
    return (np.sign(r) * np.floor(np.abs(r) + 0.5)).astype(np.int64)


def decode(m, n: int, scale: float) -> np.ndarray:
    """z_j = m(zeta^(5^j)) / scale for a real coefficient vector m (floats or ints)."""
    ej = _slot_exponents(n)
    mf = np.array([float(x) for x in m], dtype=np.float64)
    k = np.arange(n)
    v = n * np.fft.ifft(mf * np.exp(1j * np.pi * k / n))
    return v[(ej - 1) // 2] / scale
