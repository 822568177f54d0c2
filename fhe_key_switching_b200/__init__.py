"""B200 (sm_100a) RNS-CKKS hybrid key switching with in-kernel ChaCha12 key regeneration.

Thin Python binding of the C ABI in ``include/ckks_ks.h`` (argument marshalling only: every
step of the key-switching path runs in the library's CUDA kernels).  PyTorch supplies device
memory and streams.  The functions keep the C names; buffers are CUDA tensors of dtype
uint32 or int32 (reinterpreted), contiguous, laid out as the header states.

There is no CPU fallback: if the compiled library is missing, importing this package raises.

``FHE_KS_B200_BUILD=debug`` in the environment loads the debug-bounds build of the same sources
(``libckks_ks_debug.so``, from ``python fhe_key_switching_b200/build.py --debug``), whose kernels
check every access span against the call's buffers (see ckks_debug_bounds_report).
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
BUILD = os.environ.get("FHE_KS_B200_BUILD", "release")
if BUILD not in ("release", "debug"):
    raise ImportError(f"FHE_KS_B200_BUILD={BUILD!r}: expected 'release' or 'debug'")
LIB_PATH = os.path.join(_HERE, "_build", "libckks_ks_debug.so" if BUILD == "debug" else "libckks_ks.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"CUDA library {LIB_PATH} is not built; run `python fhe_key_switching_b200/build.py"
        f"{' --debug' if BUILD == 'debug' else ''}` (nvcc, sm_100a) or `python __graft_entry__.py` first")

_L = ctypes.CDLL(LIB_PATH)

CKKS_OK, CKKS_ERR_ARG, CKKS_ERR_UNSUPPORTED, CKKS_ERR_ALIGN = 0, -1, -2, -3
CKKS_ERR_WORKSPACE, CKKS_ERR_CUDA, CKKS_ERR_TIMEOUT, CKKS_ERR_BOUNDS = -4, -5, -6, -7

_u32p = ctypes.POINTER(ctypes.c_uint32)
_vp = ctypes.c_void_p
_ci, _cu, _sz = ctypes.c_int, ctypes.c_uint32, ctypes.c_size_t


class ckks_params(ctypes.Structure):
    _fields_ = [("log_n", _cu), ("n_q", _cu), ("n_p", _cu), ("dnum", _cu),
                ("q", _u32p), ("p", _u32p)]


class ckks_evk(ctypes.Structure):
    _fields_ = [("b", _vp), ("a", _vp), ("seed", ctypes.c_uint8 * 32), ("key_id", _cu)]


class ckks_bsgs_level(ctypes.Structure):
    _fields_ = [("n_baby", _ci), ("baby_galois", _u32p), ("baby_keys", ctypes.POINTER(ckks_evk)),
                ("n_giant", _ci), ("giant_galois", _u32p), ("giant_keys", ctypes.POINTER(ckks_evk)), ("pt", _vp)]


class ckks_bootstrap_plan(ctypes.Structure):
    _fields_ = [("top_level", _ci), ("n_c2s", _ci), ("c2s", ctypes.POINTER(ckks_bsgs_level)), ("n_s2c", _ci),
                ("s2c", ctypes.POINTER(ckks_bsgs_level)), ("conj_key", ctypes.POINTER(ckks_evk)),
                ("relin_key", ctypes.POINTER(ckks_evk)), ("r", _ci), ("d", _ci)]


_SIGS = {
    "ckks_gen_primes": (_ci, [_cu, _cu, _cu, _u32p, _u32p]),
    "ckks_ctx_create": (_ci, [ctypes.POINTER(ckks_params), ctypes.POINTER(_vp)]),
    "ckks_ctx_destroy": (None, [_vp]),
    "ckks_ntt_fwd": (_ci, [_vp, _vp, _ci, _ci, _vp]),
    "ckks_ntt_inv": (_ci, [_vp, _vp, _ci, _ci, _vp]),
    "ckks_automorph": (_ci, [_vp, _vp, _vp, _ci, _cu, _vp]),
    "ckks_modup": (_ci, [_vp, _vp, _ci, _vp, _vp, _sz, _vp]),
    "ckks_inner_product": (_ci, [_vp, _vp, _ci, ctypes.POINTER(ckks_evk), _vp, _vp]),
    "ckks_moddown": (_ci, [_vp, _vp, _ci, _vp, _vp, _sz, _vp]),
    "ckks_keyswitch": (_ci, [_vp, _vp, _ci, ctypes.POINTER(ckks_evk), _vp, _vp, _sz, _vp]),
    "ckks_rotate": (_ci, [_vp, _vp, _ci, _cu, ctypes.POINTER(ckks_evk), _vp, _vp, _sz, _vp]),
    "ckks_rotate_hoisted": (_ci, [_vp, _vp, _ci, _ci, _u32p, ctypes.POINTER(ckks_evk), _vp, _vp,
                                  _sz, _vp]),
    "ckks_rotate_hoisted_batch": (_ci, [_vp, _ci, _vp, _ci, _ci, _u32p, ctypes.POINTER(ckks_evk), _vp, _vp,
                                        _sz, _vp]),
    "ckks_relin": (_ci, [_vp, _vp, _ci, ctypes.POINTER(ckks_evk), _vp, _vp, _sz, _vp]),
    "ckks_keyswitch_batch": (_ci, [_vp, _ci, _vp, _ci, ctypes.POINTER(ckks_evk), _vp, _vp, _sz, _vp]),
    "ckks_rotate_batch": (_ci, [_vp, _ci, _vp, _ci, _u32p, ctypes.POINTER(ckks_evk), _vp, _vp, _sz, _vp]),
    "ckks_relin_batch": (_ci, [_vp, _ci, _vp, _ci, ctypes.POINTER(ckks_evk), _vp, _vp, _sz, _vp]),
    "ckks_tensor_batch": (_ci, [_vp, _ci, _vp, _vp, _ci, _vp, _vp]),
    "ckks_tensor": (_ci, [_vp, _vp, _vp, _ci, _vp, _vp]),
    "ckks_rescale": (_ci, [_vp, _vp, _ci, _vp, _vp, _sz, _vp]),
    "ckks_bsgs_workspace_bytes": (_sz, [_vp, _ci, _ci, _ci]),
    "ckks_bsgs": (_ci, [_vp, _vp, _ci, _ci, _u32p, ctypes.POINTER(ckks_evk), _ci, _u32p, ctypes.POINTER(ckks_evk),
                        _vp, _vp, _vp, _sz, _vp]),
    "ckks_rescale_batch": (_ci, [_vp, _ci, _vp, _ci, _vp, _vp, _sz, _vp]),
    "ckks_chacha_expand": (_ci, [_vp, ctypes.POINTER(ctypes.c_uint8), _cu, _ci, _ci, _vp, _vp]),
    "ckks_workspace_bytes": (_sz, [_vp, _ci, _ci]),
    "ckks_sync_status": (_ci, [_vp, _vp, _ci]),
    "ckks_selftest_wait_expiry": (_ci, [_vp, _vp]),
    "ckks_selftest_launch_error": (_ci, [_vp, _vp]),
    "ckks_keyswitch_noalloc": (_ci, [_vp, _vp, _ci, ctypes.POINTER(ckks_evk), _vp, _vp]),
    "ckks_prof_begin": (_ci, [_vp, ctypes.c_char_p, _ci]),
    "ckks_prof_end": (_ci, [_vp, ctypes.POINTER(_ci), ctypes.POINTER(ctypes.c_double)]),
    "ckks_set_bconv_mode": (_ci, [_vp, _ci]),
    "ckks_mul_const": (_ci, [_vp, _vp, _ci, _ci, ctypes.c_longlong, _vp, _vp]),
    "ckks_add_const": (_ci, [_vp, _vp, _ci, ctypes.c_longlong, _vp, _vp]),
    "ckks_add": (_ci, [_vp, _vp, _vp, _ci, _ci, _vp, _vp]),
    "ckks_evalmod_workspace_bytes": (_sz, [_vp, _ci]),
    "ckks_evalmod_batch_workspace_bytes": (_sz, [_vp, _ci, _ci]),
    "ckks_evalmod_batch": (_ci, [_vp, _ci, _vp, _ci, ctypes.c_double, _ci, _ci, ctypes.POINTER(ckks_evk), _vp,
                                 ctypes.POINTER(_ci), ctypes.POINTER(ctypes.c_double), _vp, _sz, _vp]),
    "ckks_evalmod": (_ci, [_vp, _vp, _ci, ctypes.c_double, _ci, _ci, ctypes.POINTER(ckks_evk), _vp,
                           ctypes.POINTER(_ci), ctypes.POINTER(ctypes.c_double), _vp, _sz, _vp]),
    "ckks_modraise": (_ci, [_vp, _vp, _ci, _vp, _vp, _sz, _vp]),
    "ckks_mul_i": (_ci, [_vp, _vp, _ci, _ci, _vp, _vp]),
    "ckks_bootstrap_workspace_bytes": (_sz, [_vp, ctypes.POINTER(ckks_bootstrap_plan)]),
    "ckks_bootstrap": (_ci, [_vp, _vp, ctypes.POINTER(ckks_bootstrap_plan), _vp, ctypes.POINTER(_ci),
                             ctypes.POINTER(ctypes.c_double), _vp, _sz, _vp]),
    "ckks_encode": (_ci, [_vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double), ctypes.c_double,
                          _ci, _ci, _vp, _vp, _sz, _vp]),
    "ckks_int_probe": (_ci, [_ci, _ci, _ci, _vp, _vp, ctypes.POINTER(ctypes.c_float),
                             ctypes.POINTER(ctypes.c_double)]),
    "ckks_debug_bounds_enabled": (_ci, []),
    "ckks_debug_bounds_report": (_ci, [ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(_ci),
                                       ctypes.POINTER(ctypes.c_uint64), ctypes.POINTER(ctypes.c_uint64), _ci]),
    "ckks_debug_bounds_site_name": (ctypes.c_char_p, [_ci]),
    "ckks_selftest_bounds": (_ci, [_vp, _vp]),
    "ckks_last_error": (ctypes.c_char_p, []),
}
for _name, (_res, _args) in _SIGS.items():
    _f = getattr(_L, _name)
    _f.restype = _res
    _f.argtypes = _args

EXPORTED = tuple(_SIGS)


class CkksError(RuntimeError):
    def __init__(self, code: int, where: str):
        msg = _L.ckks_last_error().decode(errors="replace")
        super().__init__(f"{where} failed ({code}): {msg}")
        self.code = code


def _check(code: int, where: str) -> int:
    if code != CKKS_OK:
        raise CkksError(code, where)
    return code


def _ptr(t) -> int:
    """Device pointer of a CUDA tensor (no copy, no dtype conversion)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ----------------------------------------------------------------------------- parameters

def ckks_gen_primes(log_n: int, n_q: int, n_p: int):
    """The library's prime chain rule; returns (q list, p list)."""
    q = (ctypes.c_uint32 * max(n_q, 1))()
    p = (ctypes.c_uint32 * max(n_p, 1))()
    _check(_L.ckks_gen_primes(log_n, n_q, n_p, q, p), "ckks_gen_primes")
    return list(q)[:n_q], list(p)[:n_p]


class Context:
    """Owns a ckks_ctx (device tables for one parameter set)."""

    def __init__(self, log_n: int, q, p, dnum: int):
        qa = (ctypes.c_uint32 * len(q))(*q)
        pa = (ctypes.c_uint32 * len(p))(*p)
        prm = ckks_params(log_n, len(q), len(p), dnum, qa, pa)
        h = _vp()
        _check(_L.ckks_ctx_create(ctypes.byref(prm), ctypes.byref(h)), "ckks_ctx_create")
        self.handle = h
        self.log_n, self.n, self.q, self.p, self.dnum = log_n, 1 << log_n, list(q), list(p), dnum
        self.n_q, self.n_p = len(q), len(p)
        self.alpha = -(-self.n_q // dnum)

    def close(self):
        if getattr(self, "handle", None):
            _L.ckks_ctx_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def _as_parameter_(self):
        return self.handle

    def workspace_bytes(self, level: int, n_rot: int = 1) -> int:
        return int(_L.ckks_workspace_bytes(self.handle, level, n_rot))

    def workspace(self, level: int, n_rot: int = 1, device=None):
        import torch
        return torch.empty(self.workspace_bytes(level, n_rot), dtype=torch.uint8,
                           device=device or torch.device("cuda", torch.cuda.current_device()))


def ckks_ctx_create(log_n: int, q, p, dnum: int) -> Context:
    return Context(log_n, q, p, dnum)


def make_evk(b, seed: bytes, key_id: int, a=None) -> ckks_evk:
    """Key-switching key record: b (and optionally a stored a) are CUDA tensors
    [D][n_q+n_p][N].  The record holds references to them, so their device memory stays
    allocated for as long as the record exists (the C struct itself only carries pointers)."""
    k = ckks_evk()
    k.b = _ptr(b)
    k.a = _ptr(a) if a is not None else None
    if len(seed) != 32:
        raise ValueError("seed must be 32 bytes")
    ctypes.memmove(k.seed, seed, 32)
    k.key_id = key_id
    k._tensors = (b, a)
    return k


# ----------------------------------------------------------------------------- operations

def ckks_ntt_fwd(ctx, poly, first_limb: int, n_limbs: int, stream=None):
    _check(_L.ckks_ntt_fwd(ctx.handle, _ptr(poly), first_limb, n_limbs, _stream(stream)), "ckks_ntt_fwd")


def ckks_ntt_inv(ctx, poly, first_limb: int, n_limbs: int, stream=None):
    _check(_L.ckks_ntt_inv(ctx.handle, _ptr(poly), first_limb, n_limbs, _stream(stream)), "ckks_ntt_inv")


def ckks_automorph(ctx, inp, out, n_limbs: int, galois: int, stream=None):
    _check(_L.ckks_automorph(ctx.handle, _ptr(inp), _ptr(out), n_limbs, galois, _stream(stream)),
           "ckks_automorph")


def ckks_modup(ctx, c, level: int, dtilde, ws, stream=None):
    _check(_L.ckks_modup(ctx.handle, _ptr(c), level, _ptr(dtilde), _ptr(ws), ws.numel() * ws.element_size(),
                         _stream(stream)), "ckks_modup")


def ckks_inner_product(ctx, dtilde, level: int, evk: ckks_evk, acc, stream=None):
    _check(_L.ckks_inner_product(ctx.handle, _ptr(dtilde), level, ctypes.byref(evk), _ptr(acc),
                                 _stream(stream)), "ckks_inner_product")


def ckks_moddown(ctx, acc, level: int, out, ws, stream=None):
    _check(_L.ckks_moddown(ctx.handle, _ptr(acc), level, _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                           _stream(stream)), "ckks_moddown")


def ckks_keyswitch(ctx, c, level: int, evk: ckks_evk, out, ws, stream=None):
    _check(_L.ckks_keyswitch(ctx.handle, _ptr(c), level, ctypes.byref(evk), _ptr(out), _ptr(ws),
                             ws.numel() * ws.element_size(), _stream(stream)), "ckks_keyswitch")


def ckks_keyswitch_noalloc(ctx, c, level: int, evk: ckks_evk, out, stream=None):
    """ckks_keyswitch with the library's fixed device workspace: allocates nothing (for callers
    whose host framework owns all device memory); calls must not overlap on the GPU."""
    _check(_L.ckks_keyswitch_noalloc(ctx.handle, _ptr(c), level, ctypes.byref(evk), _ptr(out),
                                     _stream(stream)), "ckks_keyswitch_noalloc")


NOALLOC_SCRATCH_BYTES = 8 << 20


def ckks_rotate(ctx, ct, level: int, galois: int, evk: ckks_evk, out, ws, stream=None):
    _check(_L.ckks_rotate(ctx.handle, _ptr(ct), level, galois, ctypes.byref(evk), _ptr(out), _ptr(ws),
                          ws.numel() * ws.element_size(), _stream(stream)), "ckks_rotate")


def ckks_rotate_hoisted(ctx, ct, level: int, galois, evks, out, ws, stream=None):
    n = len(galois)
    ga = (ctypes.c_uint32 * max(n, 1))(*galois)
    ka = (ckks_evk * max(n, 1))(*evks)
    _check(_L.ckks_rotate_hoisted(ctx.handle, _ptr(ct), level, n, ga, ka, _ptr(out), _ptr(ws),
                                  ws.numel() * ws.element_size(), _stream(stream)), "ckks_rotate_hoisted")


def ckks_relin(ctx, d, level: int, evk: ckks_evk, out, ws, stream=None):
    _check(_L.ckks_relin(ctx.handle, _ptr(d), level, ctypes.byref(evk), _ptr(out), _ptr(ws),
                         ws.numel() * ws.element_size(), _stream(stream)), "ckks_relin")


def ckks_tensor(ctx, x, y, level: int, d, stream=None):
    _check(_L.ckks_tensor(ctx.handle, _ptr(x), _ptr(y), level, _ptr(d), _stream(stream)), "ckks_tensor")


def _evk_array(evks):
    n = len(evks)
    return (ckks_evk * max(n, 1))(*evks)


def ckks_keyswitch_batch(ctx, c, level: int, evks, out, ws, stream=None):
    """Batch of len(evks) key switches: c [n][l+1][N] -> out [n][2][l+1][N]."""
    _check(_L.ckks_keyswitch_batch(ctx.handle, len(evks), _ptr(c), level, _evk_array(evks), _ptr(out), _ptr(ws),
                                   ws.numel() * ws.element_size(), _stream(stream)), "ckks_keyswitch_batch")


def ckks_rotate_batch(ctx, ct, level: int, galois, evks, out, ws, stream=None):
    """Batch of rotations: ct [n][2][l+1][N], galois and evks of n entries -> out [n][2][l+1][N]."""
    n = len(galois)
    ga = (ctypes.c_uint32 * max(n, 1))(*galois)
    _check(_L.ckks_rotate_batch(ctx.handle, n, _ptr(ct), level, ga, _evk_array(evks), _ptr(out), _ptr(ws),
                                ws.numel() * ws.element_size(), _stream(stream)), "ckks_rotate_batch")


def ckks_relin_batch(ctx, d, level: int, evks, out, ws, stream=None):
    """Batch of relinearisations: d [n][3][l+1][N] -> out [n][2][l+1][N]."""
    _check(_L.ckks_relin_batch(ctx.handle, len(evks), _ptr(d), level, _evk_array(evks), _ptr(out), _ptr(ws),
                               ws.numel() * ws.element_size(), _stream(stream)), "ckks_relin_batch")


def ckks_tensor_batch(ctx, n: int, x, y, level: int, d, stream=None):
    """Batch of tensor products: x, y [n][2][l+1][N] -> d [n][3][l+1][N]."""
    _check(_L.ckks_tensor_batch(ctx.handle, n, _ptr(x), _ptr(y), level, _ptr(d), _stream(stream)),
           "ckks_tensor_batch")


def ckks_rescale(ctx, ct, level: int, out, ws, stream=None):
    """Rescale by q_level: ct [2][l+1][N] -> out [2][l][N]."""
    _check(_L.ckks_rescale(ctx.handle, _ptr(ct), level, _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                           _stream(stream)), "ckks_rescale")


def ckks_rescale_batch(ctx, n: int, ct, level: int, out, ws, stream=None):
    """Batch of rescales: ct [n][2][l+1][N] -> out [n][2][l][N]."""
    _check(_L.ckks_rescale_batch(ctx.handle, n, _ptr(ct), level, _ptr(out), _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream)), "ckks_rescale_batch")


def ckks_bsgs_workspace(ctx, level: int, n_baby: int, n_giant: int, device=None):
    import torch
    nb = int(_L.ckks_bsgs_workspace_bytes(ctx.handle, level, n_baby, n_giant))
    if nb == 0:
        raise ValueError("ckks_bsgs_workspace_bytes: arguments out of range")
    return torch.empty(nb, dtype=torch.uint8,
                       device=device or torch.device("cuda", torch.cuda.current_device()))


def ckks_bsgs(ctx, ct, level: int, baby_galois, baby_evks, giant_galois, giant_evks, pt, out, ws, stream=None):
    """Baby-step giant-step transform: out = sum_j rot_Gj(sum_k pt[j][k] * rot_Bk(ct)).
    baby_evks / giant_evks: one ckks_evk per step (None where the Galois element is 1)."""
    nb, ng = len(baby_galois), len(giant_galois)
    empty = ckks_evk()
    bk = (ckks_evk * nb)(*[e if e is not None else empty for e in baby_evks])
    gk = (ckks_evk * ng)(*[e if e is not None else empty for e in giant_evks])
    bg = (ctypes.c_uint32 * nb)(*baby_galois)
    gg = (ctypes.c_uint32 * ng)(*giant_galois)
    _check(_L.ckks_bsgs(ctx.handle, _ptr(ct), level, nb, bg, bk, ng, gg, gk, _ptr(pt), _ptr(out), _ptr(ws),
                        ws.numel() * ws.element_size(), _stream(stream)), "ckks_bsgs")


def ckks_chacha_expand(ctx, seed: bytes, key_id: int, digit: int, limb: int, out, stream=None):
    sb = (ctypes.c_uint8 * 32).from_buffer_copy(seed)
    _check(_L.ckks_chacha_expand(ctx.handle, sb, key_id, digit, limb, _ptr(out), _stream(stream)),
           "ckks_chacha_expand")


def ckks_sync_status(ctx, stream=None, timeout_ms: int = 10000) -> int:
    return int(_L.ckks_sync_status(ctx.handle if ctx is not None else None, _stream(stream), timeout_ms))


def ckks_selftest_wait_expiry(ctx, stream=None):
    _check(_L.ckks_selftest_wait_expiry(ctx.handle, _stream(stream)), "ckks_selftest_wait_expiry")


def ckks_selftest_launch_error(ctx, stream=None) -> int:
    """The status of a launch the CUDA runtime rejects (CKKS_ERR_CUDA); see ckks_last_error()."""
    return int(_L.ckks_selftest_launch_error(ctx.handle, _stream(stream)))


def ckks_last_error() -> str:
    return _L.ckks_last_error().decode(errors="replace")


def ckks_debug_bounds_enabled() -> bool:
    return bool(_L.ckks_debug_bounds_enabled())


def ckks_debug_bounds_report(clear: bool = True):
    """(failed checks, first site's name, its address, its size in bytes) since the last clear."""
    count, site, addr, nbytes = ctypes.c_uint64(), _ci(), ctypes.c_uint64(), ctypes.c_uint64()
    _check(_L.ckks_debug_bounds_report(ctypes.byref(count), ctypes.byref(site), ctypes.byref(addr),
                                       ctypes.byref(nbytes), int(clear)), "ckks_debug_bounds_report")
    name = _L.ckks_debug_bounds_site_name(site.value).decode()
    return int(count.value), name, int(addr.value), int(nbytes.value)


def ckks_debug_bounds_site_name(site: int) -> str:
    return _L.ckks_debug_bounds_site_name(site).decode()


def ckks_selftest_bounds(ctx, stream=None):
    _check(_L.ckks_selftest_bounds(ctx.handle, _stream(stream)), "ckks_selftest_bounds")


def ckks_prof_begin(ctx, kernel: str, max_launches: int):
    _check(_L.ckks_prof_begin(ctx.handle, kernel.encode(), max_launches), "ckks_prof_begin")


def ckks_prof_end(ctx):
    """(launches, total_ms) recorded since ckks_prof_begin."""
    n = _ci()
    ms = ctypes.c_double()
    _check(_L.ckks_prof_end(ctx.handle, ctypes.byref(n), ctypes.byref(ms)), "ckks_prof_end")
    return n.value, ms.value


def ckks_encode(ctx, slots, scale: float, level: int, out, ws, with_special: bool = False, stream=None):
    """CKKS encoding of N/2 complex slots (a host sequence of complex numbers) at `scale` into out
    [(level+1) (+ n_p)][N] (CUDA uint32, evaluation domain); ws: CUDA buffer of >= 8 N bytes."""
    n = len(slots)
    if n != ctx.n // 2:
        raise ValueError(f"expected N/2 = {ctx.n // 2} slots, got {n}")
    re = (ctypes.c_double * n)(*[complex(v).real for v in slots])
    im = (ctypes.c_double * n)(*[complex(v).imag for v in slots])
    _check(_L.ckks_encode(ctx.handle, re, im, float(scale), level, 1 if with_special else 0, _ptr(out), _ptr(ws),
                          ws.numel() * ws.element_size(), _stream(stream)), "ckks_encode")


def ckks_mul_const(ctx, ct, n_comp: int, level: int, v: int, out, stream=None):
    _check(_L.ckks_mul_const(ctx.handle, _ptr(ct), n_comp, level, v, _ptr(out), _stream(stream)), "ckks_mul_const")


def ckks_add_const(ctx, ct, level: int, v: int, out, stream=None):
    _check(_L.ckks_add_const(ctx.handle, _ptr(ct), level, v, _ptr(out), _stream(stream)), "ckks_add_const")


def ckks_add(ctx, x, y, n_comp: int, level: int, out, stream=None):
    _check(_L.ckks_add(ctx.handle, _ptr(x), _ptr(y), n_comp, level, _ptr(out), _stream(stream)), "ckks_add")


def ckks_evalmod_workspace(ctx, level: int, device=None):
    import torch
    nb = int(_L.ckks_evalmod_workspace_bytes(ctx.handle, level))
    if nb == 0:
        raise ValueError("ckks_evalmod_workspace_bytes: level out of range")
    return torch.empty(nb, dtype=torch.uint8, device=device or torch.device("cuda", torch.cuda.current_device()))


def ckks_evalmod(ctx, ct, level: int, scale: float, r: int, d: int, relin_evk: ckks_evk, out, ws, stream=None):
    """EvalMod: out's slots ~ sin(2 pi x) / (2 pi) for ct's real slots x; returns (out_level, out_scale)."""
    lv = _ci()
    sc = ctypes.c_double()
    _check(_L.ckks_evalmod(ctx.handle, _ptr(ct), level, float(scale), r, d, ctypes.byref(relin_evk), _ptr(out),
                           ctypes.byref(lv), ctypes.byref(sc), _ptr(ws), ws.numel() * ws.element_size(),
                           _stream(stream)), "ckks_evalmod")
    return lv.value, sc.value


def ckks_evalmod_batch_workspace(ctx, level: int, n: int, device=None):
    import torch
    nb = int(_L.ckks_evalmod_batch_workspace_bytes(ctx.handle, level, n))
    if nb == 0:
        raise ValueError("ckks_evalmod_batch_workspace_bytes: level or batch out of range")
    return torch.empty(nb, dtype=torch.uint8, device=device or torch.device("cuda", torch.cuda.current_device()))


def ckks_evalmod_batch(ctx, ct, level: int, scale: float, r: int, d: int, relin_evk: ckks_evk, out, ws,
                       stream=None):
    """EvalMod on the n ciphertexts of ct [n][2][level+1][N]; returns (out_level, out_scale)."""
    lv = _ci()
    sc = ctypes.c_double()
    _check(_L.ckks_evalmod_batch(ctx.handle, int(ct.shape[0]), _ptr(ct), level, float(scale), r, d,
                                 ctypes.byref(relin_evk), _ptr(out), ctypes.byref(lv), ctypes.byref(sc), _ptr(ws),
                                 ws.numel() * ws.element_size(), _stream(stream)), "ckks_evalmod_batch")
    return lv.value, sc.value


def ckks_modraise(ctx, ct, level: int, out, ws, stream=None):
    """ModRaise: ct [2][1][N] at level 0 -> out [2][level+1][N] (centred lift of the q_0 residues)."""
    _check(_L.ckks_modraise(ctx.handle, _ptr(ct), level, _ptr(out), _ptr(ws), ws.numel() * ws.element_size(),
                            _stream(stream)), "ckks_modraise")


CKKS_BCONV_CUDA_CORES, CKKS_BCONV_TENSOR, CKKS_BCONV_AUTO = 0, 1, 2


def ckks_set_bconv_mode(ctx, mode: int):
    """Base-conversion engine of later calls on ctx: CKKS_BCONV_AUTO (default: the tensor cores for
    large launches), CKKS_BCONV_TENSOR (8-bit contraction on the tensor cores) or
    CKKS_BCONV_CUDA_CORES; same output bits either way."""
    _check(_L.ckks_set_bconv_mode(ctx.handle, mode), "ckks_set_bconv_mode")


def ckks_int_probe(op: int, blocks: int, iters: int, sink, stream=None):
    """One integer-throughput probe launch (a measurement aid): returns (elapsed ms, operations).
    sink: CUDA uint32 tensor of blocks * 256 words."""
    if sink.numel() < blocks * 256:
        raise ValueError("sink must hold blocks * 256 words")
    ms = ctypes.c_float()
    ops = ctypes.c_double()
    code = _L.ckks_int_probe(op, blocks, iters, _ptr(sink), _stream(stream), ctypes.byref(ms), ctypes.byref(ops))
    if code != CKKS_OK:
        raise CkksError(code, "ckks_int_probe")
    return ms.value, ops.value


def galois_element(log_n: int, r: int) -> int:
    """Galois element of a rotation by r slots: 5^r mod 2N (r < 0: 5^(N/2+r))."""
    n = 1 << log_n
    return pow(5, r % (n // 2), 2 * n)


def conjugation_element(log_n: int) -> int:
    """Galois element of complex conjugation of the slots: 2N - 1 (X -> X^-1); its key has
    key_id 2N - 1 and it runs through ckks_rotate like any rotation."""
    return (2 << log_n) - 1


def ckks_mul_i(ctx, ct, n_comp: int, level: int, out, stream=None):
    """out = X^(N/2) ct: every slot times i."""
    _check(_L.ckks_mul_i(ctx.handle, _ptr(ct), n_comp, level, _ptr(out), _stream(stream)), "ckks_mul_i")


class BootstrapPlan:
    """Holds a ckks_bootstrap_plan and the host arrays and tensors it points to.
    c2s, s2c: per level (baby Galois elements, baby evks, giant Galois elements, giant evks, pt tensor),
    None standing for the key of element 1; conj_evk, relin_evk: ckks_evk."""

    def __init__(self, top_level: int, c2s, s2c, conj_evk, relin_evk, r: int, d: int):
        empty = ckks_evk()
        self._keep = []

        def levels(lst):
            arr = (ckks_bsgs_level * len(lst))()
            for i, (bg, bk, gg, gk, pt) in enumerate(lst):
                bga = (ctypes.c_uint32 * len(bg))(*bg)
                gga = (ctypes.c_uint32 * len(gg))(*gg)
                bka = (ckks_evk * len(bk))(*[e if e is not None else empty for e in bk])
                gka = (ckks_evk * len(gk))(*[e if e is not None else empty for e in gk])
                self._keep += [bga, gga, bka, gka, pt]
                arr[i] = ckks_bsgs_level(len(bg), bga, bka, len(gg), gga, gka, _ptr(pt))
            self._keep.append(arr)
            return arr

        self._conj, self._relin = conj_evk, relin_evk
        self.plan = ckks_bootstrap_plan(top_level, len(c2s), levels(c2s), len(s2c), levels(s2c),
                                        ctypes.pointer(self._conj), ctypes.pointer(self._relin), r, d)
        self.out_level = top_level - len(c2s) - (d + r + 3) - len(s2c)


def ckks_bootstrap_workspace(ctx, plan: BootstrapPlan, device=None):
    import torch
    nbytes = _L.ckks_bootstrap_workspace_bytes(ctx.handle, ctypes.byref(plan.plan))
    if nbytes == 0:
        raise CkksError(CKKS_ERR_ARG, "ckks_bootstrap_workspace_bytes")
    return torch.empty((nbytes + 3) // 4, dtype=torch.uint32, device=device or "cuda")


def ckks_bootstrap(ctx, ct, plan: BootstrapPlan, out, ws, stream=None):
    """Bootstraps ct [2][1][N] into out [2][plan.out_level+1][N]; returns (out_level, ratio)."""
    lv, ratio = _ci(), ctypes.c_double()
    _check(_L.ckks_bootstrap(ctx.handle, _ptr(ct), ctypes.byref(plan.plan), _ptr(out), ctypes.byref(lv),
                             ctypes.byref(ratio), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "ckks_bootstrap")
    return lv.value, ratio.value


def ckks_rotate_hoisted_batch(ctx, ct, level: int, galois, evks, out, ws, stream=None):
    """ct [n_ct][2][l+1][N] -> out [n_ct][n_rot][2][l+1][N]: every ciphertext rotated by every
    Galois element, one ModUp per ciphertext."""
    n_rot = len(galois)
    ga = (ctypes.c_uint32 * n_rot)(*galois)
    _check(_L.ckks_rotate_hoisted_batch(ctx.handle, ct.shape[0], _ptr(ct), level, n_rot, ga, _evk_array(evks),
                                        _ptr(out), _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "ckks_rotate_hoisted_batch")
