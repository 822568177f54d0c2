"""Oracle-built inputs and expected outputs for a workload configuration.

TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU-baseline leg).  Everything here is
computed by the CPU oracle from the seeded draws of ``workloads``; nothing comes from the
CUDA library.

Keys: the relinearisation key switches s^2 -> s (key_id 0); the rotation key for Galois
element g switches kappa_g(s) -> s (key_id g).  Ciphertexts: secret-key encryptions of the
encoded slots at the configuration's level.
"""
from __future__ import annotations

from functools import cached_property

import numpy as np

import workloads as W
from . import Ctx, encode, decode


class Scenario:
    def __init__(self, cfg: W.Config, ctx: Ctx | None = None):
        self.cfg = cfg
        self.ctx = ctx or Ctx(cfg.log_n, cfg.n_q, cfg.n_p)
        self.alpha = cfg.alpha
        self.level = cfg.level
        self.n = cfg.n
        self.scale = float(2 ** cfg.log_scale)
        self.seed_bytes = cfg.chacha_seed
        self.n_digits_full = -(-cfg.n_q // self.alpha)

    # --- secret
    @cached_property
    def s(self) -> np.ndarray:
        return W.ternary_secret(self.n, self.cfg.h, W.rng(self.cfg.seed, W.TAG_SECRET))

    @cached_property
    def s_eval(self) -> np.ndarray:
        return self.ctx.secret_eval(self.s)

    def _s2_eval(self) -> np.ndarray:
        mods = np.array(self.ctx.mod, dtype=np.uint64)[:, None]
        se = self.s_eval.astype(np.uint64)
        return ((se * se) % mods).astype(np.uint32)

    # --- keys
    def key(self, key_id: int, want_a: bool = False):
        """Key-switching key: key_id 0 = relinearisation (s^2), odd g = rotation by kappa_g."""
        if key_id == 0:
            s2 = self._s2_eval()
        else:
            s2 = self.ctx.automorph_eval(self.s_eval, key_id)
        e = W.gaussian_error(self.n, self.cfg.sigma, W.rng(self.cfg.seed, W.TAG_KEY_ERR, key_id),
                             count=self.n_digits_full)
        return self.ctx.keygen(self.alpha, self.s, s2, e, self.seed_bytes, key_id, want_a=want_a)

    # --- ciphertexts
    def slots(self, index: int) -> np.ndarray:
        return W.slots(self.cfg, W.rng(self.cfg.seed, W.TAG_SLOTS, index))

    def encrypt_slots(self, z: np.ndarray, index: int, level: int | None = None) -> np.ndarray:
        level = self.level if level is None else level
        m = encode(z, self.n, self.scale)
        e = W.gaussian_error(self.n, self.cfg.sigma, W.rng(self.cfg.seed, W.TAG_ENC_ERR, index))[0]
        a = W.uniform_residues(self.ctx.q[: level + 1], self.n, W.rng(self.cfg.seed, W.TAG_ENC_A, index))
        return self.ctx.encrypt(self.s, m, e, a, level)

    def ciphertext(self, index: int, level: int | None = None):
        z = self.slots(index)
        return z, self.encrypt_slots(z, index, level)

    def decrypt_slots(self, ct: np.ndarray, level: int | None = None, scale: float | None = None):
        level = self.level if level is None else level
        m = self.ctx.decrypt(ct, level, self.s_eval)
        return decode(m, self.n, self.scale if scale is None else scale)

    def galois(self, r: int) -> int:
        return self.ctx.galois(r)
