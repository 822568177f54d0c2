"""Workload definitions and seeded input generators for the key-switching configurations.

This module is shared by the CPU oracle, the tests and the benchmark.  It holds the parameters
of the five configurations and the random draws that the method takes as inputs (secrets,
errors, encryption randomness, message slots, synthetic residues).  It holds none of the
method's arithmetic: no modular reduction of method data, no NTT, no key derivation.  Both the
oracle and the CUDA library compute everything else on their own.

Workloads (named by ring size and shape):

* ``n12-dnum2``    -- N=2^12, 4 ciphertext primes + 1 special prime, dnum=2, h=64, scale 2^25,
  one rotation by 1 and one relinearisation.
* ``n12-dnum4``    -- the same chain with dnum=4 (one prime per digit).  With dnum=2 a single
  special prime P ~ 2^30 is far below the digit modulus ~ 2^60, so n12-dnum2 cannot decrypt
  to 2^-10; n12-dnum4 carries the decode-accuracy check on the same chain.
* ``n14-hoisted8`` -- N=2^14, 12 + 4 primes, dnum=3, scale 2^28; 8 hoisted rotations
  (+-1, +-2, +-4, +-8) and one ct x ct multiply then relinearisation.
* ``n16-full``     -- N=2^16, 36 + 12 primes, dnum=3, h=192, scale 2^28; a single rotation and a
  single relinearisation at full level (35).
* ``n16-bsgs32``   -- the N=2^16 chain at level 24 with dnum=4: 32 hoisted rotations of one
  ciphertext, baby steps 1..16 and giant steps 16*k for k=2..17 (32 distinct keys).
* ``n16-stream64`` -- the N=2^16 chain at level 20 with dnum=4: 64 independent ct x ct tensor
  products, each relinearised and then rotated by 2^(i mod 15); slots Gaussian sigma=1
  clipped to [-4, 4].
* ``n12-boot``     -- a test chain for the whole bootstrap: N=2^12, 24 + 6 primes, dnum=4, a
  level-0 ciphertext at scale 2^29 raised to level 23.  Its secret has Hamming weight 2, which is
  insecure and chosen on purpose: the raised plaintext m + q_0 I then has |I| <= 1, inside the
  range on which the 12-level EvalMod (degree 12, three double angles) is accurate, so that the
  output can be decoded and compared with the input.
* ``n16-boot``     -- the same on the N=2^16 chain of n16-full with dnum=4 (the benchmark's bootstrap
  shape): level 0 -> 35 -> 17, secret of Hamming weight 2.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class Config:
    key: str
    log_n: int
    n_q: int              # ciphertext primes q_0..q_{n_q-1}
    n_p: int              # special primes p_0..p_{n_p-1}
    dnum: int             # number of gadget digits the keys are generated with
    level: int            # active level: level+1 ciphertext limbs
    h: int                # Hamming weight of the ternary secret
    sigma: float          # error standard deviation
    log_scale: int        # encoding scale Delta = 2^log_scale
    slots: str            # "uniform" or "gauss_clip4"
    rot_steps: tuple = ()          # rotation steps (slot shift r; negative = right)
    hoisted: bool = False          # rotations share one ModUp
    n_pairs: int = 0               # number of independent ct x ct pairs (n16-stream64)
    relin: bool = True
    seed: int = 0                  # RNG seed of the workload's draws

    @property
    def n(self) -> int:
        return 1 << self.log_n

    @property
    def alpha(self) -> int:
        """Primes per gadget digit: ceil((L+1)/dnum)."""
        return -(-self.n_q // self.dnum)

    @property
    def chacha_seed(self) -> bytes:
        return chacha_seed(self.key)


def _stream_steps() -> tuple:
    return tuple(1 << (i % 15) for i in range(64))


CONFIGS = {
    "n12-dnum2": Config("n12-dnum2", 12, 4, 1, 2, 3, 64, 3.2, 25, "uniform", rot_steps=(1,), seed=1001),
    "n12-dnum4": Config("n12-dnum4", 12, 4, 1, 4, 3, 64, 3.2, 25, "uniform", rot_steps=(1,), seed=1011),
    "n14-hoisted8": Config("n14-hoisted8", 14, 12, 4, 3, 11, 192, 3.2, 28, "uniform",
                           rot_steps=(1, -1, 2, -2, 4, -4, 8, -8), hoisted=True, seed=1002),
    "n16-full": Config("n16-full", 16, 36, 12, 3, 35, 192, 3.2, 28, "uniform", rot_steps=(1,), seed=1003),
    "n16-bsgs32": Config("n16-bsgs32", 16, 36, 12, 4, 24, 192, 3.2, 28, "uniform",
                         rot_steps=tuple(range(1, 17)) + tuple(16 * k for k in range(2, 18)),
                         hoisted=True, relin=False, seed=1004),
    "n16-stream64": Config("n16-stream64", 16, 36, 12, 4, 20, 192, 3.2, 28, "gauss_clip4",
                           rot_steps=_stream_steps(), n_pairs=64, seed=1005),
    "n12-boot": Config("n12-boot", 12, 24, 6, 4, 23, 2, 3.2, 29, "uniform", relin=False, seed=1006),
    "n16-boot": Config("n16-boot", 16, 36, 12, 4, 35, 2, 3.2, 29, "uniform", relin=False, seed=1007),
}


def chacha_seed(key: str) -> bytes:
    """32-byte key-expansion seed: SHA-256 of the ASCII string ``fhe-ks-evk/<workload name>``."""
    return hashlib.sha256(f"fhe-ks-evk/{key}".encode("ascii")).digest()


def rng(seed: int, *tags: int) -> np.random.Generator:
    """Independent PCG64 stream for (seed, tag, tag, ...); tags separate the draws."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *tags])))


# Tags for the draws, so each purpose gets its own stream.
TAG_SECRET, TAG_KEY_ERR, TAG_ENC_A, TAG_ENC_ERR, TAG_SLOTS, TAG_SYNTH = 1, 2, 3, 4, 5, 6


def ternary_secret(n: int, h: int, gen: np.random.Generator) -> np.ndarray:
    """Ternary secret with exactly h nonzero coefficients, each +-1, at uniform positions."""
    s = np.zeros(n, dtype=np.int64)
    pos = gen.choice(n, size=h, replace=False)
    s[pos] = gen.choice(np.array([-1, 1], dtype=np.int64), size=h)
    return s


def gaussian_error(n: int, sigma: float, gen: np.random.Generator, count: int = 1) -> np.ndarray:
    """Rounded continuous Gaussian of standard deviation sigma, truncated at 6 sigma.

    Draws beyond 6 sigma are redrawn.  Returns int64 of shape [count, n]."""
    x = gen.normal(0.0, sigma, size=(count, n))
    bad = np.abs(x) > 6 * sigma
    while bad.any():
        x[bad] = gen.normal(0.0, sigma, size=int(bad.sum()))
        bad = np.abs(x) > 6 * sigma
    return np.rint(x).astype(np.int64)


def uniform_residues(moduli, n: int, gen: np.random.Generator) -> np.ndarray:
    """uint32 [len(moduli)][n], row t uniform in [0, moduli[t])."""
    out = np.empty((len(moduli), n), dtype=np.uint32)
    for t, m in enumerate(moduli):
        out[t] = gen.integers(0, int(m), size=n, dtype=np.uint64).astype(np.uint32)
    return out


def slots(cfg: Config, gen: np.random.Generator) -> np.ndarray:
    """N/2 complex message slots: both parts U[-1,1], or N(0,1) clipped to [-4,4]."""
    m = cfg.n // 2
    if cfg.slots == "uniform":
        re = gen.uniform(-1.0, 1.0, size=m)
        im = gen.uniform(-1.0, 1.0, size=m)
    elif cfg.slots == "gauss_clip4":
        re = np.clip(gen.normal(0.0, 1.0, size=m), -4.0, 4.0)
        im = np.clip(gen.normal(0.0, 1.0, size=m), -4.0, 4.0)
    else:
        raise ValueError(cfg.slots)
    return re + 1j * im


def random_bytes(n: int, gen: np.random.Generator) -> bytes:
    return gen.integers(0, 256, size=n, dtype=np.uint8).tobytes()
