"""Pins for the oracle's ChaCha core and the key's uniform-half expander.

The 20-round core is checked against the RFC 8439 block vectors (tests/golden) and against an
independent implementation (OpenSSL's ChaCha20 through the `cryptography` package).  The
12-round variant is the same code with another round count; it is pinned by the published
reduced-round vector for the all-zero key (draft-strombergson-chacha-test-vectors, TC1).
"""
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "chacha_vectors.txt")


def _vectors():
    out = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        r, key, ctr, nonce, blk = line.split()
        out.append((int(r), bytes.fromhex(key), int(ctr), bytes.fromhex(nonce), bytes.fromhex(blk)))
    return out


@pytest.mark.parametrize("vec", _vectors(), ids=lambda v: f"r{v[0]}c{v[2]}")
def test_golden_blocks(oracle_mod, vec):
    rounds, key, ctr, nonce, blk = vec
    assert oracle_mod.chacha_block(key, ctr, nonce, rounds) == blk


def test_chacha20_matches_openssl(oracle_mod):
    from cryptography.hazmat.primitives.ciphers import Cipher, algorithms
    rng = np.random.default_rng(7)
    for _ in range(20):
        key = rng.integers(0, 256, 32, dtype=np.uint8).tobytes()
        nonce = rng.integers(0, 256, 12, dtype=np.uint8).tobytes()
        ctr = int(rng.integers(0, 2**32 - 4))
        enc = Cipher(algorithms.ChaCha20(key, ctr.to_bytes(4, "little") + nonce), mode=None).encryptor()
        stream = enc.update(bytes(64 * 3))
        for b in range(3):
            assert oracle_mod.chacha_block(key, ctr + b, nonce, 20) == stream[64 * b: 64 * (b + 1)]


def test_round_count_matters(oracle_mod):
    key, nonce = bytes(range(32)), bytes(12)
    assert oracle_mod.chacha_block(key, 0, nonce, 12) != oracle_mod.chacha_block(key, 0, nonce, 20)


def test_expand_layout(oracle_mod):
    """Coefficient n = 64-bit LE word (n mod 8) of the ChaCha12 block n/8 with nonce
    (key_id, digit, limb), reduced mod q_t; the block itself comes from the pinned core."""
    ctx = oracle_mod.Ctx(6, 3, 2)
    seed = bytes(range(100, 132))
    for (kid, j, t) in [(0, 0, 0), (5, 1, 2), (2**31 + 1, 2, 4)]:
        a = ctx.chacha_expand(seed, kid, j, t)
        q = ctx.mod[t]
        nonce = np.array([kid, j, t], dtype="<u4").tobytes()
        for b in range(ctx.n // 8):
            blk = oracle_mod.chacha_block(seed, b, nonce, 12)
            words = np.frombuffer(blk, dtype="<u8")
            assert [int(w) % q for w in words] == a[8 * b: 8 * b + 8].tolist()
        assert a.max() < q


def test_expand_uniformity(oracle_mod):
    """Residues mod q look uniform (mean ~ q/2, all below q), and distinct nonces differ."""
    ctx = oracle_mod.Ctx(12, 2, 1)
    seed = bytes(32)
    a = ctx.chacha_expand(seed, 0, 0, 0).astype(np.float64)
    q = ctx.mod[0]
    assert abs(a.mean() / q - 0.5) < 0.02 and a.max() < q
    b = ctx.chacha_expand(seed, 0, 0, 1)
    c = ctx.chacha_expand(seed, 1, 0, 0)
    d = ctx.chacha_expand(seed, 0, 1, 0)
    assert not np.array_equal(a, b) and not np.array_equal(a, c) and not np.array_equal(a, d)
