// chacha.cuh -- the ChaCha12 block function and the key's regenerated a half.
#pragma once
#include "modarith.cuh"

// ---------------------------------------------------------------- ChaCha12
// Block function (Bernstein 2008) with the RFC 8439 sec. 2.3 state: "expand 32-byte k",
// the key as 8 little-endian words, a 32-bit block counter, three nonce words; 12 rounds
// (6 column/diagonal double rounds) then the feed-forward addition.
struct ChachaKey {
    u32 k[8];
};

__device__ __forceinline__ u32 rotl(u32 v, int c) { return __funnelshift_l(v, v, c); }

#define CKKS_QR(a, b, c, d)                 \
    a += b; d ^= a; d = rotl(d, 16);        \
    c += d; b ^= c; b = rotl(b, 12);        \
    a += b; d ^= a; d = rotl(d, 8);         \
    c += d; b ^= c; b = rotl(b, 7);

__device__ __forceinline__ void chacha12_block(const ChachaKey &key, u32 counter, u32 n0, u32 n1,
                                               u32 n2, u32 (&o)[16]) {
    const u32 c0 = 0x61707865u, c1 = 0x3320646eu, c2 = 0x79622d32u, c3 = 0x6b206574u;
    u32 x0 = c0, x1 = c1, x2 = c2, x3 = c3;
    u32 x4 = key.k[0], x5 = key.k[1], x6 = key.k[2], x7 = key.k[3];
    u32 x8 = key.k[4], x9 = key.k[5], x10 = key.k[6], x11 = key.k[7];
    u32 x12 = counter, x13 = n0, x14 = n1, x15 = n2;
#pragma unroll
    for (int r = 0; r < 6; r++) {
        CKKS_QR(x0, x4, x8, x12) CKKS_QR(x1, x5, x9, x13)
        CKKS_QR(x2, x6, x10, x14) CKKS_QR(x3, x7, x11, x15)
        CKKS_QR(x0, x5, x10, x15) CKKS_QR(x1, x6, x11, x12)
        CKKS_QR(x2, x7, x8, x13) CKKS_QR(x3, x4, x9, x14)
    }
    o[0] = x0 + c0; o[1] = x1 + c1; o[2] = x2 + c2; o[3] = x3 + c3;
    o[4] = x4 + key.k[0]; o[5] = x5 + key.k[1]; o[6] = x6 + key.k[2]; o[7] = x7 + key.k[3];
    o[8] = x8 + key.k[4]; o[9] = x9 + key.k[5]; o[10] = x10 + key.k[6]; o[11] = x11 + key.k[7];
    o[12] = x12 + counter; o[13] = x13 + n0; o[14] = x14 + n1; o[15] = x15 + n2;
}

// a[n] for the 8 coefficients of block b: 64-bit LE word m = (o[2m] | o[2m+1] << 32) mod q,
// lazily in [0, 4q) (canonical when CANON).
template <bool CANON>
__device__ __forceinline__ void chacha_coeffs(const ChachaKey &key, u32 key_id, u32 digit, u32 limb,
                                              u32 block, const PrimeInfo &pi, u32 (&a)[8]) {
    u32 o[16];
    chacha12_block(key, block, key_id, digit, limb, o);
#pragma unroll
    for (int m = 0; m < 8; m++) {
        u32 v = shoup_mul(o[2 * m + 1], pi.r64, pi.r64p, pi.q) + shoup_mul(o[2 * m], 1u, pi.onep, pi.q);
        if (CANON) v = csub(csub(v, 2 * pi.q), pi.q);
        a[m] = v;
    }
}
