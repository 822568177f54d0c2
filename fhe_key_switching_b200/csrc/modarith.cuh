// modarith.cuh -- 32-bit modular arithmetic for primes q < 2^30 (so 4q < 2^32).
//
// Shoup multiplication by a constant w < q with companion w' = floor(w * 2^32 / q):
//   a*w - umulhi(a, w')*q  lies in [0, 2q) for any a < 2^32.
// Lazy ranges follow Harvey ("Faster arithmetic for number-theoretic transforms", 2014):
// forward (Cooley-Tukey) butterflies keep values in [0, 4q), inverse (Gentleman-Sande)
// butterflies in [0, 2q).
#pragma once
#include <cstdint>

typedef uint32_t u32;
typedef uint64_t u64;

// a - m if a >= m, else a  (one subtract and one unsigned min)
__device__ __forceinline__ u32 csub(u32 a, u32 m) { return min(a, a - m); }

__device__ __forceinline__ u32 shoup_mul(u32 a, u32 w, u32 wp, u32 q) {
    u32 qh = __umulhi(a, wp);
    return a * w - qh * q;
}

// Forward butterfly: (x, y) -> (x + w y, x - w y), inputs and outputs in [0, 4q).
__device__ __forceinline__ void ct_bfly(u32 &x, u32 &y, u32 w, u32 wp, u32 q, u32 two_q) {
    u32 a = csub(x, two_q);
    u32 t = shoup_mul(y, w, wp, q);
    x = a + t;
    y = a - t + two_q;
}

// Inverse butterfly: (x, y) -> (x + y, (x - y) w), inputs and outputs in [0, 2q).
__device__ __forceinline__ void gs_bfly(u32 &x, u32 &y, u32 w, u32 wp, u32 q, u32 two_q) {
    u32 s = csub(x + y, two_q);
    u32 d = x - y + two_q;
    y = shoup_mul(d, w, wp, q);
    x = s;
}

// Reduce any 64-bit value: x = hi 2^32 + lo = hi [2^32]_q + lo (mod q).  r64 = [2^32]_q with
// its Shoup companion r64p; onep = floor(2^32 / q) is the companion of w = 1.
// Result in [0, 4q).
__device__ __forceinline__ u32 reduce64_lazy(u64 x, u32 q, u32 r64, u32 r64p, u32 onep) {
    u32 hi = (u32)(x >> 32), lo = (u32)x;
    return shoup_mul(hi, r64, r64p, q) + shoup_mul(lo, 1u, onep, q);
}

__device__ __forceinline__ u32 reduce64(u64 x, u32 q, u32 r64, u32 r64p, u32 onep) {
    u32 r = reduce64_lazy(x, q, r64, r64p, onep);
    return csub(csub(r, 2 * q), q);
}

// Per-prime constants used by the kernels (one 32-byte record per global limb).
struct PrimeInfo {
    u32 q;        // the prime
    u32 r64;      // 2^32 mod q
    u32 r64p;     // Shoup companion of r64
    u32 onep;     // floor(2^32 / q)
    u32 n_inv;    // N^-1 mod q
    u32 n_invp;   // Shoup companion
    u32 half;     // (q - 1) / 2, the centred-lift threshold
    u32 qinv;     // -q^-1 mod 2^32 (Montgomery)
};

// Montgomery product a*b*2^-32 mod q, in [0, 2q) whenever a*b < 4q^2 (e.g. a < q, b < 4q).
__device__ __forceinline__ u32 mont_mul(u32 a, u32 b, u32 q, u32 qinv) {
    const u32 lo = a * b;
    const u32 hi = __umulhi(a, b);
    const u32 m = lo * qinv;
    // (a*b + m*q) / 2^32: the low words cancel, with a carry exactly when lo != 0
    return hi + __umulhi(m, q) + (lo != 0u ? 1u : 0u);
}
