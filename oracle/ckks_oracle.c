/*
 * ckks_oracle.c -- plain, slow CPU oracle for RNS-CKKS hybrid key switching.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg may load this library.  It shares no code, header, table or constant generator with the
 * CUDA library; both are written separately from the same specification.
 *
 * What it computes (the method the Perseus write-up builds on):
 *   "Perseus: A Full-Stack System for Homomorphic Model Inference" (paperdot listing of
 *   arXiv:2611.04488, abstract) and the ai4snews write-up of it (Interpretation, 2nd
 *   paragraph): the uniformly random half of every key-switching key is regenerated with a
 *   counter-mode ChaCha12 expander inside the kernels that use the key, over a 32-bit RNS
 *   CKKS chain.  The pages do not define the arithmetic below; it follows the standard
 *   constructions, restated here from their definitions:
 *     - full-RNS CKKS and fast base conversion (Cheon, Han, Kim, Kim, Song, SAC 2018);
 *     - hybrid key switching with dnum gadget digits (Han, Ki, CT-RSA 2020);
 *     - the ChaCha block function with the state layout of RFC 8439 sec. 2.3.
 *   Where these leave a choice open, the reading taken is stated at the function.
 *
 * Style: every modular product is (a * b) % q on uint64_t with a, b < 2^30; nothing is lazy,
 * nothing is fused.  Loops over independent limbs carry an OpenMP pragma that does not
 * change the arithmetic.
 *
 * Data layout: RNS polynomials are uint32_t [limb][N], canonical residues in [0, q).
 * Evaluation-domain storage index k holds the value at psi^(2*brv(k)+1) (bit-reversed order).
 * Global limb index t: 0..n_q-1 are the ciphertext primes q_t, n_q..n_q+n_p-1 the special
 * primes p_{t-n_q}.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef uint64_t u64;
typedef uint32_t u32;
typedef int64_t i64;

/* ------------------------------------------------------------------ scalar arithmetic */

static u64 mulmod(u64 a, u64 b, u64 m) { return (a * b) % m; }

static u64 powmod(u64 b, u64 e, u64 m) {
    u64 r = 1 % m;
    b %= m;
    while (e) {
        if (e & 1) r = mulmod(r, b, m);
        b = mulmod(b, b, m);
        e >>= 1;
    }
    return r;
}

/* inverse modulo a prime m, by Fermat's little theorem */
static u64 invmod(u64 a, u64 m) { return powmod(a, m - 2, m); }

/* signed integer reduced into [0, m) */
static u64 smod(i64 v, u64 m) {
    i64 r = v % (i64)m;
    return (u64)(r < 0 ? r + (i64)m : r);
}

static u32 brv(u32 x, int bits) {
    u32 r = 0;
    for (int i = 0; i < bits; i++) r |= ((x >> i) & 1u) << (bits - 1 - i);
    return r;
}

/* ------------------------------------------------------------------ primes and roots */

/* Primality by trial division (x < 2^31). */
int or_is_prime(u64 x) {
    if (x < 2) return 0;
    if (x % 2 == 0) return x == 2;
    for (u64 d = 3; d * d <= x; d += 2)
        if (x % d == 0) return 0;
    return 1;
}

/* Prime chain rule: scan x = 1 (mod 2N) downward from the largest such x below 2^30 and keep
 * the primes, in the order found.  The caller takes the first n_p as the special primes
 * p_0 > p_1 > ... and the next n_q as the ciphertext primes q_0 > q_1 > ...
 * ("32-bit RNS CKKS chain": every prime below 2^30 so that 4q < 2^32.)  Returns count found. */
int or_gen_primes(int log_n, int count, u32 *out) {
    u64 two_n = 2ull << log_n;
    u64 x = (1ull << 30) - two_n + 1;
    int found = 0;
    while (found < count && x > two_n) {
        if (or_is_prime(x)) out[found++] = (u32)x;
        x -= two_n;
    }
    return found;
}

/* psi_q = h^((q-1)/2N) mod q for the smallest integer h >= 2 with psi_q^N = -1 (mod q);
 * psi_q is then a primitive 2N-th root of unity. */
u32 or_find_psi(u32 q, int log_n) {
    u64 n = 1ull << log_n;
    for (u64 h = 2; h < q; h++) {
        u64 psi = powmod(h, (q - 1) / (2 * n), q);
        if (powmod(psi, n, q) == q - 1) return (u32)psi;
    }
    return 0;
}

/* ------------------------------------------------------------------ context */

typedef struct {
    int log_n, n, n_q, n_p;
    u32 *mod;          /* [n_q + n_p] */
    u32 *psi;          /* [n_q + n_p] */
    u32 *psi_pow;      /* [n_q + n_p][N]: psi^i */
    u32 *psi_inv_pow;  /* [n_q + n_p][N]: psi^-i */
} or_ctx;

or_ctx *or_ctx_create(int log_n, int n_q, int n_p, const u32 *q, const u32 *p) {
    or_ctx *c = (or_ctx *)calloc(1, sizeof(or_ctx));
    int nt = n_q + n_p, n = 1 << log_n;
    c->log_n = log_n; c->n = n; c->n_q = n_q; c->n_p = n_p;
    c->mod = (u32 *)malloc(sizeof(u32) * nt);
    c->psi = (u32 *)malloc(sizeof(u32) * nt);
    c->psi_pow = (u32 *)malloc(sizeof(u32) * (size_t)nt * n);
    c->psi_inv_pow = (u32 *)malloc(sizeof(u32) * (size_t)nt * n);
    for (int t = 0; t < n_q; t++) c->mod[t] = q[t];
    for (int t = 0; t < n_p; t++) c->mod[n_q + t] = p[t];
#pragma omp parallel for
    for (int t = 0; t < nt; t++) {
        u64 m = c->mod[t];
        u64 psi = or_find_psi((u32)m, log_n);
        u64 psi_inv = invmod(psi, m);
        c->psi[t] = (u32)psi;
        /* powers psi^i and psi^-i for i < N */
        u64 pw = 1, pwi = 1;
        for (int i = 0; i < n; i++) {
            c->psi_pow[(size_t)t * n + i] = (u32)pw;
            c->psi_inv_pow[(size_t)t * n + i] = (u32)pwi;
            pw = mulmod(pw, psi, m);
            pwi = mulmod(pwi, psi_inv, m);
        }
    }
    return c;
}

void or_ctx_destroy(or_ctx *c) {
    if (!c) return;
    free(c->mod); free(c->psi); free(c->psi_pow); free(c->psi_inv_pow); free(c);
}

u32 or_ctx_psi(const or_ctx *c, int t) { return c->psi[t]; }

/* ------------------------------------------------------------------ NTT
 * Negacyclic NTT, defined as  A[k] = sum_{n<N} a[n] * psi^((2*brv(k)+1)*n)  mod q.
 * Factored as the definition reads: with b[n] = a[n] psi^n and omega = psi^2 (a primitive N-th
 * root of unity), A[k] = B[brv(k)] where B[j] = sum_n b[n] omega^(n j) is the cyclic DFT of b.
 * B is computed by the textbook iterative radix-2 decimation in time (inputs permuted to
 * bit-reversed order, then stages of length 2, 4, ..., N with twiddle powers of
 * omega^(N/len)), and read back at the bit-reversed index.  The inverse reads B[j] = A[brv(j)],
 * runs the same transform with omega^-1, multiplies by N^-1 and untwists by psi^-n.
 */
static void cyclic_dft(u32 *x, int n, int log_n, u64 omega, u64 q) {
    for (int i = 0; i < n; i++) {                     /* bit-reversal permutation */
        int r = (int)brv((u32)i, log_n);
        if (r > i) { u32 tmp = x[i]; x[i] = x[r]; x[r] = tmp; }
    }
    for (int len = 2; len <= n; len *= 2) {
        u64 w_len = 1;                                /* omega^(N/len) */
        for (int e = 0; e < n / len; e++) w_len = mulmod(w_len, omega, q);
        for (int start = 0; start < n; start += len) {
            u64 w = 1;
            for (int j = 0; j < len / 2; j++) {
                u64 u = x[start + j], v = mulmod(x[start + j + len / 2], w, q);
                x[start + j] = (u32)((u + v) % q);
                x[start + j + len / 2] = (u32)((u + q - v) % q);
                w = mulmod(w, w_len, q);
            }
        }
    }
}

void or_ntt_fwd_limb(const or_ctx *c, int t, u32 *a) {
    int n = c->n, log_n = c->log_n;
    u64 q = c->mod[t];
    const u32 *pw = c->psi_pow + (size_t)t * n;
    u32 *b = (u32 *)malloc(sizeof(u32) * (size_t)n);
    for (int i = 0; i < n; i++) b[i] = (u32)mulmod(a[i], pw[i], q);
    cyclic_dft(b, n, log_n, mulmod(c->psi[t], c->psi[t], q), q);
    for (int k = 0; k < n; k++) a[k] = b[brv((u32)k, log_n)];
    free(b);
}

void or_ntt_inv_limb(const or_ctx *c, int t, u32 *a) {
    int n = c->n, log_n = c->log_n;
    u64 q = c->mod[t];
    const u32 *pwi = c->psi_inv_pow + (size_t)t * n;
    u32 *b = (u32 *)malloc(sizeof(u32) * (size_t)n);
    for (int j = 0; j < n; j++) b[j] = a[brv((u32)j, log_n)];
    u64 psi_inv = pwi[1 % n];
    cyclic_dft(b, n, log_n, mulmod(psi_inv, psi_inv, q), q);
    u64 n_inv = invmod((u64)n % q, q);
    for (int i = 0; i < n; i++) a[i] = (u32)mulmod(mulmod(b[i], n_inv, q), pwi[i], q);
    free(b);
}

/* batch over limbs first_limb .. first_limb+n_limbs-1 of a [limb][N] buffer whose row 0 is
 * global limb first_limb */
void or_ntt_fwd(const or_ctx *c, u32 *poly, int first_limb, int n_limbs) {
#pragma omp parallel for
    for (int l = 0; l < n_limbs; l++) or_ntt_fwd_limb(c, first_limb + l, poly + (size_t)l * c->n);
}

void or_ntt_inv(const or_ctx *c, u32 *poly, int first_limb, int n_limbs) {
#pragma omp parallel for
    for (int l = 0; l < n_limbs; l++) or_ntt_inv_limb(c, first_limb + l, poly + (size_t)l * c->n);
}

/* ------------------------------------------------------------------ automorphism
 * kappa_g : a(X) -> a(X^g), g odd.  In coefficients, a[n] moves to n*g mod 2N, negated when
 * that index is >= N.  In evaluation storage, out[k] = in[k'] with
 * 2*brv(k')+1 = (2*brv(k)+1)*g (mod 2N), since kappa_g(a)(psi^e) = a(psi^(e*g)).
 */
void or_automorph_coef(const or_ctx *c, int t, const u32 *in, u32 *out, u32 g) {
    int n = c->n;
    u64 q = c->mod[t], two_n = 2ull * n;
    for (int i = 0; i < n; i++) {
        u64 e = ((u64)i * g) % two_n;
        if (e < (u64)n) out[e] = in[i];
        else out[e - n] = (u32)((q - in[i]) % q);
    }
}

void or_automorph_eval(const or_ctx *c, const u32 *in, u32 *out, int n_limbs, u32 g) {
    int n = c->n, log_n = c->log_n;
    u64 two_n = 2ull * n;
    for (int k = 0; k < n; k++) {
        u64 e = ((2ull * brv((u32)k, log_n) + 1) * g) % two_n;
        u32 kp = brv((u32)((e - 1) / 2), log_n);
        for (int l = 0; l < n_limbs; l++) out[(size_t)l * n + k] = in[(size_t)l * n + kp];
    }
}

/* Galois element of a rotation by r slots: 5^r mod 2N (r < 0 uses 5^(N/2 + r)). */
u32 or_galois_elt(int log_n, int r) {
    u64 n = 1ull << log_n, two_n = 2 * n, half = n / 2;
    i64 e = r % (i64)half;
    if (e < 0) e += (i64)half;
    u64 g = 1;
    for (i64 i = 0; i < e; i++) g = (g * 5) % two_n;
    return (u32)g;
}

/* ------------------------------------------------------------------ ChaCha
 * ChaCha block function (Bernstein 2008) with the RFC 8439 sec. 2.3 state: words 0-3 the
 * constant "expand 32-byte k", words 4-11 the 256-bit key as little-endian words, word 12
 * the block counter, words 13-15 the nonce.  `rounds` is 20 for ChaCha20 and 12 for
 * ChaCha12 (rounds/2 double rounds: a column round then a diagonal round); the final state
 * is the permuted state plus the input state, word by word.
 */
static u32 rotl32(u32 v, int c) { return (v << c) | (v >> (32 - c)); }

static void quarter(u32 *x, int a, int b, int c, int d) {
    x[a] += x[b]; x[d] ^= x[a]; x[d] = rotl32(x[d], 16);
    x[c] += x[d]; x[b] ^= x[c]; x[b] = rotl32(x[b], 12);
    x[a] += x[b]; x[d] ^= x[a]; x[d] = rotl32(x[d], 8);
    x[c] += x[d]; x[b] ^= x[c]; x[b] = rotl32(x[b], 7);
}

void or_chacha_block(const u32 key[8], u32 counter, const u32 nonce[3], int rounds, u32 out[16]) {
    u32 s[16], x[16];
    s[0] = 0x61707865u; s[1] = 0x3320646eu; s[2] = 0x79622d32u; s[3] = 0x6b206574u;
    for (int i = 0; i < 8; i++) s[4 + i] = key[i];
    s[12] = counter;
    s[13] = nonce[0]; s[14] = nonce[1]; s[15] = nonce[2];
    memcpy(x, s, sizeof(s));
    for (int r = 0; r < rounds; r += 2) {
        quarter(x, 0, 4, 8, 12); quarter(x, 1, 5, 9, 13);
        quarter(x, 2, 6, 10, 14); quarter(x, 3, 7, 11, 15);
        quarter(x, 0, 5, 10, 15); quarter(x, 1, 6, 11, 12);
        quarter(x, 2, 7, 8, 13); quarter(x, 3, 4, 9, 14);
    }
    for (int i = 0; i < 16; i++) out[i] = x[i] + s[i];
}

static void seed_words(const uint8_t seed[32], u32 key[8]) {
    for (int i = 0; i < 8; i++)
        key[i] = (u32)seed[4 * i] | ((u32)seed[4 * i + 1] << 8) | ((u32)seed[4 * i + 2] << 16) |
                 ((u32)seed[4 * i + 3] << 24);
}

/* The key's uniform half for gadget digit `digit` at global limb t, directly in evaluation
 * storage order.  Reading of "counter-mode ChaCha12 expander" (ai4snews write-up of Perseus,
 * Interpretation): ChaCha12 with key = seed, counter = block index b, nonce = (key_id, digit,
 * t); coefficient n takes the 64-bit little-endian word m = n mod 8 of block b = n / 8, i.e.
 * (w[2m] | w[2m+1] << 32), reduced mod the limb's prime by plain remainder. */
void or_chacha_expand(const or_ctx *c, const uint8_t seed[32], u32 key_id, u32 digit, int t,
                      u32 *out) {
    u32 key[8], nonce[3] = {key_id, digit, (u32)t}, blk[16];
    u64 q = c->mod[t];
    seed_words(seed, key);
    for (int b = 0; b < c->n / 8; b++) {
        or_chacha_block(key, (u32)b, nonce, 12, blk);
        for (int m = 0; m < 8; m++) {
            u64 w = (u64)blk[2 * m] | ((u64)blk[2 * m + 1] << 32);
            out[8 * b + m] = (u32)(w % q);
        }
    }
}

/* ------------------------------------------------------------------ gadget digits
 * Digit j holds the ciphertext primes j*alpha .. min((j+1)*alpha, L+1)-1 of the full chain.
 * At level l the active digits are those with j*alpha <= l; the last may be partial.
 */
static int n_digits(int n_active, int alpha) { return (n_active + alpha - 1) / alpha; }
static int digit_lo(int j, int alpha) { return j * alpha; }
static int digit_hi(int j, int alpha, int n_active) {
    int h = (j + 1) * alpha;
    return h < n_active ? h : n_active;
}

/* global limb index of extended-basis position u at level l (q_0..q_l, then p_0..p_{k-1}) */
static int ext_limb(const or_ctx *c, int level, int u) {
    return u <= level ? u : c->n_q + (u - level - 1);
}

/* ------------------------------------------------------------------ fast base conversion
 * FastBConv from the basis {r_i} (product D) to a modulus m, with centred representatives:
 *   y_i = [x_i * (D/r_i)^-1]_{r_i} taken in (-r_i/2, r_i/2], i.e. y_i - r_i when
 *   y_i > (r_i-1)/2,   out = (sum_i y_i * [D/r_i]_m) mod m.
 * The result is X + u*D for the centred CRT lift X of x and an integer |u| <= len(r)/2.
 * (Reading: the centred lift keeps u, and so the ModUp output, mean-free; with unsigned
 * representatives u ~ len(r)/2 on average and the key-switching error is multiplied by a
 * large constant polynomial, far outside the 2^-10 decoding budget at N=2^16.)
 * x: n_in limbs [i][N] in the coefficient domain.  Writes [N] residues mod m.
 */
static void bconv_one(const u32 *x, const u32 *r, int n_in, u32 m, int n, u32 *out) {
    u64 *dhat_inv = (u64 *)malloc(sizeof(u64) * n_in);   /* [(D/r_i)^-1]_{r_i} */
    u64 *dhat_m = (u64 *)malloc(sizeof(u64) * n_in);     /* [D/r_i]_m */
    for (int i = 0; i < n_in; i++) {
        u64 prod_ri = 1, prod_m = 1;
        for (int l = 0; l < n_in; l++) {
            if (l == i) continue;
            prod_ri = mulmod(prod_ri, r[l] % r[i], r[i]);
            prod_m = mulmod(prod_m, r[l] % m, m);
        }
        dhat_inv[i] = invmod(prod_ri, r[i]);
        dhat_m[i] = prod_m;
    }
    for (int k = 0; k < n; k++) {
        u64 acc = 0;
        for (int i = 0; i < n_in; i++) {
            u64 y = mulmod(x[(size_t)i * n + k], dhat_inv[i], r[i]);
            if (y > (r[i] - 1) / 2) {          /* negative representative y - r_i */
                u64 neg = mulmod(r[i] - y, dhat_m[i], m);
                acc = (acc + m - neg) % m;
            } else {
                acc = (acc + mulmod(y, dhat_m[i], m)) % m;
            }
        }
        out[k] = (u32)acc;
    }
    free(dhat_inv); free(dhat_m);
}

/* ------------------------------------------------------------------ ModUp
 * Hybrid key switching, ModUp (Han-Ki): for each active digit j of c (level l, eval domain),
 * lift [c]_{D_j} to the extended basis Q_l * P.  Digit limbs keep their evaluation values;
 * every other limb t gets NTT_t(FastBConv(iNTT(c restricted to digit j)) mod t).
 * Output dt: [beta][ext][N], ext = l+1+k, extended-basis order q_0..q_l, p_0..p_{k-1}.
 */
void or_modup(const or_ctx *c, const u32 *cpoly, int level, int alpha, u32 *dt) {
    int n = c->n, na = level + 1, ext = na + c->n_p, beta = n_digits(na, alpha);
    for (int j = 0; j < beta; j++) {
        int lo = digit_lo(j, alpha), hi = digit_hi(j, alpha, na), a_j = hi - lo;
        u32 *x = (u32 *)malloc(sizeof(u32) * (size_t)a_j * n);
        u32 *r = (u32 *)malloc(sizeof(u32) * a_j);
        memcpy(x, cpoly + (size_t)lo * n, sizeof(u32) * (size_t)a_j * n);
        for (int i = 0; i < a_j; i++) r[i] = c->mod[lo + i];
        or_ntt_inv(c, x, lo, a_j);                 /* digit limbs to coefficients */
        u32 *dj = dt + (size_t)j * ext * n;
#pragma omp parallel for
        for (int u = 0; u < ext; u++) {
            int t = ext_limb(c, level, u);
            if (u >= lo && u < hi) {
                memcpy(dj + (size_t)u * n, cpoly + (size_t)u * n, sizeof(u32) * n);
            } else {
                bconv_one(x, r, a_j, c->mod[t], n, dj + (size_t)u * n);
                or_ntt_fwd_limb(c, t, dj + (size_t)u * n);
            }
        }
        free(x); free(r);
    }
}

/* ------------------------------------------------------------------ key inner product
 * acc0[u] = sum_j dt_j[u] * b_j[t],  acc1[u] = sum_j dt_j[u] * a_j[t]  (mod the limb's
 * prime), over the extended basis at level l, t = global limb of position u.  b is the
 * stored half, [D][n_q+n_p][N] over the full chain; a_j[t] is regenerated by
 * or_chacha_expand(seed, key_id, j, t) ("the two kernels that use the key", ai4snews
 * write-up of Perseus, Interpretation).  If a_stored is non-NULL it is read instead
 * (same layout as b).
 */
void or_inner_product(const or_ctx *c, const u32 *dt, int level, int alpha, const u32 *b,
                      const u32 *a_stored, const uint8_t seed[32], u32 key_id, u32 *acc0,
                      u32 *acc1) {
    int n = c->n, na = level + 1, ext = na + c->n_p, beta = n_digits(na, alpha);
    int nt = c->n_q + c->n_p;
#pragma omp parallel for
    for (int u = 0; u < ext; u++) {
        int t = ext_limb(c, level, u);
        u64 q = c->mod[t];
        u32 *a = (u32 *)malloc(sizeof(u32) * n);
        u32 *r0 = acc0 + (size_t)u * n, *r1 = acc1 + (size_t)u * n;
        for (int k = 0; k < n; k++) r0[k] = r1[k] = 0;
        for (int j = 0; j < beta; j++) {
            const u32 *d = dt + ((size_t)j * ext + u) * n;
            const u32 *bj = b + ((size_t)j * nt + t) * n;
            if (a_stored) memcpy(a, a_stored + ((size_t)j * nt + t) * n, sizeof(u32) * n);
            else or_chacha_expand(c, seed, key_id, (u32)j, t, a);
            for (int k = 0; k < n; k++) {
                r0[k] = (u32)((r0[k] + mulmod(d[k], bj[k], q)) % q);
                r1[k] = (u32)((r1[k] + mulmod(d[k], a[k], q)) % q);
            }
        }
        free(a);
    }
}

/* ------------------------------------------------------------------ ModDown
 * ModDown (Cheon et al.): iNTT the k special limbs of acc, FastBConv P -> each q_i (centred
 * representatives, as in ModUp), NTT, then out_i = (acc_i - conv_i) * [P^-1]_{q_i}.  No +P/2
 * offset: with the centred lift the division error is already mean-free.
 * acc: [ext][N] eval domain; out: [l+1][N] eval domain.
 */
void or_moddown(const or_ctx *c, const u32 *acc, int level, u32 *out) {
    int n = c->n, na = level + 1, k = c->n_p;
    u32 *x = (u32 *)malloc(sizeof(u32) * (size_t)k * n);
    const u32 *pr = c->mod + c->n_q;
    memcpy(x, acc + (size_t)na * n, sizeof(u32) * (size_t)k * n);
    or_ntt_inv(c, x, c->n_q, k);
#pragma omp parallel for
    for (int i = 0; i < na; i++) {
        u64 q = c->mod[i];
        u64 p_mod = 1;
        for (int l = 0; l < k; l++) p_mod = mulmod(p_mod, pr[l] % q, q);
        u64 p_inv = invmod(p_mod, q);
        u32 *conv = out + (size_t)i * n;
        bconv_one(x, pr, k, (u32)q, n, conv);
        or_ntt_fwd_limb(c, i, conv);
        const u32 *ai = acc + (size_t)i * n;
        for (int m = 0; m < n; m++)
            conv[m] = (u32)mulmod((ai[m] + q - conv[m]) % q, p_inv, q);
    }
    free(x);
}

/* ------------------------------------------------------------------ key switching
 * KS(c) = (ModDown(acc0), ModDown(acc1)) with acc = inner product of ModUp(c) with the key.
 * out: [2][l+1][N].
 */
void or_keyswitch(const or_ctx *c, const u32 *cpoly, int level, int alpha, const u32 *b,
                  const u32 *a_stored, const uint8_t seed[32], u32 key_id, u32 *out) {
    int n = c->n, na = level + 1, ext = na + c->n_p, beta = n_digits(na, alpha);
    u32 *dt = (u32 *)malloc(sizeof(u32) * (size_t)beta * ext * n);
    u32 *acc0 = (u32 *)malloc(sizeof(u32) * (size_t)ext * n);
    u32 *acc1 = (u32 *)malloc(sizeof(u32) * (size_t)ext * n);
    or_modup(c, cpoly, level, alpha, dt);
    or_inner_product(c, dt, level, alpha, b, a_stored, seed, key_id, acc0, acc1);
    or_moddown(c, acc0, level, out);
    or_moddown(c, acc1, level, out + (size_t)na * n);
    free(dt); free(acc0); free(acc1);
}

static void add_into(const or_ctx *c, u32 *dst, const u32 *src, int n_limbs) {
    int n = c->n;
    for (int l = 0; l < n_limbs; l++) {
        u64 q = c->mod[l];
        for (int k = 0; k < n; k++) {
            size_t i = (size_t)l * n + k;
            dst[i] = (u32)(((u64)dst[i] + src[i]) % q);
        }
    }
}

/* Rotation by the Galois element g: kappa_g on both components first, then key switching of
 * kappa_g(c1) with the key for kappa_g(s), then kappa_g(c0) added to the first component.
 * ct, out: [2][l+1][N]. */
void or_rotate(const or_ctx *c, const u32 *ct, int level, int alpha, u32 g, const u32 *b,
               const u32 *a_stored, const uint8_t seed[32], u32 key_id, u32 *out) {
    int n = c->n, na = level + 1;
    u32 *rot = (u32 *)malloc(sizeof(u32) * 2 * (size_t)na * n);
    or_automorph_eval(c, ct, rot, na, g);
    or_automorph_eval(c, ct + (size_t)na * n, rot + (size_t)na * n, na, g);
    or_keyswitch(c, rot + (size_t)na * n, level, alpha, b, a_stored, seed, key_id, out);
    add_into(c, out, rot, na);
    free(rot);
}

/* Hoisted rotations: one ModUp of the unrotated c1, then for each r the extended digits
 * permuted by kappa_{g_r}, the inner product with key r, ModDown, and kappa_{g_r}(c0) added.
 * keys_b[r], keys_a[r] (may be NULL), seeds + 32*r, key_ids[r]; out: [n_rot][2][l+1][N]. */
void or_rotate_hoisted(const or_ctx *c, const u32 *ct, int level, int alpha, int n_rot,
                       const u32 *g, const u32 *const *keys_b, const u32 *const *keys_a,
                       const uint8_t *seeds, const u32 *key_ids, u32 *out) {
    int n = c->n, na = level + 1, ext = na + c->n_p, beta = n_digits(na, alpha);
    size_t dt_words = (size_t)beta * ext * n;
    u32 *dt = (u32 *)malloc(sizeof(u32) * dt_words);
    u32 *dtr = (u32 *)malloc(sizeof(u32) * dt_words);
    u32 *acc0 = (u32 *)malloc(sizeof(u32) * (size_t)ext * n);
    u32 *acc1 = (u32 *)malloc(sizeof(u32) * (size_t)ext * n);
    u32 *c0r = (u32 *)malloc(sizeof(u32) * (size_t)na * n);
    or_modup(c, ct + (size_t)na * n, level, alpha, dt);
    for (int r = 0; r < n_rot; r++) {
        u32 *o = out + (size_t)r * 2 * na * n;
        for (int j = 0; j < beta; j++)
            or_automorph_eval(c, dt + (size_t)j * ext * n, dtr + (size_t)j * ext * n, ext, g[r]);
        or_inner_product(c, dtr, level, alpha, keys_b[r], keys_a ? keys_a[r] : NULL,
                         seeds + 32 * r, key_ids[r], acc0, acc1);
        or_moddown(c, acc0, level, o);
        or_moddown(c, acc1, level, o + (size_t)na * n);
        or_automorph_eval(c, ct, c0r, na, g[r]);
        add_into(c, o, c0r, na);
    }
    free(dt); free(dtr); free(acc0); free(acc1); free(c0r);
}

/* Relinearisation: d = (d0, d1, d2) decrypting under (1, s, s^2); key switching of d2 with
 * the key for s^2, added to (d0, d1).  d: [3][l+1][N]; out: [2][l+1][N]. */
void or_relin(const or_ctx *c, const u32 *d, int level, int alpha, const u32 *b,
              const u32 *a_stored, const uint8_t seed[32], u32 key_id, u32 *out) {
    int n = c->n, na = level + 1;
    or_keyswitch(c, d + 2 * (size_t)na * n, level, alpha, b, a_stored, seed, key_id, out);
    add_into(c, out, d, na);
    add_into(c, out + (size_t)na * n, d + (size_t)na * n, na);
}

/* Tensor product of x = (x0, x1) and y = (y0, y1), pointwise in the evaluation domain:
 * d0 = x0*y0, d1 = x0*y1 + x1*y0, d2 = x1*y1.  x, y: [2][l+1][N]; d: [3][l+1][N]. */
void or_tensor(const or_ctx *c, const u32 *x, const u32 *y, int level, u32 *d) {
    int n = c->n, na = level + 1;
    size_t pl = (size_t)na * n;
    for (int l = 0; l < na; l++) {
        u64 q = c->mod[l];
        for (int k = 0; k < n; k++) {
            size_t i = (size_t)l * n + k;
            u64 x0 = x[i], x1 = x[pl + i], y0 = y[i], y1 = y[pl + i];
            d[i] = (u32)mulmod(x0, y0, q);
            d[pl + i] = (u32)((mulmod(x0, y1, q) + mulmod(x1, y0, q)) % q);
            d[2 * pl + i] = (u32)mulmod(x1, y1, q);
        }
    }
}

/* Rescaling by the last active prime (full-RNS CKKS, Cheon, Han, Kim, Kim, Song, SAC 2018,
 * the RNS rescale: the pages name no rescale of their own).  For each component, with C the
 * integer polynomial whose residues are the component's limbs 0..l:
 *   out = (C - [C]_{q_l}) / q_l   reduced modulo q_0 .. q_{l-1},
 * where [C]_{q_l} is the centred residue of C modulo q_l, in (-q_l/2, q_l/2] (the same
 * centred lift the base conversion uses).  The division is exact, so per limb
 *   out_i = (c_i - [C]_{q_l} mod q_i) * q_l^-1  (mod q_i).
 * [C]_{q_l} is a coefficient-domain quantity: limb l is brought to coefficients by the inverse
 * NTT, lifted, reduced modulo q_i and brought back by the forward NTT of prime q_i.
 * ct: [n_comp][l+1][N] (evaluation domain); out: [n_comp][l][N].  level >= 1. */
void or_rescale(const or_ctx *c, const u32 *ct, int n_comp, int level, u32 *out) {
    int n = c->n, na = level + 1;
    u64 ql = c->mod[level];
    u32 *last = (u32 *)malloc(sizeof(u32) * (size_t)n);
    for (int comp = 0; comp < n_comp; comp++) {
        const u32 *cc = ct + (size_t)comp * na * n;
        memcpy(last, cc + (size_t)level * n, sizeof(u32) * (size_t)n);
        or_ntt_inv_limb(c, level, last);
#pragma omp parallel for
        for (int i = 0; i < level; i++) {
            u64 q = c->mod[i];
            u64 ql_inv = invmod(ql % q, q);
            u32 *o = out + ((size_t)comp * level + i) * n;
            for (int m = 0; m < n; m++) {
                i64 v = last[m] > (ql - 1) / 2 ? (i64)last[m] - (i64)ql : (i64)last[m];
                o[m] = (u32)smod(v, q);
            }
            or_ntt_fwd_limb(c, i, o);
            const u32 *ci = cc + (size_t)i * n;
            for (int m = 0; m < n; m++) o[m] = (u32)mulmod((ci[m] + q - o[m]) % q, ql_inv, q);
        }
    }
    free(last);
}

/* ------------------------------------------------------------------ keys, encryption
 * Signed coefficient vector -> evaluation-domain limb t. */
void or_signed_to_eval(const or_ctx *c, const i64 *v, int t, u32 *out) {
    u64 q = c->mod[t];
    for (int k = 0; k < c->n; k++) out[k] = (u32)smod(v[k], q);
    or_ntt_fwd_limb(c, t, out);
}

/* Key-switching key from s' to s (Han-Ki gadget in RNS form): for digit j of the full chain
 * and every limb t of Q*P,
 *   a_j[t] = ChaCha12 expansion (seed, key_id, j, t),
 *   b_j[t] = -a_j[t]*s[t] + e_j[t] + [t in digit j] * [P]_{q_t} * s'[t]    (mod t),
 * all in the evaluation domain; [P]_{q_t} * [t in digit j] is the RNS form of the gadget
 * P * (Q/D_j) * [(Q/D_j)^-1]_{D_j}.
 * s, e: signed coefficients (s [N], e [D][N]); s2_eval: s' in the evaluation domain
 * [n_q+n_p][N].  b: [D][n_q+n_p][N]; a_out (optional) gets the a half, same layout. */
void or_keygen(const or_ctx *c, int alpha, const i64 *s, const u32 *s2_eval, const i64 *e,
               const uint8_t seed[32], u32 key_id, u32 *b, u32 *a_out) {
    int n = c->n, nt = c->n_q + c->n_p, nd = n_digits(c->n_q, alpha);
#pragma omp parallel for
    for (int t = 0; t < nt; t++) {
        u64 q = c->mod[t];
        u64 p_mod = 1;
        for (int l = 0; l < c->n_p; l++) p_mod = mulmod(p_mod, c->mod[c->n_q + l] % q, q);
        u32 *s_ev = (u32 *)malloc(sizeof(u32) * n);
        u32 *e_ev = (u32 *)malloc(sizeof(u32) * n);
        u32 *a = (u32 *)malloc(sizeof(u32) * n);
        or_signed_to_eval(c, s, t, s_ev);
        for (int j = 0; j < nd; j++) {
            int in_digit = t < c->n_q && t >= digit_lo(j, alpha) && t < digit_hi(j, alpha, c->n_q);
            or_signed_to_eval(c, e + (size_t)j * n, t, e_ev);
            or_chacha_expand(c, seed, key_id, (u32)j, t, a);
            u32 *bj = b + ((size_t)j * nt + t) * n;
            for (int k = 0; k < n; k++) {
                u64 v = (q - mulmod(a[k], s_ev[k], q)) % q;
                v = (v + e_ev[k]) % q;
                if (in_digit) v = (v + mulmod(p_mod, s2_eval[(size_t)t * n + k], q)) % q;
                bj[k] = (u32)v;
            }
            if (a_out) memcpy(a_out + ((size_t)j * nt + t) * n, a, sizeof(u32) * n);
        }
        free(s_ev); free(e_ev); free(a);
    }
}

/* Secret-key encryption at level l: ct = (-a*s + m + e, a) in the evaluation domain, with a
 * uniform (given, evaluation domain, [l+1][N]) and m, e signed coefficients [N]. */
void or_encrypt(const or_ctx *c, const i64 *s, const i64 *m, const i64 *e, const u32 *a,
                int level, u32 *ct) {
    int n = c->n, na = level + 1;
    i64 *me = (i64 *)malloc(sizeof(i64) * n);
    for (int k = 0; k < n; k++) me[k] = m[k] + e[k];
#pragma omp parallel for
    for (int t = 0; t < na; t++) {
        u64 q = c->mod[t];
        u32 *s_ev = (u32 *)malloc(sizeof(u32) * n);
        u32 *me_ev = (u32 *)malloc(sizeof(u32) * n);
        or_signed_to_eval(c, s, t, s_ev);
        or_signed_to_eval(c, me, t, me_ev);
        for (int k = 0; k < n; k++) {
            size_t i = (size_t)t * n + k;
            u64 v = (q - mulmod(a[i], s_ev[k], q)) % q;
            ct[i] = (u32)((v + me_ev[k]) % q);
            ct[(size_t)na * n + i] = a[i];
        }
        free(s_ev); free(me_ev);
    }
    free(me);
}

/* Decryption to the coefficient domain: m = c0 + c1*s (+ c2*s^2 when n_comp == 3), then
 * iNTT; residues [l+1][N].  s_eval: [n_q+n_p][N] evaluation-domain secret. */
void or_decrypt(const or_ctx *c, const u32 *ct, int n_comp, int level, const u32 *s_eval,
                u32 *m_out) {
    int n = c->n, na = level + 1;
    for (int t = 0; t < na; t++) {
        u64 q = c->mod[t];
        for (int k = 0; k < n; k++) {
            size_t i = (size_t)t * n + k;
            u64 sv = s_eval[(size_t)t * n + k];
            u64 v = (ct[i] + mulmod(ct[(size_t)na * n + i], sv, q)) % q;
            if (n_comp == 3) v = (v + mulmod(ct[2 * (size_t)na * n + i], mulmod(sv, sv, q), q)) % q;
            m_out[i] = (u32)v;
        }
    }
    or_ntt_inv(c, m_out, 0, na);
}
