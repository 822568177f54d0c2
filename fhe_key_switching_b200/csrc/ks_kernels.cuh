// ks_kernels.cuh -- base conversion, ChaCha12-fused key inner product, ModDown combine,
// tensor product and automorphism kernels.
#pragma once
#include "chacha.cuh"
#include "ntt.cuh"

// ---------------------------------------------------------------- ChaCha12 expansion (debug export)
__global__ void k_chacha_expand(ChachaKey key, u32 key_id, u32 digit, u32 limb,
                                const PrimeInfo *pinfo, u32 *out, int n) {
    const int b = blockIdx.x * blockDim.x + threadIdx.x;
    if (b >= n / 8) return;
    if (!CKKS_SPAN(pinfo + limb, 1, CKKS_DBG_NTT_TABLES) || !CKKS_SPAN(out + 8 * b, 8, CKKS_DBG_CHACHA_OUT)) return;
    const PrimeInfo pi = pinfo[limb];
    u32 a[8];
    chacha_coeffs<true>(key, key_id, digit, limb, (u32)b, pi, a);
    uint4 *o = reinterpret_cast<uint4 *>(out + 8 * b);
    o[0] = make_uint4(a[0], a[1], a[2], a[3]);
    o[1] = make_uint4(a[4], a[5], a[6], a[7]);
}

// ---------------------------------------------------------------- fast base conversion
// For group g (a ModUp digit or a ModDown operand) with inputs y_i (coefficient domain,
// canonical, already multiplied by (D/r_i)^-1) and every target k of the group:
//   out_k = sum_i y_i [D/r_i]_t - v [D]_t  (mod t),  v = #{i : y_i > (r_i - 1)/2},
// i.e. the sum over the centred representatives y_i - r_i [y_i > (r_i-1)/2].
struct BconvArgs {
    const u32 *y;            // input rows
    u32 *out;                // output rows
    const PrimeInfo *pinfo;
    const u32 *bmat;         // per group config: [n_in][n_primes] = [D/r_i]_t
    const u32 *negd;         // per group config: [n_primes] = [-D]_t
    JobMap map;              // targets: per_group, split, bases, out rows, skip_alpha
    int n_primes;            // row length of bmat/negd tables (global limbs)
    int log_n;
    // inputs of group g: rows in_row0 + g * in_group_rows + i, primes in_prime0 + g*in_prime_step + i
    int in_row0, in_group_rows, in_prime0, in_prime_step;
    int n_in_full;           // inputs per group (the last group may have fewer: n_in_last)
    int n_in_last;
    int n_groups;
    int cfg_per_group;       // table config index = g * cfg_per_group + (n_in(g) - 1) (ModUp), or 0
    int cfg_stride;          // words per config in bmat = max_in * n_primes
    int g_base;              // logical group of blockIdx.y = 0 (a launch may cover a subset)
    int nchunk;              // target chunks per item: blockIdx.z = item * nchunk + chunk
    int tchunk;              // targets per chunk (a multiple of 4)
    size_t y_item, out_item; // item strides (words)
};

constexpr int BCONV_THREADS = 256;
constexpr int BCONV_MAX_IN = 64;
constexpr int BCONV_TCHUNK = 12;      // targets per block for small launches (see BconvArgs::tchunk)

// MAXIN: compile-time bound on the group's input count (inputs live in registers).
// Each thread converts 2 consecutive coefficients.
template <int MAXIN>
__global__ void __launch_bounds__(BCONV_THREADS)
k_bconv(BconvArgs a) {
    extern __shared__ u32 smb[];          // [n_in + 1][T] constants (row n_in: [-D]_t), then half[n_in]
    const int g = a.g_base + blockIdx.y;
    const int item = blockIdx.z / a.nchunk, chunk = blockIdx.z % a.nchunk;
    const u32 *yb = a.y + item * a.y_item;
    u32 *ob = a.out + item * a.out_item;
    const int n = 1 << a.log_n;
    const int n_in = (g == a.n_groups - 1) ? a.n_in_last : a.n_in_full;
    const int cfg = a.cfg_per_group ? g * a.cfg_per_group + (n_in - 1) : 0;
    const u32 *bm = a.bmat + (size_t)cfg * a.cfg_stride;
    const u32 *nd = a.negd + (size_t)cfg * a.n_primes;
    const int T = a.map.per_group;
    const int row0 = a.in_row0 + g * a.in_group_rows;
    const int p0 = a.in_prime0 + g * a.in_prime_step;
    if (!CKKS_SPAN(bm, (size_t)n_in * a.n_primes, CKKS_DBG_BCONV_TABLES) ||
        !CKKS_SPAN(nd, a.n_primes, CKKS_DBG_BCONV_TABLES) || !CKKS_SPAN(a.pinfo + p0, n_in, CKKS_DBG_BCONV_TABLES) ||
        !CKKS_SPAN(a.pinfo + a.map.lo_base, a.map.split, CKKS_DBG_BCONV_TABLES) ||
        (T > a.map.split && !CKKS_SPAN(a.pinfo + a.map.hi_base, T - a.map.split, CKKS_DBG_BCONV_TABLES)))
        return;                                               // (the same for the whole block)
    CKKS_POISON_DYNAMIC(smb);
    u32 *half = smb + (n_in + 1) * T;
    for (int idx = threadIdx.x; idx < (n_in + 1) * T; idx += blockDim.x) {
        const int i = idx / T, kk = idx - i * T;
        const int t = kk < a.map.split ? a.map.lo_base + kk : a.map.hi_base + (kk - a.map.split);
        smb[idx] = (i < n_in) ? bm[(size_t)i * a.n_primes + t] : nd[t];
    }
    for (int i = threadIdx.x; i < n_in; i += blockDim.x) half[i] = a.pinfo[p0 + i].half;
    __syncthreads();
    const int c2 = blockIdx.x * blockDim.x + threadIdx.x;   // coefficient pair
    if (2 * c2 >= n) return;
    u32 y0[MAXIN], y1[MAXIN];
    u32 v0 = 0, v1 = 0;
    const bool ok_in = CKKS_SPAN2(yb + (size_t)row0 * n + 2 * c2, yb + (size_t)(row0 + n_in - 1) * n + 2 * c2 + 1,
                                  CKKS_DBG_BCONV_IN);
#pragma unroll
    for (int i = 0; i < MAXIN; i++) {
        if (i < n_in) {
            const uint2 t = ok_in ? reinterpret_cast<const uint2 *>(yb + (size_t)(row0 + i) * n)[c2] : make_uint2(0u, 0u);
            const u32 h = half[i];
            y0[i] = t.x; y1[i] = t.y;
            v0 += t.x > h ? 1u : 0u;
            v1 += t.y > h ? 1u : 0u;
        }
    }
    const int lo = a.map.skip_alpha > 0 ? g * a.map.skip_alpha : 0;
    const int hi = a.map.skip_alpha > 0 ? min(lo + a.map.skip_alpha, a.map.split) : 0;
    const int k_end = min(T, (chunk + 1) * a.tchunk);
    const bool ok_out = chunk * a.tchunk >= k_end ||
                        CKKS_SPAN2(ob + ((size_t)g * a.map.out_group_rows + a.map.out_k_base + chunk * a.tchunk) * n + 2 * c2,
                                   ob + ((size_t)g * a.map.out_group_rows + a.map.out_k_base + k_end - 1) * n + 2 * c2 + 1,
                                   CKKS_DBG_BCONV_OUT);
    for (int kk = chunk * a.tchunk; kk < k_end; kk++) {
        if (kk >= lo && kk < hi) continue;
        const int t = kk < a.map.split ? a.map.lo_base + kk : a.map.hi_base + (kk - a.map.split);
        const PrimeInfo pi = a.pinfo[t];
        const u32 nd_t = smb[n_in * T + kk];
        u64 s0 = (u64)v0 * nd_t, s1 = (u64)v1 * nd_t;
#pragma unroll
        for (int i = 0; i < MAXIN; i++) {
            if (i < n_in) {
                const u32 bc = smb[i * T + kk];
                s0 += (u64)y0[i] * bc;
                s1 += (u64)y1[i] * bc;
                if ((i % 14) == 13) {          // keep the 64-bit sums below 2^64
                    s0 = reduce64_lazy(s0, pi.q, pi.r64, pi.r64p, pi.onep);
                    s1 = reduce64_lazy(s1, pi.q, pi.r64, pi.r64p, pi.onep);
                }
            }
        }
        const uint2 r = make_uint2(reduce64(s0, pi.q, pi.r64, pi.r64p, pi.onep),
                                   reduce64(s1, pi.q, pi.r64, pi.r64p, pi.onep));
        if (ok_out) reinterpret_cast<uint2 *>(ob + ((size_t)g * a.map.out_group_rows + a.map.out_k_base + kk) * n)[c2] = r;
    }
}

// Exact-count variant: NIN inputs known at compile time; each thread converts BCONV_CPT = 4
// consecutive coefficients for 4 targets at a time (16 independent 64-bit sums).  Staged in
// shared memory: the constants as [NIN + 1][T4] words with T4 = T rounded up to 4 (row NIN
// holds [-D]_t, multiplied by the count v of negative representatives), so one 128-bit load
// gives 4 targets' constants, then each target's (t, [2^32]_t, its Shoup companion,
// floor(2^32/t)) as one 128-bit record.
// Output is lazily reduced, in [0, 4t): every consumer is a forward NTT, whose butterflies take
// inputs in [0, 4t) and whose output is canonical.
constexpr int BCONV_CPT = 4;

__host__ __device__ constexpr size_t bconv_n_smem_words(int nin, int t4) { return (size_t)(nin + 5) * t4; }

template <int NIN>
__global__ void __launch_bounds__(BCONV_THREADS)
k_bconv_n(BconvArgs a) {
    constexpr int CPT = BCONV_CPT;
    extern __shared__ __align__(16) u32 smc[];
    const int g = a.g_base + blockIdx.y;
    const int item = blockIdx.z / a.nchunk, chunk = blockIdx.z % a.nchunk;
    const u32 *yb = a.y + item * a.y_item;
    u32 *ob = a.out + item * a.out_item;
    const int n = 1 << a.log_n;
    const int cfg = a.cfg_per_group ? g * a.cfg_per_group + (NIN - 1) : 0;
    const u32 *bm = a.bmat + (size_t)cfg * a.cfg_stride;
    const u32 *nd = a.negd + (size_t)cfg * a.n_primes;
    const int T = a.map.per_group;
    const int T4 = (T + 3) & ~3;
    const int row0 = a.in_row0 + g * a.in_group_rows;
    const int p0 = a.in_prime0 + g * a.in_prime_step;
    if (!CKKS_SPAN(bm, (size_t)NIN * a.n_primes, CKKS_DBG_BCONV_TABLES) ||
        !CKKS_SPAN(nd, a.n_primes, CKKS_DBG_BCONV_TABLES) || !CKKS_SPAN(a.pinfo + p0, NIN, CKKS_DBG_BCONV_TABLES) ||
        !CKKS_SPAN(a.pinfo + a.map.lo_base, a.map.split, CKKS_DBG_BCONV_TABLES) ||
        (T > a.map.split && !CKKS_SPAN(a.pinfo + a.map.hi_base, T - a.map.split, CKKS_DBG_BCONV_TABLES)))
        return;                                               // (the same for the whole block)
    CKKS_POISON_DYNAMIC(smc);
    for (int idx = threadIdx.x; idx < (NIN + 1) * T4; idx += blockDim.x) {
        const int i = idx / T4, kk = idx - i * T4;
        u32 val = 0;
        if (kk < T) {
            const int t = kk < a.map.split ? a.map.lo_base + kk : a.map.hi_base + (kk - a.map.split);
            val = (i < NIN) ? bm[(size_t)i * a.n_primes + t] : nd[t];
        }
        smc[idx] = val;
    }
    uint4 *sq = reinterpret_cast<uint4 *>(smc + (NIN + 1) * T4);
    for (int kk = threadIdx.x; kk < T4; kk += blockDim.x) {
        uint4 v = make_uint4(0, 0, 0, 0);
        if (kk < T) {
            const int t = kk < a.map.split ? a.map.lo_base + kk : a.map.hi_base + (kk - a.map.split);
            const PrimeInfo pi = a.pinfo[t];
            v = make_uint4(pi.q, pi.r64, pi.r64p, pi.onep);
        }
        sq[kk] = v;
    }
    __syncthreads();
    const int cv = blockIdx.x * blockDim.x + threadIdx.x;   // coefficients CPT cv .. CPT cv + 3
    if (CPT * cv >= n) return;
    u32 y[CPT][NIN + 1];
    u32 v[CPT] = {0, 0, 0, 0};
    const bool ok_in = CKKS_SPAN2(yb + (size_t)row0 * n + CPT * cv, yb + (size_t)(row0 + NIN - 1) * n + CPT * cv + CPT - 1,
                                  CKKS_DBG_BCONV_IN);
#pragma unroll
    for (int i = 0; i < NIN; i++) {
        const u32 h = a.pinfo[p0 + i].half;
        const uint4 w = ok_in ? reinterpret_cast<const uint4 *>(yb + (size_t)(row0 + i) * n)[cv] : make_uint4(0u, 0u, 0u, 0u);
        const u32 t[CPT] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int c = 0; c < CPT; c++) { y[c][i] = t[c]; v[c] += t[c] > h ? 1u : 0u; }
    }
#pragma unroll
    for (int c = 0; c < CPT; c++) y[c][NIN] = v[c];
    const int lo = a.map.skip_alpha > 0 ? g * a.map.skip_alpha : 0;
    const int hi = a.map.skip_alpha > 0 ? min(lo + a.map.skip_alpha, a.map.split) : 0;
    const int k_beg = chunk * a.tchunk;
    const int k_end = min(T, k_beg + a.tchunk);
    const bool ok_out = k_beg >= k_end ||
                        CKKS_SPAN2(ob + ((size_t)g * a.map.out_group_rows + a.map.out_k_base + k_beg) * n + CPT * cv,
                                   ob + ((size_t)g * a.map.out_group_rows + a.map.out_k_base + k_end - 1) * n + CPT * cv +
                                       CPT - 1,
                                   CKKS_DBG_BCONV_OUT);
    for (int k4 = k_beg; k4 < k_end; k4 += 4) {
        u64 s[CPT][4];
#pragma unroll
        for (int c = 0; c < CPT; c++)
#pragma unroll
            for (int m = 0; m < 4; m++) s[c][m] = 0;
#pragma unroll
        for (int i = 0; i <= NIN; i++) {
            const uint4 b4 = *reinterpret_cast<const uint4 *>(smc + i * T4 + k4);
            const u32 bb[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
            for (int m = 0; m < 4; m++)
#pragma unroll
                for (int c = 0; c < CPT; c++) s[c][m] += (u64)y[c][i] * bb[m];
        }
#pragma unroll
        for (int m = 0; m < 4; m++) {
            const int kk = k4 + m;
            if (kk >= k_end || (kk >= lo && kk < hi)) continue;
            const uint4 pq = sq[kk];
            u32 r[CPT];
#pragma unroll
            for (int c = 0; c < CPT; c++) r[c] = reduce64_lazy(s[c][m], pq.x, pq.y, pq.z, pq.w);
            u32 *dst = ob + ((size_t)g * a.map.out_group_rows + a.map.out_k_base + kk) * n;
            if (ok_out) reinterpret_cast<uint4 *>(dst)[cv] = make_uint4(r[0], r[1], r[2], r[3]);
        }
    }
}

// ---------------------------------------------------------------- key inner product
// acc0[u] = sum_j dt_j[u] b_j[t], acc1[u] = sum_j dt_j[u] a_j[t] over the active digits, with
// a_j[t] regenerated by ChaCha12 (or read from a stored a half).  For u inside digit j the
// extended digit equals the input polynomial itself (cdig).  hoist_g != 0: every dt row is
// read through kappa_{hoist_g} (hoisted rotation); cdig_g != 0: cdig is read through
// kappa_{cdig_g} (single rotation, whose ModUp input was kappa_g(c1)).
struct IpArgs {
    const u32 *dt;           // [beta][ext][N]
    const u32 *cdig;         // [l+1][N]: digit limbs (nullptr: read them from dt)
    const u32 *b;            // [D][n_primes][N]
    const u32 *a_stored;     // nullptr: regenerate
    u32 *acc;                // [2][ext][N]
    const PrimeInfo *pinfo;
    ChachaKey key;
    u32 key_id;
    int log_n, level, n_q, n_primes, alpha, beta, ext;
    u32 hoist_g, cdig_g;
};

constexpr int IP_THREADS = 128;

__global__ void __launch_bounds__(IP_THREADS)
k_inner_product(IpArgs a) {
    const int n = 1 << a.log_n;
    const int blk = blockIdx.x * blockDim.x + threadIdx.x;   // 8 coefficients each
    if (blk >= n / 8) return;
    const int u = blockIdx.y;
    const int na = a.level + 1;
    const int t = u < na ? u : a.n_q + (u - na);
    if (!CKKS_SPAN(a.pinfo + t, 1, CKKS_DBG_IP_TABLES)) return;
    const PrimeInfo pi = a.pinfo[t];
    u64 s0[8], s1[8];
#pragma unroll
    for (int m = 0; m < 8; m++) s0[m] = s1[m] = 0;
    for (int j = 0; j < a.beta; j++) {
        const bool in_digit = a.cdig && u < na && u >= j * a.alpha && u < min(j * a.alpha + a.alpha, na);
        const u32 *src = in_digit ? a.cdig + (size_t)u * n : a.dt + ((size_t)j * a.ext + u) * n;
        const u32 g = in_digit ? (a.hoist_g ? a.hoist_g : a.cdig_g) : a.hoist_g;
        u32 d[8];
        if (g) {
            const bool ok = CKKS_SPAN(src, n, CKKS_DBG_IP_IN);             // automorph_src < n
#pragma unroll
            for (int m = 0; m < 8; m++) d[m] = ok ? src[automorph_src((u32)(8 * blk + m), g, a.log_n)] : 0u;
        } else {
            const uint4 *s4 = reinterpret_cast<const uint4 *>(src + 8 * blk);
            const bool ok = CKKS_SPAN(s4, 2, CKKS_DBG_IP_IN);
            const uint4 p = ok ? s4[0] : make_uint4(0u, 0u, 0u, 0u), q4 = ok ? s4[1] : make_uint4(0u, 0u, 0u, 0u);
            d[0] = p.x; d[1] = p.y; d[2] = p.z; d[3] = p.w;
            d[4] = q4.x; d[5] = q4.y; d[6] = q4.z; d[7] = q4.w;
        }
        const uint4 *b4 = reinterpret_cast<const uint4 *>(a.b + ((size_t)j * a.n_primes + t) * n + 8 * blk);
        const bool ok_b = CKKS_SPAN(b4, 2, CKKS_DBG_IP_KEY);
        const uint4 bp = ok_b ? b4[0] : make_uint4(0u, 0u, 0u, 0u), bq = ok_b ? b4[1] : make_uint4(0u, 0u, 0u, 0u);
        const u32 bb[8] = {bp.x, bp.y, bp.z, bp.w, bq.x, bq.y, bq.z, bq.w};
        u32 av[8];
        if (a.a_stored) {
            const uint4 *a4 = reinterpret_cast<const uint4 *>(a.a_stored + ((size_t)j * a.n_primes + t) * n + 8 * blk);
            const bool ok_a = CKKS_SPAN(a4, 2, CKKS_DBG_IP_KEY);
            const uint4 ap = ok_a ? a4[0] : make_uint4(0u, 0u, 0u, 0u), aq = ok_a ? a4[1] : make_uint4(0u, 0u, 0u, 0u);
            av[0] = ap.x; av[1] = ap.y; av[2] = ap.z; av[3] = ap.w;
            av[4] = aq.x; av[5] = aq.y; av[6] = aq.z; av[7] = aq.w;
        } else {
            chacha_coeffs<false>(a.key, a.key_id, (u32)j, (u32)t, (u32)blk, pi, av);
        }
#pragma unroll
        for (int m = 0; m < 8; m++) {
            s0[m] += (u64)d[m] * bb[m];          // < 2^60 per term
            s1[m] += (u64)d[m] * av[m];          // a lazy < 4q: < 2^62 per term
        }
        if ((j & 1) == 1) {
#pragma unroll
            for (int m = 0; m < 8; m++) {
                s0[m] = reduce64_lazy(s0[m], pi.q, pi.r64, pi.r64p, pi.onep);
                s1[m] = reduce64_lazy(s1[m], pi.q, pi.r64, pi.r64p, pi.onep);
            }
        }
    }
    u32 r0[8], r1[8];
#pragma unroll
    for (int m = 0; m < 8; m++) {
        r0[m] = reduce64(s0[m], pi.q, pi.r64, pi.r64p, pi.onep);
        r1[m] = reduce64(s1[m], pi.q, pi.r64, pi.r64p, pi.onep);
    }
    uint4 *o0 = reinterpret_cast<uint4 *>(a.acc + (size_t)u * n + 8 * blk);
    uint4 *o1 = reinterpret_cast<uint4 *>(a.acc + ((size_t)a.ext + u) * n + 8 * blk);
    if (!CKKS_SPAN(o0, 2, CKKS_DBG_IP_OUT) || !CKKS_SPAN(o1, 2, CKKS_DBG_IP_OUT)) return;
    o0[0] = make_uint4(r0[0], r0[1], r0[2], r0[3]);
    o0[1] = make_uint4(r0[4], r0[5], r0[6], r0[7]);
    o1[0] = make_uint4(r1[0], r1[1], r1[2], r1[3]);
    o1[1] = make_uint4(r1[4], r1[5], r1[6], r1[7]);
}

// ---------------------------------------------------------------- tensor product
__global__ void k_tensor(const u32 *x, const u32 *y, u32 *d, const PrimeInfo *pinfo, int log_n,
                         int level) {
    const int n = 1 << log_n;
    const int c4 = blockIdx.x * blockDim.x + threadIdx.x;
    if (c4 >= n / 4) return;
    const int i = blockIdx.y;
    const size_t pl = (size_t)(level + 1) * n;
    const PrimeInfo pi = pinfo[i];
    const size_t off = (size_t)i * n;
    x += blockIdx.z * 2 * pl;
    y += blockIdx.z * 2 * pl;
    d += blockIdx.z * 3 * pl;
    if (!CKKS_SPAN(pinfo + i, 1, CKKS_DBG_TENSOR) || !CKKS_SPAN2(x + off + 4 * c4, x + pl + off + 4 * c4 + 3, CKKS_DBG_TENSOR) ||
        !CKKS_SPAN2(y + off + 4 * c4, y + pl + off + 4 * c4 + 3, CKKS_DBG_TENSOR) ||
        !CKKS_SPAN2(d + off + 4 * c4, d + 2 * pl + off + 4 * c4 + 3, CKKS_DBG_TENSOR))
        return;
    const uint4 x0 = reinterpret_cast<const uint4 *>(x + off)[c4];
    const uint4 x1 = reinterpret_cast<const uint4 *>(x + pl + off)[c4];
    const uint4 y0 = reinterpret_cast<const uint4 *>(y + off)[c4];
    const uint4 y1 = reinterpret_cast<const uint4 *>(y + pl + off)[c4];
    const u32 a0[4] = {x0.x, x0.y, x0.z, x0.w}, a1[4] = {x1.x, x1.y, x1.z, x1.w};
    const u32 b0[4] = {y0.x, y0.y, y0.z, y0.w}, b1[4] = {y1.x, y1.y, y1.z, y1.w};
    u32 r0[4], r1[4], r2[4];
#pragma unroll
    for (int m = 0; m < 4; m++) {
        r0[m] = reduce64((u64)a0[m] * b0[m], pi.q, pi.r64, pi.r64p, pi.onep);
        r1[m] = reduce64((u64)a0[m] * b1[m] + (u64)a1[m] * b0[m], pi.q, pi.r64, pi.r64p, pi.onep);
        r2[m] = reduce64((u64)a1[m] * b1[m], pi.q, pi.r64, pi.r64p, pi.onep);
    }
    reinterpret_cast<uint4 *>(d + off)[c4] = make_uint4(r0[0], r0[1], r0[2], r0[3]);
    reinterpret_cast<uint4 *>(d + pl + off)[c4] = make_uint4(r1[0], r1[1], r1[2], r1[3]);
    reinterpret_cast<uint4 *>(d + 2 * pl + off)[c4] = make_uint4(r2[0], r2[1], r2[2], r2[3]);
}

// ---------------------------------------------------------------- automorphism
__global__ void k_automorph(const u32 *in, u32 *out, int log_n, u32 g) {
    const int n = 1 << log_n;
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= n) return;
    const size_t off = (size_t)blockIdx.y * n;
    if (!CKKS_SPAN(in + off, n, CKKS_DBG_AUTOMORPH) || !CKKS_SPAN(out + off + k, 1, CKKS_DBG_AUTOMORPH)) return;
    out[off + k] = in[off + automorph_src((u32)k, g, log_n)];
}

// Signed integer coefficients into RNS rows: out[row][k] = m[k] mod t (canonical), the rows
// mapped to primes like an NTT job map (the forward NTT follows).
__global__ void k_encode_rns(const long long *m, u32 *out, const PrimeInfo *pinfo, JobMap map, int log_n) {
    const int n = 1 << log_n;
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= n) return;
    int prime, kk;
    size_t in_row, out_row;
    if (!map_job(map, blockIdx.y, prime, in_row, out_row, kk)) return;
    if (!CKKS_SPAN(pinfo + prime, 1, CKKS_DBG_ENCODE) || !CKKS_SPAN(m + k, 1, CKKS_DBG_ENCODE) ||
        !CKKS_SPAN(out + out_row * n + k, 1, CKKS_DBG_ENCODE))
        return;
    const long long q = pinfo[prime].q;
    long long r = m[k] % q;
    if (r < 0) r += q;
    out[out_row * n + k] = (u32)r;
}

// digit limbs of the extended output: dtilde[j][u] = c[u] for u inside digit j
__global__ void k_copy_digit_limbs(const u32 *c, u32 *dt, int log_n, int level, int alpha, int ext) {
    const int n = 1 << log_n;
    const int c4 = blockIdx.x * blockDim.x + threadIdx.x;
    if (c4 >= n / 4) return;
    const int u = blockIdx.y;            // 0..level
    const int j = u / alpha;
    if (!CKKS_SPAN(c + (size_t)u * n + 4 * c4, 4, CKKS_DBG_COPY_DIGIT) ||
        !CKKS_SPAN(dt + ((size_t)j * ext + u) * n + 4 * c4, 4, CKKS_DBG_COPY_DIGIT))
        return;
    reinterpret_cast<uint4 *>(dt + ((size_t)j * ext + u) * n)[c4] =
        reinterpret_cast<const uint4 *>(c + (size_t)u * n)[c4];
}

// ---------------------------------------------------------------- fused row kernels
// The 16-slot layout (k_ip_row): 16 rows x 16 threads per block; at the end of a forward row
// pass (row_fwd_regs) thread (r, lo) holds the 16 consecutive evaluation slots
// k = 256*row + 16*lo + v, v = 0..15.  The other row kernels hold one row per warp (ntt.cuh).

__device__ __forceinline__ void load16_vec(const u32 *p, u32 (&x)[16]) {
    const uint4 *p4 = reinterpret_cast<const uint4 *>(p);
#pragma unroll
    for (int v = 0; v < 4; v++) {
        const uint4 t = p4[v];
        x[4 * v] = t.x; x[4 * v + 1] = t.y; x[4 * v + 2] = t.z; x[4 * v + 3] = t.w;
    }
}

__device__ __forceinline__ void store16_vec(u32 *p, const u32 (&x)[16]) {
    uint4 *p4 = reinterpret_cast<uint4 *>(p);
#pragma unroll
    for (int v = 0; v < 4; v++) p4[v] = make_uint4(x[4 * v], x[4 * v + 1], x[4 * v + 2], x[4 * v + 3]);
}

// the same behind the debug-bounds check of the 16 words (zeros / nothing when it fails)
__device__ __forceinline__ void load16_chk(const u32 *p, u32 (&x)[16], int site) {
    if (CKKS_SPAN(p, 16, site)) {
        load16_vec(p, x);
    } else {
#pragma unroll
        for (int v = 0; v < 16; v++) x[v] = 0u;
    }
}

__device__ __forceinline__ void store16_chk(u32 *p, const u32 (&x)[16], int site) {
    if (CKKS_SPAN(p, 16, site)) store16_vec(p, x);
}

// x[v] = row[lo + 16 v], the round-0 input of a row pass, behind the check of its span
__device__ __forceinline__ void load_row16_chk(const u32 *row, int lo, u32 (&x)[16], int site) {
    const bool ok = CKKS_SPAN2(row + lo, row + lo + 16 * 15, site);
#pragma unroll
    for (int v = 0; v < 16; v++) x[v] = ok ? row[lo + 16 * v] : 0u;
}

// Forward row pass of one row held as round-0 input x[v] = row element lo + 16 v; returns the
// canonical evaluation values of elements 16 lo + v.  srow: this row's 272-word exchange area.
__device__ __forceinline__ void row_fwd_regs(u32 (&x)[16], const tw_t *tw, u32 base, int lo, u32 *srow,
                                             u32 q) {
    const u32 two_q = 2 * q;
    fwd_top4(x, tw, base, q, two_q);
#pragma unroll
    for (int u = 0; u < 16; u++) srow[lo + 17 * u] = x[u];
    __syncwarp();
#pragma unroll
    for (int u = 0; u < 16; u++) x[u] = srow[17 * lo + u];
    __syncwarp();
    fwd_low<8>(x, tw, base, (u32)lo, q, two_q);
#pragma unroll
    for (int u = 0; u < 16; u++) x[u] = csub(csub(x[u], two_q), q);
}

// Inverse row pass of one row held as x[v] = element 16 lo + v (values in [0, 2q)); returns
// elements lo + 16 v, lazily in [0, 2q).
__device__ __forceinline__ void row_inv_regs(u32 (&x)[16], const tw_t *tw, u32 base, int lo, u32 *srow,
                                             u32 q) {
    const u32 two_q = 2 * q;
    inv_low<8>(x, tw, base, (u32)lo, q, two_q);
#pragma unroll
    for (int u = 0; u < 16; u++) srow[17 * lo + u] = x[u];
    __syncwarp();
#pragma unroll
    for (int u = 0; u < 16; u++) x[u] = srow[lo + 17 * u];
    __syncwarp();
    inv_top4(x, tw, base, q, two_q);
}

// Key inner product, with the last forward NTT pass of ModUp fused in (k_ip_row8 below): for every
// active digit j, the extended digit dt_j[u] is completed in registers (forward row pass of the
// column-pass output x[j][u], or the input polynomial itself for u inside digit j), the key's a
// half for (digit j, limb t) is regenerated by ChaCha12 for the same slots, and
//   acc0 += dt_j[u] * b_j[t],  acc1 += dt_j[u] * a_j[t]   (Montgomery products, mod t).
// Rotations: hoist_g != 0 reads every dt_j[u] through kappa_{hoist_g} (hoisted rotation:
// the source row is transformed, then permuted inside the row); cdig_g != 0 reads only the
// input polynomial's digit limbs through kappa_{cdig_g} (single rotation).
// Items whose a half is the same (same seed and key id, regenerated) form a group of up to
// IP_GROUP_MAX: its block regenerates a_j once for all active digits into shared memory and
// then runs the group's items one after another, each with its own b half, inputs and
// rotation.  A group of one keeps the keystream in registers.
// Output: acc rows, canonical evaluation values.
constexpr int IP_GROUP_MAX = 8;
constexpr int IP_GROUP_MAX_BETA = 4;             // digits whose a half fits the shared buffer
constexpr size_t IP_GROUP_SMEM = (size_t)IP_GROUP_MAX_BETA * 16 * ROW_THREADS * sizeof(u32);

struct IpRowArgs {
    const u32 *x;            // [beta][ext][N] ModUp column-pass output (non-digit limbs)
    const u32 *cdig;         // [l+1][N] input polynomial, evaluation domain
    u32 *acc;                // [2][ext][N]
    size_t x_item, cdig_item, acc_item;        // item strides (words; 0 = shared)
    int item_div;            // item z reads x and cdig of source z / item_div (hoisted batches of
                             // several ciphertexts: item_div rotations per ciphertext; 0 reads as 1)
    const tw_t *twf, *twi;
    const PrimeInfo *pinfo;
    int log_n, level, n_q, n_primes, alpha, beta, ext;
    // per item: the key and the rotation
    const u32 *b[KS_MAXB];        // [D][n_primes][N]
    const u32 *a_stored[KS_MAXB]; // nullptr: regenerate
    ChachaKey key[KS_MAXB];
    u32 key_id[KS_MAXB];
    u32 hoist_g[KS_MAXB], cdig_g[KS_MAXB];
    // groups (blockIdx.z): items grp_item[grp_first[g] .. grp_first[g] + grp_count[g] - 1]
    int grp_first[KS_MAXB], grp_count[KS_MAXB], grp_item[KS_MAXB];
};

// The 16-slot inner product (16 rows x 16 threads per block, 16 consecutive slots and two
// ChaCha12 blocks per thread, 128 registers).  XDONE = true is what runs now: a hoisted batch whose
// shared ModUp already holds every non-digit limb in the evaluation domain (run_modup_rows
// transformed them once); those rows are read like the digit limbs, through kappa_{hoist_g},
// instead of being transformed again for every item.  XDONE = false, the same layout with the row
// pass fused in, was the benchmark's kernel until k_ip_row8 replaced it and is no longer launched;
// it stays in this template because the XDONE = true kernel compiled without it measured 1.5-3%
// slower on the hoisted lines (same box).
template <bool XDONE>
__global__ void __launch_bounds__(ROW_THREADS)
k_ip_row(IpRowArgs a) {
    __shared__ u32 sm[16 * 272];
    extern __shared__ u32 sa[];                      // shared a half: [digit][16][ROW_THREADS]
    const int n = 1 << a.log_n;
    const int na = a.level + 1;
    const int u = blockIdx.y;
    const int g0 = a.grp_first[blockIdx.z], gcnt = a.grp_count[blockIdx.z];
    const int t = u < na ? u : a.n_q + (u - na);
    if (!CKKS_SPAN(a.pinfo + t, 1, CKKS_DBG_IPROW_TABLES) || !CKKS_SPAN(a.twf + (size_t)t * n, n, CKKS_DBG_IPROW_TABLES))
        return;                                               // (the same for the whole block)
    CKKS_POISON(sm, sizeof(sm));
    CKKS_POISON_DYNAMIC(sa);
    const PrimeInfo pi = a.pinfo[t];
    const u32 q = pi.q, two_q = 2 * q;
    const int r = threadIdx.x >> 4, lo = threadIdx.x & 15;
    const int row = blockIdx.x * 16 + r;
    const u32 R1 = (u32)(n >> 8);
    u32 *srow = sm + r * 272;
    const int k0 = row * 256 + 16 * lo;              // first evaluation slot of this thread
    const tw_t *twf = a.twf + (size_t)t * n;
    if (gcnt > 1) {                                  // the group's shared a half, once per digit
        const int item = a.grp_item[g0];
        for (int j = 0; j < a.beta; j++) {
            u32 h[8];
            u32 *dst = sa + (size_t)j * 16 * ROW_THREADS + threadIdx.x;
            chacha_coeffs<false>(a.key[item], a.key_id[item], (u32)j, (u32)t, (u32)(k0 >> 3), pi, h);
#pragma unroll
            for (int v = 0; v < 8; v++) dst[v * ROW_THREADS] = h[v];
            chacha_coeffs<false>(a.key[item], a.key_id[item], (u32)j, (u32)t, (u32)(k0 >> 3) + 1u, pi, h);
#pragma unroll
            for (int v = 0; v < 8; v++) dst[(8 + v) * ROW_THREADS] = h[v];
        }
        __syncthreads();
    }
    for (int it = 0; it < gcnt; it++) {
        const int item = a.grp_item[g0 + it];
        const int src_item = item / max(1, a.item_div);
        const u32 *xb = a.x + src_item * a.x_item;
        const u32 *cdb = a.cdig + src_item * a.cdig_item;
        u32 *accb = a.acc + item * a.acc_item;
        const u32 *bkey = a.b[item];
        const u32 *astore = a.a_stored[item];
        const u32 hoist_g = a.hoist_g[item], cdig_g = a.cdig_g[item];
        // hoisted rotation: source row of this row under kappa_g
        const int src_row = hoist_g ? (int)(automorph_src((u32)(row * 256), hoist_g, a.log_n) >> 8) : row;
        u32 acc0[16], acc1[16];
#pragma unroll
        for (int v = 0; v < 16; v++) acc0[v] = acc1[v] = 0;
        for (int j = 0; j < a.beta; j++) {
            const bool in_digit = u < na && u >= j * a.alpha && u < min(j * a.alpha + a.alpha, na);
            u32 x[16];
            if (in_digit || XDONE) {
                const u32 *src = in_digit ? cdb + (size_t)u * n : xb + ((size_t)j * a.ext + u) * n;
                const u32 g = in_digit ? (hoist_g ? hoist_g : cdig_g) : hoist_g;
                if (g) {
                    const bool ok = CKKS_SPAN(src, n, CKKS_DBG_IPROW_CDIG);       // automorph_src < n
#pragma unroll
                    for (int v = 0; v < 16; v++) x[v] = ok ? src[automorph_src((u32)(k0 + v), g, a.log_n)] : 0u;
                } else {
                    load16_chk(src + k0, x, CKKS_DBG_IPROW_CDIG);
                }
            } else {
                const u32 *src = xb + ((size_t)j * a.ext + u) * n + (size_t)src_row * 256;
                load_row16_chk(src, lo, x, CKKS_DBG_IPROW_X);
                row_fwd_regs(x, twf, R1 + (u32)src_row, lo, srow, q);
                if (hoist_g) {        // permute inside the row: slot k takes source slot src(k)
#pragma unroll
                    for (int v = 0; v < 16; v++) srow[17 * lo + v] = x[v];
                    __syncwarp();
#pragma unroll
                    for (int v = 0; v < 16; v++) {
                        const u32 m = automorph_src((u32)(k0 + v), hoist_g, a.log_n) & 255u;
                        x[v] = srow[m + (m >> 4)];
                    }
                    __syncwarp();
                }
            }
            u32 bv[16], av[16];
            load16_chk(bkey + ((size_t)j * a.n_primes + t) * n + k0, bv, CKKS_DBG_IPROW_KEY);
            if (gcnt > 1) {
                const u32 *src = sa + (size_t)j * 16 * ROW_THREADS + threadIdx.x;
#pragma unroll
                for (int v = 0; v < 16; v++) av[v] = src[v * ROW_THREADS];
            } else if (astore) {
                load16_chk(astore + ((size_t)j * a.n_primes + t) * n + k0, av, CKKS_DBG_IPROW_KEY);
            } else {
                u32 h[8];
                chacha_coeffs<false>(a.key[item], a.key_id[item], (u32)j, (u32)t, (u32)(k0 >> 3), pi, h);
#pragma unroll
                for (int v = 0; v < 8; v++) av[v] = h[v];
                chacha_coeffs<false>(a.key[item], a.key_id[item], (u32)j, (u32)t, (u32)(k0 >> 3) + 1u, pi, h);
#pragma unroll
                for (int v = 0; v < 8; v++) av[8 + v] = h[v];
            }
#pragma unroll
            for (int v = 0; v < 16; v++) {
                acc0[v] = csub(acc0[v] + mont_mul(x[v], bv[v], q, pi.qinv), two_q);
                acc1[v] = csub(acc1[v] + mont_mul(x[v], av[v], q, pi.qinv), two_q);
            }
        }
        // undo the Montgomery factor 2^-32
#pragma unroll
        for (int v = 0; v < 16; v++) {
            acc0[v] = csub(shoup_mul(acc0[v], pi.r64, pi.r64p, q), q);
            acc1[v] = csub(shoup_mul(acc1[v], pi.r64, pi.r64p, q), q);
        }
        store16_chk(accb + (size_t)u * n + (size_t)row * 256 + 16 * lo, acc0, CKKS_DBG_IPROW_OUT);
        store16_chk(accb + ((size_t)a.ext + u) * n + (size_t)row * 256 + 16 * lo, acc1, CKKS_DBG_IPROW_OUT);
    }
}

// ---- the inner product with one row per warp: 32 threads x 8 values per 256-point row
// (k_ip_row8), its forward row pass in registers (row8_fwd, ntt.cuh).
__device__ __forceinline__ void load8_chk(const u32 *p, u32 (&x)[8], int site) {
    if (CKKS_SPAN(p, 8, site)) {
        const uint4 *p4 = reinterpret_cast<const uint4 *>(p);
        const uint4 t0 = p4[0], t1 = p4[1];
        x[0] = t0.x; x[1] = t0.y; x[2] = t0.z; x[3] = t0.w; x[4] = t1.x; x[5] = t1.y; x[6] = t1.z; x[7] = t1.w;
    } else {
#pragma unroll
        for (int v = 0; v < 8; v++) x[v] = 0u;
    }
}

__device__ __forceinline__ void store8_chk(u32 *p, const u32 (&x)[8], int site) {
    if (CKKS_SPAN(p, 8, site)) {
        uint4 *p4 = reinterpret_cast<uint4 *>(p);
        p4[0] = make_uint4(x[0], x[1], x[2], x[3]);
        p4[1] = make_uint4(x[4], x[5], x[6], x[7]);
    }
}


// The inner product with the row pass fused in (every launch but a hoisted batch's over finished
// rows): one 256-slot row per warp, a thread holding the 8 consecutive slots
// k0 = 256 row + 8 lo .. + 7, so one ChaCha12 block per digit; 80 registers, 3 blocks of 8 warps
// per SM.  Shared a half of a group: [digit][8][ROW_THREADS].
__global__ void __launch_bounds__(ROW_THREADS, 3)
k_ip_row8(IpRowArgs a) {
    __shared__ u32 sm[ROW_ROWS * ROW_SMEM];
    extern __shared__ u32 sa[];
    const int n = 1 << a.log_n;
    const int na = a.level + 1;
    const int u = blockIdx.y;
    const int g0 = a.grp_first[blockIdx.z], gcnt = a.grp_count[blockIdx.z];
    const int t = u < na ? u : a.n_q + (u - na);
    if (!CKKS_SPAN(a.pinfo + t, 1, CKKS_DBG_IPROW_TABLES) || !CKKS_SPAN(a.twf + (size_t)t * n, n, CKKS_DBG_IPROW_TABLES))
        return;                                               // (the same for the whole block)
    CKKS_POISON(sm, sizeof(sm));
    CKKS_POISON_DYNAMIC(sa);
    const PrimeInfo pi = a.pinfo[t];
    const u32 q = pi.q, two_q = 2 * q;
    const int r = threadIdx.x >> 5, lo = threadIdx.x & 31;
    const int row = blockIdx.x * ROW_ROWS + r;
    const u32 R1 = (u32)(n >> 8);
    u32 *srow = sm + r * ROW_SMEM;
    const int k0 = row * 256 + 8 * lo;               // first evaluation slot of this thread
    const u32 blk = (u32)(k0 >> 3);                  // its ChaCha12 block
    const tw_t *twf = a.twf + (size_t)t * n;
    if (gcnt > 1) {                                  // the group's shared a half, once per digit
        const int item = a.grp_item[g0];
        for (int j = 0; j < a.beta; j++) {
            u32 h[8];
            u32 *dst = sa + (size_t)j * 8 * ROW_THREADS + threadIdx.x;
            chacha_coeffs<false>(a.key[item], a.key_id[item], (u32)j, (u32)t, blk, pi, h);
#pragma unroll
            for (int v = 0; v < 8; v++) dst[v * ROW_THREADS] = h[v];
        }
        __syncthreads();
    }
    for (int it = 0; it < gcnt; it++) {
        const int item = a.grp_item[g0 + it];
        const int src_item = item / max(1, a.item_div);
        const u32 *xb = a.x + src_item * a.x_item;
        const u32 *cdb = a.cdig + src_item * a.cdig_item;
        u32 *accb = a.acc + item * a.acc_item;
        const u32 *bkey = a.b[item];
        const u32 *astore = a.a_stored[item];
        const u32 hoist_g = a.hoist_g[item], cdig_g = a.cdig_g[item];
        const int src_row = hoist_g ? (int)(automorph_src((u32)(row * 256), hoist_g, a.log_n) >> 8) : row;
        u32 acc0[8], acc1[8];
#pragma unroll
        for (int v = 0; v < 8; v++) acc0[v] = acc1[v] = 0;
        for (int j = 0; j < a.beta; j++) {
            const bool in_digit = u < na && u >= j * a.alpha && u < min(j * a.alpha + a.alpha, na);
            u32 x[8];
            if (in_digit) {
                const u32 *src = cdb + (size_t)u * n;
                const u32 g = hoist_g ? hoist_g : cdig_g;
                if (g) {
                    const bool ok = CKKS_SPAN(src, n, CKKS_DBG_IPROW_CDIG);       // automorph_src < n
#pragma unroll
                    for (int v = 0; v < 8; v++) x[v] = ok ? src[automorph_src((u32)(k0 + v), g, a.log_n)] : 0u;
                } else {
                    load8_chk(src + k0, x, CKKS_DBG_IPROW_CDIG);
                }
            } else {
                const u32 *src = xb + ((size_t)j * a.ext + u) * n + (size_t)src_row * 256;
                const bool ok = CKKS_SPAN2(src + lo, src + lo + 32 * 7, CKKS_DBG_IPROW_X);
#pragma unroll
                for (int v = 0; v < 8; v++) x[v] = ok ? src[lo + 32 * v] : 0u;
                row8_fwd(x, twf, R1 + (u32)src_row, lo, srow, q);
                if (hoist_g) {        // permute inside the row: slot k takes source slot src(k)
#pragma unroll
                    for (int v = 0; v < 8; v++) srow[row8_x2(8 * lo + v)] = x[v];
                    __syncwarp();
#pragma unroll
                    for (int v = 0; v < 8; v++) {
                        const int m = (int)(automorph_src((u32)(k0 + v), hoist_g, a.log_n) & 255u);
                        x[v] = srow[row8_x2(m)];
                    }
                    __syncwarp();
                }
            }
            u32 bv[8], av[8];
            load8_chk(bkey + ((size_t)j * a.n_primes + t) * n + k0, bv, CKKS_DBG_IPROW_KEY);
            if (gcnt > 1) {
                const u32 *src = sa + (size_t)j * 8 * ROW_THREADS + threadIdx.x;
#pragma unroll
                for (int v = 0; v < 8; v++) av[v] = src[v * ROW_THREADS];
            } else if (astore) {
                load8_chk(astore + ((size_t)j * a.n_primes + t) * n + k0, av, CKKS_DBG_IPROW_KEY);
            } else {
                chacha_coeffs<false>(a.key[item], a.key_id[item], (u32)j, (u32)t, blk, pi, av);
            }
#pragma unroll
            for (int v = 0; v < 8; v++) {
                acc0[v] = csub(acc0[v] + mont_mul(x[v], bv[v], q, pi.qinv), two_q);
                acc1[v] = csub(acc1[v] + mont_mul(x[v], av[v], q, pi.qinv), two_q);
            }
        }
        // undo the Montgomery factor 2^-32
#pragma unroll
        for (int v = 0; v < 8; v++) {
            acc0[v] = csub(shoup_mul(acc0[v], pi.r64, pi.r64p, q), q);
            acc1[v] = csub(shoup_mul(acc1[v], pi.r64, pi.r64p, q), q);
        }
        store8_chk(accb + (size_t)u * n + k0, acc0, CKKS_DBG_IPROW_OUT);
        store8_chk(accb + ((size_t)a.ext + u) * n + k0, acc1, CKKS_DBG_IPROW_OUT);
    }
}

// Last forward NTT pass of ModDown's converted limbs fused with the combine:
//   out_c[i] = (acc_c[i] - conv_c[i]) [P^-1]_{q_i} + add_c[i]   (mod q_i).
// conv: column-pass output [n_comp][l+1][N]; acc: [2][ext][N] (rows 0..l of each component).
// add: nullptr, [2][l+1][N] (both components), or component 0 only, gathered through
// kappa_{add_g} when add_g != 0.
struct RowCombineArgs {
    const u32 *conv;
    const u32 *acc;
    const u32 *add;
    u32 *out;                // [n_comp][l+1][N]
    size_t conv_item, acc_item, add_item, out_item;   // item strides (words; 0 = shared)
    int add_div;             // item z adds the polynomial of source z / add_div (0 reads as 1)
    const tw_t *twf;
    const PrimeInfo *pinfo;
    const tw_t *pinv;
    int log_n, level, ext, acc_comp_rows, add_comps, n_comp;
    u32 add_g[KS_MAXB];
};

// One 256-slot row per warp and 8 slots per thread (the layout of k_ip_row8): 32 registers, 8 blocks
// per SM, so the latency of the three input streams is hidden by occupancy.
__global__ void __launch_bounds__(ROW_THREADS)
k_row_combine(RowCombineArgs a) {
    __shared__ u32 sm[ROW_ROWS * ROW_SMEM];
    const int n = 1 << a.log_n;
    const int i = blockIdx.y, comp = blockIdx.z % a.n_comp, item = blockIdx.z / a.n_comp;
    const u32 add_g = a.add_g[item];
    const int na = a.level + 1;
    if (!CKKS_SPAN(a.pinfo + i, 1, CKKS_DBG_COMBINE_TABLES) || !CKKS_SPAN(a.pinv + i, 1, CKKS_DBG_COMBINE_TABLES) ||
        !CKKS_SPAN(a.twf + (size_t)i * n, n, CKKS_DBG_COMBINE_TABLES))
        return;                                               // (the same for the whole block)
    CKKS_POISON(sm, sizeof(sm));
    const PrimeInfo pi = a.pinfo[i];
    const u32 q = pi.q;
    const int r = threadIdx.x >> 5, lo = threadIdx.x & 31;
    const int row = blockIdx.x * ROW_ROWS + r;
    const int k0 = row * 256 + 8 * lo;
    u32 *srow = sm + r * ROW_SMEM;
    u32 x[8];
    const u32 *src = a.conv + item * a.conv_item + ((size_t)comp * na + i) * n + (size_t)row * 256;
    const bool ok = CKKS_SPAN2(src + lo, src + lo + 32 * 7, CKKS_DBG_COMBINE_IN);
#pragma unroll
    for (int v = 0; v < 8; v++) x[v] = ok ? src[lo + 32 * v] : 0u;
    row8_fwd(x, a.twf + (size_t)i * n, (u32)(n >> 8) + (u32)row, lo, srow, q);
    u32 ac[8];
    load8_chk(a.acc + item * a.acc_item + ((size_t)comp * a.acc_comp_rows + i) * n + k0, ac, CKKS_DBG_COMBINE_IN);
    const tw_t w = a.pinv[i];
#pragma unroll
    for (int v = 0; v < 8; v++) x[v] = csub(shoup_mul(ac[v] + q - x[v], w.x, w.y, q), q);
    if (comp < a.add_comps) {
        const u32 *ad = a.add + (item / max(1, a.add_div)) * a.add_item + ((size_t)comp * na + i) * n;
        u32 y[8];
        if (add_g) {
            const bool okg = CKKS_SPAN(ad, n, CKKS_DBG_COMBINE_ADD);          // automorph_src < n
#pragma unroll
            for (int v = 0; v < 8; v++) y[v] = okg ? ad[automorph_src((u32)(k0 + v), add_g, a.log_n)] : 0u;
        } else {
            load8_chk(ad + k0, y, CKKS_DBG_COMBINE_ADD);
        }
#pragma unroll
        for (int v = 0; v < 8; v++) x[v] = csub(x[v] + y[v], q);
    }
    store8_chk(a.out + item * a.out_item + ((size_t)comp * na + i) * n + k0, x, CKKS_DBG_COMBINE_OUT);
}

// ---------------------------------------------------------------- baby-step giant-step transform
// Plaintext-diagonal sums of a baby-step giant-step linear transform with double hoisting
// (Bossuat, Mouchet, Troncoso-Pastoriza, Hubaux, Eurocrypt 2021, Sec. 6), in the extended
// basis PQ before any ModDown:
//   V_j[comp][u] = sum_k pt[j][k][u] * X_k[comp][u]   (mod t, t the prime of extended row u),
// X_k = (acc0_k + [P]_t kappa_{g_k}(c0), acc1_k) for a rotated baby, whose accumulators come
// from the hoisted inner product (the P c0 term only on rows u <= l, where P is invertible),
// and X_k = ([P]_t c0, [P]_t c1) on rows u <= l, 0 on the special rows, for the identity baby.
// A thread covers 2 coefficients of one extended row; a launch covers babies k0 .. k0+kc-1
// (their X in registers) and every giant step, carrying partial sums in V between launches.
// n must be a multiple of 512 (true for every supported N).
constexpr int BSGS_KC = 16;
constexpr int BSGS_THREADS = 256;

struct BsgsArgs {
    const u32 *acc;          // baby accumulators: item z at acc + z * acc_item, [2][ext][N]
    size_t acc_item;
    const u32 *ct;           // input ciphertext [2][l+1][N]
    const u32 *pt;           // plaintexts [n_giant][n_baby][ext][N], canonical
    u32 *v;                  // giant sums: item j at v + j * v_item, [2][ext][N]
    size_t v_item;
    const PrimeInfo *pinfo;
    const tw_t *pmod;        // [n_q]: [P]_{q_i} and its Shoup companion
    int log_n, level, n_q, ext, n_baby, n_giant, k0, kc;
    int *err;                // device error word: CKKS_DEV_ERR_WAIT is or-ed in when a wait expires
    int item_of[KS_MAXB];    // baby k -> accumulator item, -1 for the identity baby
    u32 galois[KS_MAXB];     // baby k's Galois element
};

// ---- bulk asynchronous copies into shared memory, completed on an mbarrier (sm_90+ PTX)
__device__ __forceinline__ u32 smem_addr(const void *p) { return (u32)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(u64 *bar, u32 count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(u64 *bar, u32 bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

// global -> this CTA's shared memory, `bytes` a multiple of 16, both addresses 16-byte aligned
__device__ __forceinline__ void bulk_load(void *dst, const void *src, u32 bytes, u64 *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(smem_addr(dst)), "l"(src), "r"(bytes), "r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(u64 *bar, u32 phase) {
    u32 ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_addr(bar)), "r"(phase) : "memory");
    return ok != 0;
}

constexpr int CKKS_DEV_ERR_WAIT = 1;              // a bounded device wait expired
constexpr u64 MBAR_WAIT_NS = 1000000000ull;       // wait bound: 1 s of the global timer
constexpr u32 MBAR_WAIT_TRIES = 1u << 30;         // backstop on the number of try_wait rounds

__device__ __forceinline__ u64 global_ns() {
    u64 t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Waits for `phase` of `bar`; false when MBAR_WAIT_NS (or the round backstop) expires.
__device__ __forceinline__ bool mbar_wait_bounded(u64 *bar, u32 phase) {
    if (mbar_try_wait(bar, phase)) return true;
    const u64 t0 = global_ns();
    for (u32 i = 0; i < MBAR_WAIT_TRIES; i++) {
        if (mbar_try_wait(bar, phase)) return true;
        if (global_ns() - t0 > MBAR_WAIT_NS) return false;
    }
    return false;
}

// Self-test of the bounded-wait failure path: one block waits on an mbarrier that expects two
// arrivals and receives one, so the wait expires after MBAR_WAIT_NS and the error word is set.
// No copy is involved and nothing else waits on this block.
__global__ void k_wait_expiry_probe(int *err) {
    __shared__ __align__(8) u64 bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 2);
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(&bar)) : "memory");
    }
    __syncthreads();
    const bool expired = !mbar_wait_bounded(&bar, 0u);
    if (threadIdx.x == 0 && expired && CKKS_SPAN(err, 1, CKKS_DBG_ERR_WORD)) atomicOr(err, CKKS_DEV_ERR_WAIT);
}

// The plaintexts stream through shared memory: a block covers 512 coefficients (2 per thread)
// of one extended row, and stage s holds one giant step's kc plaintext chunks of 2 KB, loaded
// by one thread with bulk copies on the stage's mbarrier, BSGS_STAGES giant steps ahead of
// the computation.  The babies' terms X stay in registers.
constexpr int BSGS_STAGES = 3;
constexpr int BSGS_CHUNK = 2 * BSGS_THREADS;                 // coefficients per block
constexpr size_t BSGS_SMEM = (size_t)BSGS_STAGES * BSGS_KC * BSGS_CHUNK * sizeof(u32);

__global__ void __launch_bounds__(BSGS_THREADS)
k_bsgs_combine(BsgsArgs a) {
    extern __shared__ __align__(128) u32 sp[];               // [stage][kk][BSGS_CHUNK]
    __shared__ __align__(8) u64 full[BSGS_STAGES];
    const int n = 1 << a.log_n;
    const int tid = threadIdx.x;
    const int c2 = blockIdx.x * BSGS_THREADS + tid;          // coefficient pair of this thread
    const int u = blockIdx.y;
    const int na = a.level + 1;
    const int t = u < na ? u : a.n_q + (u - na);
    if (!CKKS_SPAN(a.pinfo + t, 1, CKKS_DBG_BSGS_TABLES) || (u < na && !CKKS_SPAN(a.pmod + u, 1, CKKS_DBG_BSGS_TABLES)))
        return;                                               // (the same for the whole block)
    CKKS_POISON_DYNAMIC(sp);
    const PrimeInfo pi = a.pinfo[t];
    const u32 q = pi.q;
    const tw_t pm = u < na ? a.pmod[u] : make_uint2(0u, 0u);
    const size_t r0 = (size_t)u * n, r1 = ((size_t)a.ext + u) * n;     // component rows in [2][ext]
    const size_t plane = (size_t)a.ext * n;                  // one plaintext
    const u32 stage_bytes = (u32)(a.kc * BSGS_CHUNK * sizeof(u32));
    const u32 *pbase = a.pt + (size_t)a.k0 * plane + r0 + (size_t)blockIdx.x * BSGS_CHUNK;
    if (tid == 0) {
        for (int st = 0; st < BSGS_STAGES; st++) mbar_init(&full[st], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    // thread 0: giant step j's plaintext chunks into stage j % BSGS_STAGES
    auto issue = [&](int j) {
        const int st = j % BSGS_STAGES;
        const u32 *src = pbase + (size_t)j * a.n_baby * plane;
#ifdef CKKS_DEBUG_BOUNDS
        // a chunk outside the registered regions is not copied, and the stage expects its bytes less
        u32 okm = 0, bytes = 0;
        (void)stage_bytes;
        for (int kk = 0; kk < a.kc; kk++)
            if (CKKS_SPAN(src + (size_t)kk * plane, BSGS_CHUNK, CKKS_DBG_BSGS_PT)) {
                okm |= 1u << kk;
                bytes += BSGS_CHUNK * sizeof(u32);
            }
        mbar_expect_tx(&full[st], bytes);
        for (int kk = 0; kk < a.kc; kk++)
            if ((okm >> kk) & 1u)
                bulk_load(sp + ((size_t)st * BSGS_KC + kk) * BSGS_CHUNK, src + (size_t)kk * plane,
                          BSGS_CHUNK * sizeof(u32), &full[st]);
#else
        mbar_expect_tx(&full[st], stage_bytes);
        for (int kk = 0; kk < a.kc; kk++)
            bulk_load(sp + ((size_t)st * BSGS_KC + kk) * BSGS_CHUNK, src + (size_t)kk * plane,
                      BSGS_CHUNK * sizeof(u32), &full[st]);
#endif
    };
    if (tid == 0)
        for (int j = 0; j < BSGS_STAGES && j < a.n_giant; j++) issue(j);
    // the babies' terms for this thread's two coefficients (overlaps the first copies)
    u32 x0[BSGS_KC][2], x1[BSGS_KC][2];
#pragma unroll
    for (int kk = 0; kk < BSGS_KC; kk++) {
        x0[kk][0] = x0[kk][1] = x1[kk][0] = x1[kk][1] = 0;
        if (kk < a.kc) {
            const int k = a.k0 + kk;
            const int z = a.item_of[k];
            if (z < 0) {
                if (u < na && CKKS_SPAN2(a.ct + (size_t)u * n + 2 * c2, a.ct + ((size_t)na + u) * n + 2 * c2 + 1,
                                         CKKS_DBG_BSGS_IN)) {
                    const uint2 v0 = reinterpret_cast<const uint2 *>(a.ct + (size_t)u * n)[c2];
                    const uint2 v1 = reinterpret_cast<const uint2 *>(a.ct + ((size_t)na + u) * n)[c2];
                    x0[kk][0] = csub(shoup_mul(v0.x, pm.x, pm.y, q), q);
                    x0[kk][1] = csub(shoup_mul(v0.y, pm.x, pm.y, q), q);
                    x1[kk][0] = csub(shoup_mul(v1.x, pm.x, pm.y, q), q);
                    x1[kk][1] = csub(shoup_mul(v1.y, pm.x, pm.y, q), q);
                }
            } else {
                const u32 *ac = a.acc + (size_t)z * a.acc_item;
                const bool ok = CKKS_SPAN2(ac + r0 + 2 * c2, ac + r1 + 2 * c2 + 1, CKKS_DBG_BSGS_IN);
                const uint2 v0 = ok ? reinterpret_cast<const uint2 *>(ac + r0)[c2] : make_uint2(0u, 0u);
                const uint2 v1 = ok ? reinterpret_cast<const uint2 *>(ac + r1)[c2] : make_uint2(0u, 0u);
                u32 e0 = v0.x, e1 = v0.y;
                if (u < na && CKKS_SPAN(a.ct + (size_t)u * n, n, CKKS_DBG_BSGS_IN)) {     // automorph_src < n
                    const u32 *c0 = a.ct + (size_t)u * n;
                    const u32 g = a.galois[k];
                    e0 = csub(e0 + csub(shoup_mul(c0[automorph_src((u32)(2 * c2), g, a.log_n)], pm.x, pm.y, q), q), q);
                    e1 = csub(e1 + csub(shoup_mul(c0[automorph_src((u32)(2 * c2 + 1), g, a.log_n)], pm.x, pm.y, q), q), q);
                }
                x0[kk][0] = e0; x0[kk][1] = e1;
                x1[kk][0] = v1.x; x1[kk][1] = v1.y;
            }
        }
    }
    for (int j = 0; j < a.n_giant; j++) {
        const int st = j % BSGS_STAGES;
        const bool expired = !mbar_wait_bounded(&full[st], (u32)(j / BSGS_STAGES) & 1u);
        if (__syncthreads_or(expired)) {
            // leave together: record the failure, let this block's copies in flight land
            if (tid == 0) {
                if (CKKS_SPAN(a.err, 1, CKKS_DBG_ERR_WORD)) atomicOr(a.err, CKKS_DEV_ERR_WAIT);
                for (int jj = j; jj < j + BSGS_STAGES && jj < a.n_giant; jj++)
                    (void)mbar_wait_bounded(&full[jj % BSGS_STAGES], (u32)(jj / BSGS_STAGES) & 1u);
            }
            return;
        }
        u32 *vj = a.v + (size_t)j * a.v_item;
        const bool ok_v = CKKS_SPAN2(vj + r0 + 2 * c2, vj + r1 + 2 * c2 + 1, CKKS_DBG_BSGS_V);
        // a canonical carry plus 16 products of two values below q < 2^30 stays below 2^64
        u64 s00 = 0, s01 = 0, s10 = 0, s11 = 0;              // [component][coefficient]
        if (a.k0 && ok_v) {
            const uint2 w0 = reinterpret_cast<const uint2 *>(vj + r0)[c2];
            const uint2 w1 = reinterpret_cast<const uint2 *>(vj + r1)[c2];
            s00 = w0.x; s01 = w0.y; s10 = w1.x; s11 = w1.y;
        }
        const uint2 *ps = reinterpret_cast<const uint2 *>(sp + (size_t)st * BSGS_KC * BSGS_CHUNK) + tid;
#pragma unroll
        for (int kk = 0; kk < BSGS_KC; kk++) {
            if (kk < a.kc) {
                const uint2 p = ps[(size_t)kk * (BSGS_CHUNK / 2)];
                s00 += (u64)p.x * x0[kk][0]; s01 += (u64)p.y * x0[kk][1];
                s10 += (u64)p.x * x1[kk][0]; s11 += (u64)p.y * x1[kk][1];
            }
        }
        if (ok_v) {
            reinterpret_cast<uint2 *>(vj + r0)[c2] =
                make_uint2(reduce64(s00, q, pi.r64, pi.r64p, pi.onep), reduce64(s01, q, pi.r64, pi.r64p, pi.onep));
            reinterpret_cast<uint2 *>(vj + r1)[c2] =
                make_uint2(reduce64(s10, q, pi.r64, pi.r64p, pi.onep), reduce64(s11, q, pi.r64, pi.r64p, pi.onep));
        }
        __syncthreads();                                     // stage st fully read
        if (tid == 0 && j + BSGS_STAGES < a.n_giant) issue(j + BSGS_STAGES);
    }
}

// out[r] = sum_s src_s[r] (mod q_(r mod (l+1))) over 2(l+1) rows [2][l+1][N]; 4 coefficients
// per thread.
struct SumArgs {
    const u32 *src[KS_MAXB];
    int n_src;
    u32 *out;
    const PrimeInfo *pinfo;
    int log_n, level;
};

__global__ void __launch_bounds__(256)
k_sum_parts(SumArgs a) {
    const int n = 1 << a.log_n;
    const int c4 = blockIdx.x * blockDim.x + threadIdx.x;
    if (4 * c4 >= n) return;
    const int r = blockIdx.y;
    if (!CKKS_SPAN(a.pinfo + r % (a.level + 1), 1, CKKS_DBG_SUM) ||
        !CKKS_SPAN(a.out + (size_t)r * n + 4 * c4, 4, CKKS_DBG_SUM))
        return;
    const u32 q = a.pinfo[r % (a.level + 1)].q;
    uint4 s = make_uint4(0u, 0u, 0u, 0u);
    for (int i = 0; i < a.n_src; i++) {
        if (!CKKS_SPAN(a.src[i] + (size_t)r * n + 4 * c4, 4, CKKS_DBG_SUM)) continue;
        const uint4 v = reinterpret_cast<const uint4 *>(a.src[i] + (size_t)r * n)[c4];
        s.x = csub(s.x + v.x, q); s.y = csub(s.y + v.y, q); s.z = csub(s.z + v.z, q); s.w = csub(s.w + v.w, q);
    }
    reinterpret_cast<uint4 *>(a.out + (size_t)r * n)[c4] = s;
}

// ---------------------------------------------------------------- base conversion on the tensor cores
#include "bconv_tc.cuh"
