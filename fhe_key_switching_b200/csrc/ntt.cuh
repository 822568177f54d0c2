// ntt.cuh -- two-pass negacyclic NTT for N = R1 * 256 (R1 = 2^r1, 4 <= r1 <= 8).
//
// Definition (the library's evaluation domain): A[k] = sum_n a[n] psi^((2 brv(k)+1) n) mod q.
// Schedule: the iterative Cooley-Tukey transform with the psi powers merged into the
// twiddles; global stage s pairs j and j + N/2^(s+1) with twiddle psi^brv(idx),
// idx = 2^s + (j >> (log_n - s)).  Its output is the definition above in bit-reversed order.
//
// The N coefficients are viewed as a R1 x 256 row-major matrix (j = 256*m + col for the
// column pass, j = 256*row + m for the row pass):
//   column pass = global stages 0 .. r1-1: independent length-R1 transforms down each
//                 column, twiddle idx = 2^s + (m >> (r1 - s));
//   row pass    = global stages r1 .. log_n-1: independent length-256 transforms along each
//                 row, twiddle idx = ((R1 + row) << s) + (m >> (8 - s)), s = 0..7 local.
// Each pass runs 16 elements per thread in two register rounds with one shared-memory
// exchange between them:
//   round 0: the top 4 bits of m vary in registers (m = lo + (R/16) u, u = 0..15),
//   round 1: the remaining low bits (m = 16 lo + u).
// The inverse passes undo the forward stages in reverse order with Gentleman-Sande
// butterflies and the psi^-brv(idx) table.
#pragma once
#include "debug_bounds.cuh"
#include "modarith.cuh"

// Twiddle record: (w, Shoup companion of w).
typedef uint2 tw_t;

// ---------------------------------------------------------------- register blocks

// Forward round over the top 4 bits: stage s (0..3) pairs (u, u + (8 >> s)); group g = u /
// (16 >> s) uses idx = (base << s) + g.
__device__ __forceinline__ void fwd_top4(u32 (&x)[16], const tw_t *__restrict__ tw, u32 base,
                                         u32 q, u32 two_q) {
#pragma unroll
    for (int s = 0; s < 4; s++) {
        const int d = 8 >> s;
#pragma unroll
        for (int g = 0; g < (1 << s); g++) {
            const tw_t w = __ldg(tw + (base << s) + g);
#pragma unroll
            for (int i = 0; i < d; i++) ct_bfly(x[2 * d * g + i], x[2 * d * g + i + d], w.x, w.y, q, two_q);
        }
    }
}

// Forward round over the low RLOG-4 bits of m = 16 lo + u: global-in-pass stage s = 4 ..
// RLOG-1 pairs (u, u + d), d = 2^(RLOG-1-s); group g = u / 2d uses
// idx = (base << s) + (lo << (s - RLOG + 4)) + g.
template <int RLOG>
__device__ __forceinline__ void fwd_low(u32 (&x)[16], const tw_t *__restrict__ tw, u32 base, u32 lo,
                                        u32 q, u32 two_q) {
#pragma unroll
    for (int s = 4; s < RLOG; s++) {
        const int d = 1 << (RLOG - 1 - s);
        const u32 gbase = (base << s) + (lo << (s - RLOG + 4));
#pragma unroll
        for (int g = 0; g < 16 / (2 * d); g++) {
            const tw_t w = __ldg(tw + gbase + g);
#pragma unroll
            for (int i = 0; i < d; i++) ct_bfly(x[2 * d * g + i], x[2 * d * g + i + d], w.x, w.y, q, two_q);
        }
    }
}

template <int RLOG>
__device__ __forceinline__ void inv_low(u32 (&x)[16], const tw_t *__restrict__ tw, u32 base, u32 lo,
                                        u32 q, u32 two_q) {
#pragma unroll
    for (int s = RLOG - 1; s >= 4; s--) {
        const int d = 1 << (RLOG - 1 - s);
        const u32 gbase = (base << s) + (lo << (s - RLOG + 4));
#pragma unroll
        for (int g = 0; g < 16 / (2 * d); g++) {
            const tw_t w = __ldg(tw + gbase + g);
#pragma unroll
            for (int i = 0; i < d; i++) gs_bfly(x[2 * d * g + i], x[2 * d * g + i + d], w.x, w.y, q, two_q);
        }
    }
}

__device__ __forceinline__ void inv_top4(u32 (&x)[16], const tw_t *__restrict__ tw, u32 base,
                                         u32 q, u32 two_q) {
#pragma unroll
    for (int s = 3; s >= 0; s--) {
        const int d = 8 >> s;
#pragma unroll
        for (int g = 0; g < (1 << s); g++) {
            const tw_t w = __ldg(tw + (base << s) + g);
#pragma unroll
            for (int i = 0; i < d; i++) gs_bfly(x[2 * d * g + i], x[2 * d * g + i + d], w.x, w.y, q, two_q);
        }
    }
}

// ---------------------------------------------------------------- job mapping
// A launch processes a batch of limbs ("jobs", blockIdx.y).  Job y belongs to group
// g = y / per_group at position k = y % per_group; its prime is global limb lo_base + k for
// k < split, hi_base + (k - split) otherwise (the extended basis q_0..q_l, p_0..).  With
// skip_alpha > 0, positions inside digit g ([g*alpha, min(g*alpha+alpha, split))) are skipped
// (ModUp leaves digit limbs untouched).
struct JobMap {
    int per_group, split, lo_base, hi_base;
    int in_group_rows, out_group_rows, in_k_base, out_k_base;
    int skip_alpha;
};

__device__ __forceinline__ bool map_job(const JobMap &m, int y, int &prime, size_t &in_row,
                                        size_t &out_row, int &k) {
    const int g = y / m.per_group;
    k = y - g * m.per_group;
    if (m.skip_alpha > 0) {
        const int lo = g * m.skip_alpha;
        const int hi = min(lo + m.skip_alpha, m.split);
        if (k >= lo && k < hi) return false;
    }
    prime = k < m.split ? m.lo_base + k : m.hi_base + (k - m.split);
    in_row = (size_t)g * m.in_group_rows + m.in_k_base + k;
    out_row = (size_t)g * m.out_group_rows + m.out_k_base + k;
    return true;
}

// Evaluation-domain automorphism source index: out[k] = in[src(k)] with
// 2 brv(src)+1 = (2 brv(k)+1) g mod 2N.
__device__ __forceinline__ u32 automorph_src(u32 k, u32 g, int log_n) {
    const u32 kb = __brev(k) >> (32 - log_n);
    const u32 e = ((2u * kb + 1u) * g) & ((2u << log_n) - 1u);
    return __brev((e - 1u) >> 1) >> (32 - log_n);
}

// Batches: blockIdx.z selects an item; item z reads in + z*in_item and writes out + z*out_item
// (strides in words).
constexpr int KS_MAXB = 64;                 // items per launch

struct NttArgs {
    const u32 *in;
    u32 *out;
    const tw_t *tw;         // [n_primes][N] forward or inverse table
    const PrimeInfo *pinfo; // [n_primes]
    const tw_t *scale;      // per-k output scale (inverse column pass), or nullptr
    JobMap map;
    int log_n;
    size_t in_item, out_item;
    // forward column pass only, lift_q != 0: every job of group g reads the group's single
    // input row (in_group_rows * g + in_k_base), a canonical residue y mod lift_q, and
    // transforms its centred lift (y - lift_q if y > lift_half) reduced mod the job's prime
    u32 lift_q, lift_half;
    u32 galois[KS_MAXB];    // inverse row pass: gather item z's input through kappa_g (0 = none)
};

// ---------------------------------------------------------------- column pass (stages 0..r1-1)
// Block: (R1/16) "lo" values x CPB columns; warp = 32 consecutive columns at one lo.
template <int R1LOG>
struct ColCfg {
    static constexpr int R1 = 1 << R1LOG;
    static constexpr int LOS = R1 / 16;                       // threads per column
    static constexpr int CPB = (8192 / R1) < 256 ? (8192 / R1) : 256;  // columns per block
    static constexpr int THREADS = LOS * CPB;
};

// FWD: forward stages, output lazy in [0, 4q).  !FWD: inverse stages, output multiplied by
// scale[k] (or N^-1 when scale is null) and canonical.
// Three blocks per SM (at most 42 registers for 512 threads): 7% faster than the compiler's
// unconstrained 47 registers and two blocks, with no spills.
template <int R1LOG, bool FWD>
__global__ void __launch_bounds__(ColCfg<R1LOG>::THREADS, 3)
k_ntt_col(NttArgs a) {
    using C = ColCfg<R1LOG>;
    __shared__ u32 sm[C::R1 * C::CPB];
    int prime, k;
    size_t in_row, out_row;
    if (!map_job(a.map, blockIdx.y, prime, in_row, out_row, k)) return;
    const int n = 1 << a.log_n;
    if (!CKKS_SPAN(a.pinfo + prime, 1, CKKS_DBG_NTT_TABLES) ||
        !CKKS_SPAN(a.tw + (size_t)prime * n, n, CKKS_DBG_NTT_TABLES) ||
        (!FWD && a.scale && !CKKS_SPAN(a.scale + k, 1, CKKS_DBG_NTT_TABLES)))
        return;                                               // (the same for the whole block)
    CKKS_POISON(sm, sizeof(sm));
    const PrimeInfo pi = a.pinfo[prime];
    const u32 q = pi.q, two_q = 2 * q;
    const tw_t *tw = a.tw + (size_t)prime * n;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cgroups = C::CPB / 32;
    const int lo = warp / cgroups;
    const int ccol = (warp % cgroups) * 32 + lane;          // column within block
    const int col = blockIdx.x * C::CPB + ccol;
    const u32 *src = a.in + blockIdx.z * a.in_item + (FWD && a.lift_q ? in_row - k : in_row) * n;
    u32 *dst = a.out + blockIdx.z * a.out_item + out_row * n;
    u32 x[16];
    if (FWD) {
        const bool ok_in = CKKS_SPAN2(src + (size_t)lo * 256 + col, src + (size_t)(lo + C::LOS * 15) * 256 + col,
                                      CKKS_DBG_NTT_IN);
#pragma unroll
        for (int u = 0; u < 16; u++) x[u] = ok_in ? src[(size_t)(lo + C::LOS * u) * 256 + col] : 0u;
        if (a.lift_q) {
            // y - lift_q + 2q lies in (2q - lift_q/2, 2q), inside the butterflies' [0, 4q) input
#pragma unroll
            for (int u = 0; u < 16; u++) x[u] = x[u] > a.lift_half ? x[u] + two_q - a.lift_q : x[u];
        }
        fwd_top4(x, tw, 1u, q, two_q);
#pragma unroll
        for (int u = 0; u < 16; u++) sm[(lo + C::LOS * u) * C::CPB + ccol] = x[u];
        __syncthreads();
#pragma unroll
        for (int u = 0; u < 16; u++) x[u] = sm[(16 * lo + u) * C::CPB + ccol];
        fwd_low<R1LOG>(x, tw, 1u, (u32)lo, q, two_q);
        if (CKKS_SPAN2(dst + (size_t)(16 * lo) * 256 + col, dst + (size_t)(16 * lo + 15) * 256 + col, CKKS_DBG_NTT_OUT)) {
#pragma unroll
            for (int u = 0; u < 16; u++) dst[(size_t)(16 * lo + u) * 256 + col] = x[u];
        }
    } else {
        const bool ok_in = CKKS_SPAN2(src + (size_t)(16 * lo) * 256 + col, src + (size_t)(16 * lo + 15) * 256 + col,
                                      CKKS_DBG_NTT_IN);
#pragma unroll
        for (int u = 0; u < 16; u++) x[u] = ok_in ? src[(size_t)(16 * lo + u) * 256 + col] : 0u;
        inv_low<R1LOG>(x, tw, 1u, (u32)lo, q, two_q);
#pragma unroll
        for (int u = 0; u < 16; u++) sm[(16 * lo + u) * C::CPB + ccol] = x[u];
        __syncthreads();
#pragma unroll
        for (int u = 0; u < 16; u++) x[u] = sm[(lo + C::LOS * u) * C::CPB + ccol];
        inv_top4(x, tw, 1u, q, two_q);
        u32 w = pi.n_inv, wp = pi.n_invp;
        if (a.scale) { const tw_t s = a.scale[k]; w = s.x; wp = s.y; }
        if (CKKS_SPAN2(dst + (size_t)lo * 256 + col, dst + (size_t)(lo + C::LOS * 15) * 256 + col, CKKS_DBG_NTT_OUT)) {
#pragma unroll
            for (int u = 0; u < 16; u++)
                dst[(size_t)(lo + C::LOS * u) * 256 + col] = csub(shoup_mul(x[u], w, wp, q), q);
        }
    }
}

// ---------------------------------------------------------------- row pass (stages r1..log_n-1)
// One 256-point row per warp: 32 threads x 8 values.  A row pass runs in three register rounds,
//   A: m = lo + 32 u (u = 0..7), local stages 0..2;
//   B: m = 32 (lo >> 2) + 4 u + (lo & 3), stages 3..5;
//   C: m = 8 lo + u, stages 6..7,
// local stage s pairing (m, m + 2^(7-s)) with twiddle (base << s) + (m >> (8 - s)) of the
// bit-reversed table (base = N/256 + row); the inverse runs the rounds backwards (C, B, A).  The
// exchanges go through the row's 288 words of shared memory at m + 4 (m >> 5) (A <-> B) and
// m + (m >> 3) (B <-> C), both free of bank conflicts for the two patterns that use them.
constexpr int ROW_THREADS = 256;
constexpr int ROW_ROWS = ROW_THREADS / 32;       // rows per block: one per warp
constexpr int ROW_SMEM = 288;                    // shared words per row

__device__ __forceinline__ int row8_x1(int m) { return m + 4 * (m >> 5); }
__device__ __forceinline__ int row8_x2(int m) { return m + (m >> 3); }

// Forward: x[u] = element lo + 32 u of the row (round A's input) -> canonical evaluation values of
// the elements 8 lo + u.
__device__ __forceinline__ void row8_fwd(u32 (&x)[8], const tw_t *__restrict__ tw, u32 base, int lo, u32 *srow,
                                         u32 q) {
    const u32 two_q = 2 * q;
#pragma unroll
    for (int s = 0; s < 3; s++) {
        const int d = 4 >> s;
#pragma unroll
        for (int g = 0; g < (1 << s); g++) {
            const tw_t w = __ldg(tw + (base << s) + g);
#pragma unroll
            for (int i = 0; i < d; i++) ct_bfly(x[2 * d * g + i], x[2 * d * g + i + d], w.x, w.y, q, two_q);
        }
    }
#pragma unroll
    for (int u = 0; u < 8; u++) srow[row8_x1(lo + 32 * u)] = x[u];
    __syncwarp();
    const int a = lo >> 2, b = lo & 3;
#pragma unroll
    for (int u = 0; u < 8; u++) x[u] = srow[row8_x1(32 * a + 4 * u + b)];
    __syncwarp();
#pragma unroll
    for (int s = 3; s < 6; s++) {
        const int d = 4 >> (s - 3);
#pragma unroll
        for (int g = 0; g < (1 << (s - 3)); g++) {
            const tw_t w = __ldg(tw + (base << s) + ((u32)a << (s - 3)) + g);
#pragma unroll
            for (int i = 0; i < d; i++) ct_bfly(x[2 * d * g + i], x[2 * d * g + i + d], w.x, w.y, q, two_q);
        }
    }
#pragma unroll
    for (int u = 0; u < 8; u++) srow[row8_x2(32 * a + 4 * u + b)] = x[u];
    __syncwarp();
#pragma unroll
    for (int u = 0; u < 8; u++) x[u] = srow[row8_x2(8 * lo + u)];
    __syncwarp();
#pragma unroll
    for (int s = 6; s < 8; s++) {
        const int d = 1 << (7 - s);
#pragma unroll
        for (int g = 0; g < 8 / (2 * d); g++) {
            const tw_t w = __ldg(tw + (base << s) + ((u32)lo << (s - 5)) + g);
#pragma unroll
            for (int i = 0; i < d; i++) ct_bfly(x[2 * d * g + i], x[2 * d * g + i + d], w.x, w.y, q, two_q);
        }
    }
#pragma unroll
    for (int u = 0; u < 8; u++) x[u] = csub(csub(x[u], two_q), q);
}


// Inverse: x[u] = element 8 lo + u of the row (round C's layout), inputs in [0, 2q) -> elements
// lo + 32 u after the inverse stages 7..0, lazy in [0, 2q).
__device__ __forceinline__ void row8_inv(u32 (&x)[8], const tw_t *__restrict__ tw, u32 base, int lo, u32 *srow,
                                         u32 q) {
    const u32 two_q = 2 * q;
#pragma unroll
    for (int s = 7; s >= 6; s--) {
        const int d = 1 << (7 - s);
#pragma unroll
        for (int g = 0; g < 8 / (2 * d); g++) {
            const tw_t w = __ldg(tw + (base << s) + ((u32)lo << (s - 5)) + g);
#pragma unroll
            for (int i = 0; i < d; i++) gs_bfly(x[2 * d * g + i], x[2 * d * g + i + d], w.x, w.y, q, two_q);
        }
    }
#pragma unroll
    for (int u = 0; u < 8; u++) srow[row8_x2(8 * lo + u)] = x[u];
    __syncwarp();
    const int a = lo >> 2, b = lo & 3;
#pragma unroll
    for (int u = 0; u < 8; u++) x[u] = srow[row8_x2(32 * a + 4 * u + b)];
    __syncwarp();
#pragma unroll
    for (int s = 5; s >= 3; s--) {
        const int d = 4 >> (s - 3);
#pragma unroll
        for (int g = 0; g < (1 << (s - 3)); g++) {
            const tw_t w = __ldg(tw + (base << s) + ((u32)a << (s - 3)) + g);
#pragma unroll
            for (int i = 0; i < d; i++) gs_bfly(x[2 * d * g + i], x[2 * d * g + i + d], w.x, w.y, q, two_q);
        }
    }
#pragma unroll
    for (int u = 0; u < 8; u++) srow[row8_x1(32 * a + 4 * u + b)] = x[u];
    __syncwarp();
#pragma unroll
    for (int u = 0; u < 8; u++) x[u] = srow[row8_x1(lo + 32 * u)];
    __syncwarp();
#pragma unroll
    for (int s = 2; s >= 0; s--) {
        const int d = 4 >> s;
#pragma unroll
        for (int g = 0; g < (1 << s); g++) {
            const tw_t w = __ldg(tw + (base << s) + g);
#pragma unroll
            for (int i = 0; i < d; i++) gs_bfly(x[2 * d * g + i], x[2 * d * g + i + d], w.x, w.y, q, two_q);
        }
    }
}

// FWD: forward stages, canonical output.  !FWD: inverse stages (input gathered through
// kappa_g when galois != 0), output lazy in [0, 2q).
template <bool FWD>
__global__ void __launch_bounds__(ROW_THREADS)
k_ntt_row(NttArgs a) {
    __shared__ u32 sm[ROW_ROWS * ROW_SMEM];
    int prime, k;
    size_t in_row, out_row;
    if (!map_job(a.map, blockIdx.y, prime, in_row, out_row, k)) return;
    const int n = 1 << a.log_n;
    if (!CKKS_SPAN(a.pinfo + prime, 1, CKKS_DBG_NTT_TABLES) || !CKKS_SPAN(a.tw + (size_t)prime * n, n, CKKS_DBG_NTT_TABLES))
        return;                                               // (the same for the whole block)
    CKKS_POISON(sm, sizeof(sm));
    const u32 q = a.pinfo[prime].q;
    const tw_t *tw = a.tw + (size_t)prime * n;
    const int r = threadIdx.x >> 5, lo = threadIdx.x & 31;
    const int row = blockIdx.x * ROW_ROWS + r;
    const u32 base = (u32)(n >> 8) + (u32)row;
    const u32 *src = a.in + blockIdx.z * a.in_item + in_row * n;
    u32 *dst = a.out + blockIdx.z * a.out_item + out_row * n + (size_t)row * 256;
    const u32 galois = a.galois[blockIdx.z];
    u32 *srow = sm + r * ROW_SMEM;
    u32 x[8];
    if (FWD) {
        const u32 *s = src + (size_t)row * 256;
        const bool ok_in = CKKS_SPAN2(s + lo, s + lo + 32 * 7, CKKS_DBG_NTT_IN);
#pragma unroll
        for (int u = 0; u < 8; u++) x[u] = ok_in ? s[lo + 32 * u] : 0u;
        row8_fwd(x, tw, base, lo, srow, q);
        if (CKKS_SPAN(dst + 8 * lo, 8, CKKS_DBG_NTT_OUT)) {
            uint4 *d4 = reinterpret_cast<uint4 *>(dst + 8 * lo);
            d4[0] = make_uint4(x[0], x[1], x[2], x[3]);
            d4[1] = make_uint4(x[4], x[5], x[6], x[7]);
        }
    } else {
        if (galois) {
            const bool ok_in = CKKS_SPAN(src, n, CKKS_DBG_NTT_IN);          // automorph_src < n
#pragma unroll
            for (int u = 0; u < 8; u++)
                x[u] = ok_in ? src[automorph_src((u32)(row * 256 + 8 * lo + u), galois, a.log_n)] : 0u;
        } else {
            const uint4 *s4 = reinterpret_cast<const uint4 *>(src + (size_t)row * 256 + 8 * lo);
            const bool ok_in = CKKS_SPAN(s4, 2, CKKS_DBG_NTT_IN);
            const uint4 t0 = ok_in ? s4[0] : make_uint4(0u, 0u, 0u, 0u);
            const uint4 t1 = ok_in ? s4[1] : make_uint4(0u, 0u, 0u, 0u);
            x[0] = t0.x; x[1] = t0.y; x[2] = t0.z; x[3] = t0.w; x[4] = t1.x; x[5] = t1.y; x[6] = t1.z; x[7] = t1.w;
        }
        row8_inv(x, tw, base, lo, srow, q);
        if (CKKS_SPAN2(dst + lo, dst + lo + 32 * 7, CKKS_DBG_NTT_OUT)) {
#pragma unroll
            for (int u = 0; u < 8; u++) dst[lo + 32 * u] = x[u];
        }
    }
}
