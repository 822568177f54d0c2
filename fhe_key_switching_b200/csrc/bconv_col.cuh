// bconv_col.cuh -- base conversion on the tensor cores fused with the first forward NTT pass.
//
// ModUp and ModDown convert a group's inputs onto every target limb and then run the forward
// column pass (global stages 0 .. r1-1 of ntt.cuh) on each converted limb.  k_bconv_col does both
// in one CTA for a block of TCF_C = 8 columns of the R1 x 256 coefficient matrix (all R1 rows,
// 8 R1 coefficients) and a chunk of up to tcf_max_t(R1) targets (8 at R1 = 256, 16 at 128, 32
// below: the targets' blocks share one fixed shared-memory budget):
//   - the conversion of k_bconv_tc: the same exact u8 x u8 -> s32 contraction with accumulators
//     in tensor memory and the same byte-split constants, with the rows of coefficient tile k
//     taken down the block's columns (row r: m = 16 k + r / 8, column col0 + r % 8);
//   - its outputs (lazily reduced, in [0, 4t)) kept in shared memory, one [R1][8] block per target;
//   - the column pass of each target read from there by the four epilogue warps (round 0 over
//     the top 4 bits of m, an exchange in place, round 1 over the rest, exactly as k_ntt_col),
//     and stored to the target's output row, lazily reduced in [0, 4t) like k_ntt_col's output.
// The converted limbs are never written to HBM and read back.
//
// Shared-memory block of one target: element (m, c) at m * 8 + c + 8 (m >> 4), one pad row after
// every 16 rows.  The skew keeps the epilogue's writes (4 consecutive m x 8 columns per warp),
// round 0 (m = lo + LOS v, 4 consecutive lo per warp, one 16-row group) and round 1
// (m = 16 lo + v: word 136 lo + 8 v + c, banks 8 lo + c + const) free of bank conflicts.
#pragma once
#include "ks_kernels.cuh"

constexpr int TCF_C = 8;                      // columns per CTA
constexpr int TCF_STAGES = 4;                 // A ring: the inputs of three tiles ahead are in flight
// targets per chunk at R1 = 2^r1log: the blocks of 8 R1 words (+ skew) fit 68 KB; at most 32
// (an accumulator of 128 tensor-memory columns)
__host__ __device__ constexpr int tcf_max_t(int r1log) { return r1log >= 8 ? 8 : r1log == 7 ? 16 : 32; }
constexpr int TCF_T_CAP = 32;
constexpr int TCF_B_OFF = TCF_STAGES * TC_A_BYTES;
constexpr int TCF_REC_OFF = TCF_B_OFF + 4 * (4 * TCF_T_CAP) * 16;
constexpr int TCF_X_OFF = TCF_REC_OFF + TCF_T_CAP * 16;
constexpr int TCF_X_BYTES = 68 * 1024;
// A ring + B + records + the targets' blocks: two CTAs per SM
constexpr size_t TCF_SMEM = 109 * 1024;
static_assert(TCF_X_OFF + TCF_X_BYTES <= (int)TCF_SMEM, "fused conversion: shared memory");
static_assert(TCF_STAGES == 4, "the producer loop waits with cp.async.wait_group 3");

__device__ __forceinline__ void tcf_cp_wait3() { asm volatile("cp.async.wait_group 3;" ::: "memory"); }

struct BconvColArgs {
    BconvTcArgs t;           // the conversion (BconvTcArgs::tiles is not used: R1 / 16 tiles per CTA)
    const tw_t *tw;          // forward twiddles [n_primes][N]
};

__device__ __forceinline__ int tcf_xidx(int m, int c) { return m * TCF_C + c + 8 * (m >> 4); }

// barrier 1 over the four epilogue warps (128 threads)
__device__ __forceinline__ void tcf_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// the same barrier, returning whether any of the 128 threads passed p = true
__device__ __forceinline__ bool tcf_bar_or(bool p) {
    u32 r;
    asm volatile("{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.or.pred q, 1, 128, p;\n\t"
                 "selp.u32 %0, 1, 0, q;\n\t}"
                 : "=r"(r) : "r"((u32)p) : "memory");
    return r != 0;
}

// Roles and barriers as in k_bconv_tc (warps 0-3 produce A tiles, warp 8 issues the MMAs, warps
// 4-7 read the accumulators back); the epilogue warps then run the column passes, meeting on
// barrier 1 only.  Every mbarrier wait is bounded; after an expired wait no column pass runs.
template <int R1LOG>
__global__ void __launch_bounds__(TC_THREADS) k_bconv_col(BconvColArgs args) {
    constexpr int R1 = 1 << R1LOG, LOS = R1 / 16;
    constexpr int TILES = R1 * TCF_C / TC_M;                      // R1 / 16 coefficient tiles
    constexpr int XS = R1 * TCF_C + R1 / 2;                       // words per target block
    constexpr int MAX_T = tcf_max_t(R1LOG);
    constexpr int ACC_COLS = 4 * MAX_T;                           // one accumulator
    constexpr int TMEM_COLS = 2 * ACC_COLS;                       // two (64, 128 or 256 columns)
    static_assert(MAX_T * XS * 4 <= TCF_X_BYTES && MAX_T <= TCF_T_CAP, "fused conversion: target blocks");
    const BconvTcArgs &a = args.t;
    extern __shared__ __align__(1024) unsigned char tc_sm[];
    __shared__ __align__(8) u64 a_full[TCF_STAGES], a_empty[TCF_STAGES], acc_full[2], acc_empty[2];
    __shared__ u32 tmem_base;
    __shared__ volatile int abort_flag;
    __shared__ u32 half_s[TC_MAX_IN];
    unsigned char *Bs = tc_sm + TCF_B_OFF;                        // [4 K chunks][N rows][16 B]
    uint4 *trec = reinterpret_cast<uint4 *>(tc_sm + TCF_REC_OFF); // per target: (t, 2t, Shoup(2^16), row * N)
    u32 *X = reinterpret_cast<u32 *>(tc_sm + TCF_X_OFF);          // [target][XS]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int g = a.g_base + blockIdx.y;
    const int item = blockIdx.z / a.nchunk, chunk = blockIdx.z % a.nchunk;
    const int n = 1 << a.log_n;
    const int col0 = blockIdx.x * TCF_C;
    const int n_in = (g == a.n_groups - 1) ? a.n_in_last : a.n_in_full;
    const int cfg = a.cfg_per_group ? g * a.cfg_per_group + (n_in - 1) : 0;
    const int T = a.map.per_group;
    const int lo_s = a.map.skip_alpha > 0 ? g * a.map.skip_alpha : 0;
    const int hi_s = a.map.skip_alpha > 0 ? min(lo_s + a.map.skip_alpha, a.map.split) : 0;
    const int u0 = chunk * a.tchunk;
    const int Tc = min(a.tchunk, T - (hi_s - lo_s) - u0);         // targets of this chunk
    if (Tc <= 0) return;                                          // (uniform: before any barrier)
    const int N = (4 * Tc + 15) & ~15;
    auto target_pos = [&](int u) { const int idx = u0 + u; return idx < lo_s ? idx : idx + (hi_s - lo_s); };
    auto prime_of = [&](int kk) { return kk < a.map.split ? a.map.lo_base + kk : a.map.hi_base + (kk - a.map.split); };
    const int p0 = a.in_prime0 + g * a.in_prime_step;
    const u32 *yb = a.y + item * a.y_item + (size_t)(a.in_row0 + g * a.in_group_rows) * n;
    u32 *ob = a.out + item * a.out_item + ((size_t)g * a.map.out_group_rows + a.map.out_k_base) * n;
    auto a_stage = [&](int tile) { return tc_sm + (size_t)(tile % TCF_STAGES) * TC_A_BYTES; };
    if (!CKKS_SPAN(a.pinfo + p0, n_in, CKKS_DBG_TC_TABLES) ||
        !CKKS_SPAN(a.pinfo + a.map.lo_base, a.map.split, CKKS_DBG_TC_TABLES) ||
        (T > a.map.split && !CKKS_SPAN(a.pinfo + a.map.hi_base, T - a.map.split, CKKS_DBG_TC_TABLES)))
        return;                                                   // (the same for the whole block)
    CKKS_POISON_DYNAMIC(tc_sm);
    // ---- set-up (all threads): constants, B tile, zero padding of the A rows, barriers, memory
    for (int i = tid; i < n_in; i += TC_THREADS) half_s[i] = a.pinfo[p0 + i].half;
    for (int u = tid; u < Tc; u += TC_THREADS) {
        const int kk = target_pos(u);
        const PrimeInfo pi = a.pinfo[prime_of(kk)];
        trec[u] = make_uint4(pi.q, 2u * pi.q, (pi.onep << 16) + (pi.r64p >> 16), (u32)kk * (u32)n);
    }
    for (int idx = tid; idx < 4 * N; idx += TC_THREADS) {
        const int kc = idx / N, col = idx - kc * N;
        const int u = col >> 2, c = col & 3;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (u < Tc) {
            const uint4 *e = a.tb + ((size_t)cfg * a.n_primes + prime_of(target_pos(u))) * 16 + c * 4 + kc;
            if (CKKS_SPAN(e, 1, CKKS_DBG_TC_TABLES)) v = *e;
        }
        reinterpret_cast<uint4 *>(Bs)[(size_t)kc * N + col] = v;
    }
    if (tid < TC_M)          // words n_in + 1 .. 15 of every row stay zero (the copies never write them)
        for (int st = 0; st < TCF_STAGES; st++) {
            u32 *row = reinterpret_cast<u32 *>(tc_sm + (size_t)st * TC_A_BYTES + (size_t)tid * 16);
            for (int i = n_in + 1; i < 16; i++) row[(i >> 2) * (TC_M * 4) + (i & 3)] = 0u;
        }
    if (warp == 8) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(tc_smem_u32(&tmem_base)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        if (lane == 0) {
            for (int st = 0; st < TCF_STAGES; st++) { mbar_init(&a_full[st], TC_M); mbar_init(&a_empty[st], 1); }
            for (int b = 0; b < 2; b++) { mbar_init(&acc_full[b], 1); mbar_init(&acc_empty[b], TC_M); }
            abort_flag = 0;
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
    }
    tc_fence_async_smem();                                        // B visible to the tensor cores
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const u32 tmem = tmem_base;
    auto fail_wait = [&]() {
        if (!abort_flag && CKKS_SPAN(a.err, 1, CKKS_DBG_ERR_WORD)) atomicOr(a.err, CKKS_DEV_ERR_WAIT);
        abort_flag = 1;
    };
    auto wait_or_abort = [&](u64 *bar, u32 parity) {              // false: aborted
        if (abort_flag) return false;
        if (!tc_wait_bounded(bar, parity)) { fail_wait(); return false; }
        return true;
    };
    if (warp < 4) {
        // ---- producers: row tid of every tile, TCF_STAGES - 1 tiles of copies in flight
        const int row_i = tid;
        auto finish = [&](int k) {                                // tile k's copies have landed
            uint4 *row4 = reinterpret_cast<uint4 *>(a_stage(k) + (size_t)row_i * 16);
            u32 w[16];
#pragma unroll
            for (int kc = 0; kc < 4; kc++) {
                const uint4 v4 = row4[kc * TC_M];
                w[4 * kc] = v4.x; w[4 * kc + 1] = v4.y; w[4 * kc + 2] = v4.z; w[4 * kc + 3] = v4.w;
            }
            u32 vcount = 0;
#pragma unroll
            for (int i = 0; i < TC_MAX_IN; i++)
                if (i < n_in) vcount += w[i] > half_s[i] ? 1u : 0u;
            reinterpret_cast<u32 *>(row4)[(n_in >> 2) * (TC_M * 4) + (n_in & 3)] = vcount;
            tc_fence_async_smem();                                // visible to the tensor cores
            tc_arrive(&a_full[k % TCF_STAGES]);
        };
        // row r of tile k: coefficient j = 256 m + col0 + r % 8 with m = 16 k + r / 8
        const u32 *src0 = yb + (size_t)256 * (row_i >> 3) + col0 + (row_i & 7);
        int k = 0;
        for (; k < TILES; k++) {
            if (k >= TCF_STAGES && !wait_or_abort(&a_empty[k % TCF_STAGES], (u32)(((k / TCF_STAGES) - 1) & 1))) break;
            const u32 *src = src0 + (size_t)4096 * k;
            unsigned char *row = a_stage(k) + (size_t)row_i * 16;
            const bool ok_in = CKKS_SPAN2(src, src + (size_t)(n_in - 1) * n, CKKS_DBG_TC_IN);
#pragma unroll
            for (int i = 0; i < TC_MAX_IN; i++) {
                if (i < n_in && ok_in) tc_cp_async4(row + (i >> 2) * (TC_M * 16) + (i & 3) * 4, src);
                src += n;
            }
            tc_cp_commit();
            if (k >= TCF_STAGES - 1) {
                tcf_cp_wait3();                                   // tile k - 3 has landed
                finish(k - (TCF_STAGES - 1));
            }
        }
        tc_cp_wait0();
        if (k == TILES)
            for (int t = max(0, TILES - (TCF_STAGES - 1)); t < TILES; t++) finish(t);
    } else if (warp < 8) {
        // ---- epilogue: lanes 32 (warp - 4) .. + 31 of each accumulator into the targets' blocks
        const int q = warp - 4;
        const int row_i = q * 32 + lane;
        bool ok = true;
        for (int k = 0; k < TILES; k++) {
            if (!wait_or_abort(&acc_full[k & 1], (u32)((k >> 1) & 1))) { ok = false; break; }
            tc_fence_after();
            const int xi = tcf_xidx(16 * k + (row_i >> 3), row_i & 7);
            const u32 acc = tmem + ((u32)(q * 32) << 16) + (u32)((k & 1) * ACC_COLS);
            for (int c0 = 0; c0 < 4 * Tc; c0 += 16) {
                u32 r[16];
                tc_ld16(acc + (u32)c0, r);
                tc_wait_ld();
#pragma unroll
                for (int j = 0; j < 4; j++) {
                    const int u = (c0 >> 2) + j;
                    if (u < Tc) {
                        const uint4 rec = trec[u];
                        const u32 s1 = r[4 * j] + (r[4 * j + 1] << 8);
                        const u32 s2 = r[4 * j + 2] + (r[4 * j + 3] << 8);
                        X[u * XS + xi] = shoup_mul(s2, 65536u, rec.z, rec.x) + csub(s1, rec.y);
                    }
                }
            }
            tc_fence_before();
            tc_arrive(&acc_empty[k & 1]);
        }
        // ---- the forward column pass of every target of the chunk, from shared memory
        if (!tcf_bar_or(!ok || abort_flag)) {                     // (the same decision for all 128)
            const int te = tid - 128, c = te & 7, lo = te >> 3;
            const bool act = lo < LOS;
            for (int u = 0; u < Tc; u++) {                        // round 0: the top 4 bits of m
                const uint4 rec = trec[u];
                const tw_t *tw = args.tw + (size_t)prime_of(target_pos(u)) * n;
                u32 *Xu = X + u * XS;
                if (act && CKKS_SPAN(tw, n, CKKS_DBG_TC_TABLES)) {
                    u32 x[16];
#pragma unroll
                    for (int v = 0; v < 16; v++) x[v] = Xu[tcf_xidx(lo + LOS * v, c)];
                    fwd_top4(x, tw, 1u, rec.x, rec.y);
#pragma unroll
                    for (int v = 0; v < 16; v++) Xu[tcf_xidx(lo + LOS * v, c)] = x[v];
                }
            }
            tcf_bar();
            for (int u = 0; u < Tc; u++) {                        // round 1: the remaining bits
                const uint4 rec = trec[u];
                const tw_t *tw = args.tw + (size_t)prime_of(target_pos(u)) * n;
                const u32 *Xu = X + u * XS;
                u32 *dst = ob + rec.w + col0 + c;
                if (act && CKKS_SPAN(tw, n, CKKS_DBG_TC_TABLES) &&
                    CKKS_SPAN2(dst + (size_t)(16 * lo) * 256, dst + (size_t)(16 * lo + 15) * 256, CKKS_DBG_TC_OUT)) {
                    u32 x[16];
#pragma unroll
                    for (int v = 0; v < 16; v++) x[v] = Xu[tcf_xidx(16 * lo + v, c)];
                    fwd_low<R1LOG>(x, tw, 1u, (u32)lo, rec.x, rec.y);
#pragma unroll
                    for (int v = 0; v < 16; v++) dst[(size_t)(16 * lo + v) * 256] = x[v];
                }
            }
        }
    } else if (lane == 0) {
        // ---- MMA issuer
        const u32 idesc = tc_idesc(TC_M, N);
        const u32 b_base = tc_smem_u32(Bs);
        int issued = 0;
        for (int k = 0; k < TILES; k++) {
            if (!wait_or_abort(&a_full[k % TCF_STAGES], (u32)((k / TCF_STAGES) & 1))) break;
            if (k >= 2 && !wait_or_abort(&acc_empty[k & 1], (u32)(((k >> 1) - 1) & 1))) break;
            tc_fence_after();
            const u32 a_base = tc_smem_u32(a_stage(k));
            const u32 d = tmem + (u32)((k & 1) * ACC_COLS);
#pragma unroll
            for (int s = 0; s < 2; s++)
                tc_mma(d, tc_smem_desc(a_base + (u32)(2 * s * TC_M * 16), TC_M * 16, 128),
                       tc_smem_desc(b_base + (u32)(2 * s * N * 16), (u32)N * 16, 128), idesc, (u32)s);
            tc_commit(&acc_full[k & 1]);
            tc_commit(&a_empty[k % TCF_STAGES]);
            issued = k + 1;
        }
        if (abort_flag) {
            // the MMAs of the last two issued tiles may still run: wait for them (bounded)
            for (int t = issued - 2; t < issued; t++)
                if (t >= 0) (void)tc_wait_bounded(&acc_full[t & 1], (u32)((t >> 1) & 1));
        }
    }
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}
