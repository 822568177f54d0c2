// bconv_tc.cuh -- fast base conversion as an 8-bit integer contraction on the tensor cores
// (tcgen05.mma kind::i8, accumulators in tensor memory).
//
// The conversion of one group (a ModUp digit or the ModDown special primes) is
//   out_t[n] = sum_i y_i[n] [D/r_i]_t + v[n] [-D]_t   (mod t),   v[n] = #{i : y_i[n] > (r_i-1)/2},
// the centred fast base conversion (Cheon, Han, Kim, Kim, Song, SAC 2018) that k_bconv_n computes
// with 64-bit multiply-adds.  Here it is split into bytes so that it becomes an exact u8 x u8 ->
// s32 matrix product:
//   A[n][k] = byte a of y_i[n] for k = 4i + a (i < n_in), A[n][4 n_in] = v[n], 0 beyond;
//   B'[k][t] = [[D/r_i]_t 2^(8a)]_t for k = 4i + a, B'[4 n_in][t] = [-D]_t;
//   B[k][4u + c] = byte c of B'[k][t_u]   (4 columns per target t_u);
//   G[n][4u + c] = sum_k A[n][k] B[k][4u + c]  <  64 * 255 * 255 < 2^22  (exact in s32);
//   out_t[n] = sum_c G[n][4u + c] 2^(8c) = s1 + s2 2^16 (mod t) with s1 = G0 + 2^8 G1 and
//   s2 = G2 + 2^8 G3, both below 2^31, reduced with one Shoup product by [2^16]_t = 2^16.
// Since sum_k A[n][k] B'[k][t] = sum_i y_i [D/r_i]_t + v [-D]_t exactly as integers modulo t,
// the result is the same residue as k_bconv_n's; like it, it is left lazily in [0, 4t), which
// the forward NTT that always follows accepts.
//
// Tile: M = 128 coefficients (one per tensor-memory lane), K = 64 bytes (n_in <= 15), N = 4 x
// (targets of the chunk), at most 256 columns, so that one chunk covers every target of a ModUp
// digit or of ModDown at the supported sizes and each input is gathered once.  A CTA stages the
// chunk's B once, then loops over coefficient tiles with warp-specialized roles (one producer
// thread brings each tile's n_in input rows of 512 bytes into a staging ring with bulk copies,
// producer warps transpose each coefficient's n_in inputs into one A row in shared memory, one
// lane issues the two K = 32 MMAs, epilogue warps read the accumulators back with tcgen05.ld,
// combine them and store one coalesced 128-byte row segment per warp and target; see k_bconv_tc).  Accumulators:
// two of 128 columns when N <= 128, so that the MMAs of a tile overlap the read-back of the
// previous one, else one of N columns.
// Both operands are K-major without swizzle: core matrices of 8 rows x 16 bytes, stored
// [16-byte K chunk][row][16 bytes], so the leading-dimension offset (next K chunk) is
// rows x 16 bytes and the stride-dimension offset (next 8 rows) is 128 bytes.
#pragma once
#include "ntt.cuh"

constexpr int TC_M = 128;                 // coefficients per tile = tensor-memory lanes
constexpr int TC_K = 64;                  // K bytes (two MMAs of K = 32)
constexpr int TC_MAX_IN = 15;             // 4 * 15 + 1 = 61 <= 64
constexpr int TC_MAX_T = 64;              // targets per chunk: N = 4 T <= 256 columns (one MMA)
constexpr int TC_THREADS = 288;           // 4 producer warps, 4 epilogue warps, 1 MMA warp
constexpr int TC_TILES = 16;              // coefficient tiles per CTA, at most (BconvTcArgs::tiles)
constexpr int TC_MIN_TILES = 4;           // smaller launches use the CUDA-core kernel
constexpr int TC_STAGES = 5;              // A ring: the inputs of four tiles ahead are in flight
constexpr int TC_COLS = 256;              // tensor-memory columns a CTA allocates: the accumulator(s)
// Dynamic shared memory per CTA: the A ring (5 x 8 KB) + B (<= 16 KB) + target records + the input
// staging ring (5 x 7.5 KB), at most 2 CTAs per SM (2 x 256 columns = all 512 columns of tensor
// memory: no CTA waits in alloc; 3 x 96 KB would exceed the SM's 228 KB).
constexpr size_t TC_SMEM = 96 * 1024;
constexpr int TC_A_BYTES = 4 * TC_M * 16;  // one A stage: [4 K chunks][128 rows][16 B]
constexpr int TC_RAW_BYTES = TC_MAX_IN * TC_M * 4;   // one staging stage: [input row][128 words]

struct BconvTcArgs {
    const u32 *y;            // input rows
    u32 *out;                // output rows
    const uint4 *tb;         // per (config, global prime t): [4 columns c][4 K chunks] x 16 bytes
    const PrimeInfo *pinfo;
    JobMap map;              // targets: per_group, split, bases, out rows, skip_alpha
    int n_primes, log_n;
    int in_row0, in_group_rows, in_prime0, in_prime_step;
    int n_in_full, n_in_last, n_groups, cfg_per_group, g_base;
    int nchunk, tchunk;      // target chunks per item (blockIdx.z = item * nchunk + chunk)
    int tiles;               // coefficient tiles of 128 per CTA (1 .. TC_TILES; fewer for small launches)
    size_t y_item, out_item;
    int *err;                // device error word: CKKS_DEV_ERR_WAIT when a wait expires
};

__device__ __forceinline__ u32 tc_smem_u32(const void *p) { return (u32)__cvta_generic_to_shared(p); }

// K-major, no swizzle: start address, leading-dimension byte offset (next 16-byte K chunk),
// stride-dimension byte offset (next 8 rows), descriptor version 1, layout type 0.
__device__ __forceinline__ u64 tc_smem_desc(u32 addr, u32 lbo, u32 sbo) {
    return (u64)((addr >> 4) & 0x3FFFu) | ((u64)((lbo >> 4) & 0x3FFFu) << 16) |
           ((u64)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Instruction descriptor of kind::i8: s32 accumulator, unsigned 8-bit A and B, both K-major,
// N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr u32 tc_idesc(int m, int n) {
    return (2u << 4) | ((u32)(n >> 3) << 17) | ((u32)(m >> 4) << 24);
}

__device__ __forceinline__ void tc_mma(u32 d_tmem, u64 adesc, u64 bdesc, u32 idesc, u32 accumulate) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
                 ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

__device__ __forceinline__ void tc_commit(u64 *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 ::"r"(tc_smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tc_ld16(u32 taddr, u32 (&r)[16]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
                 "%12, %13, %14, %15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                   "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
                   "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
}

__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// Bounded wait for `phase` of `bar` in which the waiting thread sleeps in try_wait (up to a
// microsecond per try, the suspend-time hint) instead of spinning; false after 1 s of the
// global timer or the try-count backstop.
__device__ __forceinline__ bool tc_wait_bounded(u64 *bar, u32 phase) {
    const u64 t0 = global_ns();
    for (u32 i = 0; i < MBAR_WAIT_TRIES; i++) {
        u32 ok;
        asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(ok) : "r"(tc_smem_u32(bar)), "r"(phase), "r"(1000u) : "memory");
        if (ok) return true;
        if (global_ns() - t0 > MBAR_WAIT_NS) return false;
    }
    return false;
}

// Included by ks_kernels.cuh after the mbarrier and bulk-copy helpers (mbar_init, mbar_expect_tx,
// bulk_load, CKKS_DEV_ERR_WAIT), which the kernel below uses.
__device__ __forceinline__ void tc_arrive(u64 *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(tc_smem_u32(bar)) : "memory");
}
constexpr int TC_B_OFF = TC_STAGES * TC_A_BYTES;                          // B after the A ring
constexpr int TC_REC_OFF = TC_B_OFF + 4 * (4 * TC_MAX_T) * 16;            // per-target records after B
constexpr int TC_RAW_OFF = TC_REC_OFF + TC_MAX_T * 16;                    // input staging ring after them
static_assert(TC_RAW_OFF % 128 == 0 && TC_RAW_BYTES % 16 == 0, "tensor-core conversion: staging alignment");
static_assert(TC_RAW_OFF + TC_STAGES * TC_RAW_BYTES <= (int)TC_SMEM, "tensor-core conversion: shared memory");

// Roles: warps 0-3 produce the A tiles (thread 0 also issues the bulk copies of every tile's input
// rows into the staging ring, TC_STAGES tiles ahead; thread t then transposes coefficient t's
// inputs into row t of the A tile and appends the centred-lift count), warp 8 (one lane) issues
// the MMAs, warps 4-7 read the accumulators back and store the outputs.  They meet on mbarriers
// only:
//   raw_full[s] (thread 0's expect_tx + the copies' bytes)  staging stage s holds tile k's inputs;
//   raw_empty[s](128 producer arrivals)   every producer has read staging stage s;
//   a_full[s]   (128 producer arrivals)  stage s holds tile k's A;
//   a_empty[s]  (tcgen05.commit)          the MMA of the stage's tile is done with it;
//   acc_full[b] (tcgen05.commit)          accumulator b holds tile k's G;
//   acc_empty[b](128 epilogue arrivals)   accumulator b has been read.
// Every wait is bounded: on expiry the CTA's abort flag and the device error word are set and
// every role leaves its loop; thread 0 then waits (bounded) for the copies it issued and the MMA
// warp for its MMAs in flight, before the CTA ends and the tensor memory is freed.
__global__ void __launch_bounds__(TC_THREADS) k_bconv_tc(BconvTcArgs a) {
    extern __shared__ __align__(1024) unsigned char tc_sm[];
    __shared__ __align__(8) u64 a_full[TC_STAGES], a_empty[TC_STAGES], acc_full[2], acc_empty[2];
    __shared__ __align__(8) u64 raw_full[TC_STAGES], raw_empty[TC_STAGES];
    __shared__ u32 tmem_base;
    __shared__ volatile int abort_flag;
    __shared__ u32 half_s[TC_MAX_IN];
    unsigned char *Bs = tc_sm + TC_B_OFF;                         // [4 K chunks][N rows][16 B]
    uint4 *trec = reinterpret_cast<uint4 *>(tc_sm + TC_REC_OFF);  // per target: (t, 2t, Shoup(2^16), row * N)
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int tiles = a.tiles;
    const int g = a.g_base + blockIdx.y;
    const int item = blockIdx.z / a.nchunk, chunk = blockIdx.z % a.nchunk;
    const int n = 1 << a.log_n;
    const int n_in = (g == a.n_groups - 1) ? a.n_in_last : a.n_in_full;
    const int cfg = a.cfg_per_group ? g * a.cfg_per_group + (n_in - 1) : 0;
    const int T = a.map.per_group;
    const int lo = a.map.skip_alpha > 0 ? g * a.map.skip_alpha : 0;
    const int hi = a.map.skip_alpha > 0 ? min(lo + a.map.skip_alpha, a.map.split) : 0;
    const int u0 = chunk * a.tchunk;
    const int Tc = min(a.tchunk, T - (hi - lo) - u0);             // targets of this chunk
    if (Tc <= 0) return;                                          // (uniform: before any barrier)
    const int N = (4 * Tc + 15) & ~15;
    // two accumulators of 128 columns when N fits one, else a single one of N <= 256 columns
    // (the MMA of tile k + 1 then waits until tile k's accumulator has been read)
    const int nacc = N <= 128 ? 2 : 1;
    auto acc_slot = [&](int k) { return nacc == 2 ? (k & 1) : 0; };
    auto acc_phase = [&](int k) { return (u32)((nacc == 2 ? (k >> 1) : k) & 1); };
    auto target_pos = [&](int u) { const int idx = u0 + u; return idx < lo ? idx : idx + (hi - lo); };
    auto prime_of = [&](int kk) { return kk < a.map.split ? a.map.lo_base + kk : a.map.hi_base + (kk - a.map.split); };
    const int p0 = a.in_prime0 + g * a.in_prime_step;
    const u32 *yb = a.y + item * a.y_item + (size_t)(a.in_row0 + g * a.in_group_rows) * n;
    u32 *ob = a.out + item * a.out_item + ((size_t)g * a.map.out_group_rows + a.map.out_k_base) * n;
    auto a_stage = [&](int tile) { return tc_sm + (size_t)(tile % TC_STAGES) * TC_A_BYTES; };
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
        // floor(2^48 / t) = 2^16 floor(2^32 / t) + floor(2^16 [2^32]_t / t), the last term being
        // the Shoup companion of [2^32]_t shifted right by 16
        trec[u] = make_uint4(pi.q, 2u * pi.q, (pi.onep << 16) + (pi.r64p >> 16), (u32)kk * (u32)n);
    }
    for (int idx = tid; idx < 4 * N; idx += TC_THREADS) {        // B: (K chunk, column) -> 16 bytes
        const int kc = idx / N, col = idx - kc * N;
        const int u = col >> 2, c = col & 3;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (u < Tc) {
            const uint4 *e = a.tb + ((size_t)cfg * a.n_primes + prime_of(target_pos(u))) * 16 + c * 4 + kc;
            if (CKKS_SPAN(e, 1, CKKS_DBG_TC_TABLES)) v = *e;
        }
        reinterpret_cast<uint4 *>(Bs)[(size_t)kc * N + col] = v;
    }
    if (warp == 8) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(tc_smem_u32(&tmem_base)), "r"(TC_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
        if (lane == 0) {
            for (int st = 0; st < TC_STAGES; st++) {
                mbar_init(&a_full[st], TC_M); mbar_init(&a_empty[st], 1);
                mbar_init(&raw_full[st], 1); mbar_init(&raw_empty[st], TC_M);
            }
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
        // ---- producers: row tid of every tile; thread 0 keeps TC_STAGES tiles of copies in flight
        const int row_i = tid;
        auto raw_stage = [&](int t) { return tc_sm + TC_RAW_OFF + (size_t)(t % TC_STAGES) * TC_RAW_BYTES; };
        auto issue = [&](int t) {                                 // thread 0: tile t's input rows
            u64 *bar = &raw_full[t % TC_STAGES];
            unsigned char *dst = raw_stage(t);
            const u32 *src = yb + (size_t)(blockIdx.x * tiles + t) * TC_M;
#ifdef CKKS_DEBUG_BOUNDS
            // a row outside the registered regions is not copied, and the stage expects its bytes less
            u32 okm = 0, bytes = 0;
            for (int i = 0; i < n_in; i++)
                if (CKKS_SPAN(src + (size_t)i * n, TC_M, CKKS_DBG_TC_IN)) { okm |= 1u << i; bytes += TC_M * 4; }
            mbar_expect_tx(bar, bytes);
            for (int i = 0; i < n_in; i++)
                if ((okm >> i) & 1u) bulk_load(dst + (size_t)i * TC_M * 4, src + (size_t)i * n, TC_M * 4, bar);
#else
            mbar_expect_tx(bar, (u32)(n_in * TC_M * 4));
            for (int i = 0; i < n_in; i++) bulk_load(dst + (size_t)i * TC_M * 4, src + (size_t)i * n, TC_M * 4, bar);
#endif
        };
        int issued = 0;
        if (tid == 0)
            for (; issued < TC_STAGES && issued < tiles; issued++) issue(issued);
        int k = 0;
        for (; k < tiles; k++) {
            const int st = k % TC_STAGES;
            const u32 ph = (u32)((k / TC_STAGES) & 1);
            if (k >= TC_STAGES && !wait_or_abort(&a_empty[st], ph ^ 1u)) break;
            if (!wait_or_abort(&raw_full[st], ph)) break;
            const u32 *raw = reinterpret_cast<const u32 *>(raw_stage(k));
            u32 w[16];
            u32 vcount = 0;
#pragma unroll
            for (int i = 0; i < 16; i++) {
                w[i] = 0u;
                if (i < n_in) {
                    w[i] = raw[i * TC_M + row_i];
                    vcount += w[i] > half_s[i] ? 1u : 0u;
                }
            }
#pragma unroll
            for (int i = 0; i < 16; i++)
                if (i == n_in) w[i] = vcount;
            uint4 *row4 = reinterpret_cast<uint4 *>(a_stage(k) + (size_t)row_i * 16);
#pragma unroll
            for (int kc = 0; kc < 4; kc++) row4[kc * TC_M] = make_uint4(w[4 * kc], w[4 * kc + 1], w[4 * kc + 2], w[4 * kc + 3]);
            tc_fence_async_smem();                                // visible to the tensor cores
            tc_arrive(&a_full[st]);
            tc_arrive(&raw_empty[st]);
            if (tid == 0 && issued < tiles) {                     // refill this staging stage
                if (!wait_or_abort(&raw_empty[st], ph)) break;
                tc_fence_async_smem();                            // the reads above before the copies' writes
                issue(issued++);
            }
        }
        if (tid == 0 && abort_flag)                               // copies still in flight: wait (bounded)
            for (int t = k; t < issued; t++) (void)tc_wait_bounded(&raw_full[t % TC_STAGES], (u32)((t / TC_STAGES) & 1));
    } else if (warp < 8) {
        // ---- epilogue: lanes 32 (warp - 4) .. + 31 of each accumulator
        const int q = warp - 4;
        const int row_i = q * 32 + lane;
        for (int k = 0; k < tiles; k++) {
            if (!wait_or_abort(&acc_full[acc_slot(k)], acc_phase(k))) break;
            tc_fence_after();
            const int nc = (blockIdx.x * tiles + k) * TC_M + row_i;
            const u32 acc = tmem + ((u32)(q * 32) << 16) + (u32)(acc_slot(k) * 128);
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
                        if (CKKS_SPAN(ob + rec.w + (u32)nc, 1, CKKS_DBG_TC_OUT))
                            ob[rec.w + (u32)nc] = shoup_mul(s2, 65536u, rec.z, rec.x) + csub(s1, rec.y);
                    }
                }
            }
            tc_fence_before();
            tc_arrive(&acc_empty[acc_slot(k)]);
        }
    } else if (lane == 0) {
        // ---- MMA issuer
        const u32 idesc = tc_idesc(TC_M, N);
        const u32 b_base = tc_smem_u32(Bs);
        int issued = 0;
        for (int k = 0; k < tiles; k++) {
            if (!wait_or_abort(&a_full[k % TC_STAGES], (u32)((k / TC_STAGES) & 1))) break;
            if (k >= nacc && !wait_or_abort(&acc_empty[acc_slot(k)], acc_phase(k - nacc))) break;
            tc_fence_after();
            const u32 a_base = tc_smem_u32(a_stage(k));
            const u32 d = tmem + (u32)(acc_slot(k) * 128);
#pragma unroll
            for (int s = 0; s < 2; s++)
                tc_mma(d, tc_smem_desc(a_base + (u32)(2 * s * TC_M * 16), TC_M * 16, 128),
                       tc_smem_desc(b_base + (u32)(2 * s * N * 16), (u32)N * 16, 128), idesc, (u32)s);
            tc_commit(&acc_full[acc_slot(k)]);
            tc_commit(&a_empty[k % TC_STAGES]);
            issued = k + 1;
        }
        if (abort_flag) {
            // the MMAs of the last nacc issued tiles may still run: wait for them (bounded)
            for (int t = issued - nacc; t < issued; t++)
                if (t >= 0) (void)tc_wait_bounded(&acc_full[acc_slot(t)], acc_phase(t));
        }
    }
    __syncthreads();
    if (warp == 8) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TC_COLS) : "memory");
    }
}
