// ip_row_ws.cuh -- the key inner product fused with ModUp's last forward NTT pass (as k_ip_row),
// with the ChaCha12 keystream and the rest on different warps.
//
// On B200 the keystream's xors and rotations can only issue on the ALU pipe (64 per SM per clock),
// while the row pass and the Montgomery products are mostly multiply-adds on the FMA pipe.  In
// k_ip_row every warp runs both, one after the other, so the two pipes take turns.  Here a block
// of 512 threads splits them: warps 8-15 (producers) regenerate the a half of every active digit
// for the block's 16 rows x 256 slots into shared memory, laid out [digit][16][256 threads] as in
// k_ip_row's shared-key groups, and signal each digit on an mbarrier; warps 0-7 (consumers), with
// k_ip_row's row mapping, complete the extended digits (row pass, rotation permutation), load the
// b half, wait (bounded) for the digit's keystream and accumulate.  Items of a launch that share a
// key share the producers' keystream, as in k_ip_row.  Used when every item regenerates its a half
// and at most IP_GROUP_MAX_BETA digits are active; the results are k_ip_row's bit for bit.
// Included by ks_kernels.cuh after k_ip_row and the mbarrier helpers.
#pragma once

constexpr int IPW_THREADS = 2 * ROW_THREADS;

__global__ void __launch_bounds__(IPW_THREADS, 1)
k_ip_row_ws(IpRowArgs a) {
    __shared__ u32 sm[16 * 272];
    __shared__ __align__(8) u64 full[IP_GROUP_MAX_BETA];
    extern __shared__ u32 sa[];                      // regenerated a half: [digit][16][ROW_THREADS]
    const int tid = threadIdx.x;
    const int p = tid & (ROW_THREADS - 1);           // slot owner: the same mapping in both roles
    const int n = 1 << a.log_n;
    const int na = a.level + 1;
    const int u = blockIdx.y;
    const int g0 = a.grp_first[blockIdx.z], gcnt = a.grp_count[blockIdx.z];
    const int t = u < na ? u : a.n_q + (u - na);
    const PrimeInfo pi = a.pinfo[t];
    const u32 q = pi.q, two_q = 2 * q;
    const int r = p >> 4, lo = p & 15;
    const int row = blockIdx.x * 16 + r;
    const int k0 = row * 256 + 16 * lo;              // first evaluation slot of this thread
    if (tid == 0) {
        for (int j = 0; j < a.beta; j++) mbar_init(&full[j], ROW_THREADS);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (tid >= ROW_THREADS) {
        // ---- producers: the group's keystream, one digit at a time
        const int item = a.grp_item[g0];
        for (int j = 0; j < a.beta; j++) {
            u32 h[8];
            u32 *dst = sa + (size_t)j * 16 * ROW_THREADS + p;
            chacha_coeffs<false>(a.key[item], a.key_id[item], (u32)j, (u32)t, (u32)(k0 >> 3), pi, h);
#pragma unroll
            for (int v = 0; v < 8; v++) dst[v * ROW_THREADS] = h[v];
            chacha_coeffs<false>(a.key[item], a.key_id[item], (u32)j, (u32)t, (u32)(k0 >> 3) + 1u, pi, h);
#pragma unroll
            for (int v = 0; v < 8; v++) dst[(8 + v) * ROW_THREADS] = h[v];
            asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(&full[j])) : "memory");
        }
        return;
    }
    // ---- consumers
    const u32 R1 = (u32)(n >> 8);
    u32 *srow = sm + r * 272;
    const tw_t *twf = a.twf + (size_t)t * n;
    u32 ready = 0;                                   // digits whose keystream has been waited for
    for (int it = 0; it < gcnt; it++) {
        const int item = a.grp_item[g0 + it];
        const u32 *xb = a.x + item * a.x_item;
        const u32 *cdb = a.cdig + item * a.cdig_item;
        u32 *accb = a.acc + item * a.acc_item;
        const u32 *bkey = a.b[item];
        const u32 hoist_g = a.hoist_g[item], cdig_g = a.cdig_g[item];
        // hoisted rotation: source row of this row under kappa_g
        const int src_row = hoist_g ? (int)(automorph_src((u32)(row * 256), hoist_g, a.log_n) >> 8) : row;
        u32 acc0[16], acc1[16];
#pragma unroll
        for (int v = 0; v < 16; v++) acc0[v] = acc1[v] = 0;
        for (int j = 0; j < a.beta; j++) {
            const bool in_digit = u < na && u >= j * a.alpha && u < min(j * a.alpha + a.alpha, na);
            u32 x[16];
            if (in_digit) {
                const u32 *src = cdb + (size_t)u * n;
                const u32 g = hoist_g ? hoist_g : cdig_g;
                if (g) {
#pragma unroll
                    for (int v = 0; v < 16; v++) x[v] = src[automorph_src((u32)(k0 + v), g, a.log_n)];
                } else {
                    load16_vec(src + k0, x);
                }
            } else {
                const u32 *src = xb + ((size_t)j * a.ext + u) * n + (size_t)src_row * 256;
#pragma unroll
                for (int v = 0; v < 16; v++) x[v] = src[lo + 16 * v];
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
            if (!(ready & (1u << j))) {   // the digit's keystream: wait once (bounded)
                if (!mbar_wait_bounded(&full[j], 0u)) atomicOr(a.err, CKKS_DEV_ERR_WAIT);
                ready |= 1u << j;
            }
            u32 bv[16], av[16];
            load16_vec(bkey + ((size_t)j * a.n_primes + t) * n + k0, bv);
            const u32 *src = sa + (size_t)j * 16 * ROW_THREADS + p;
#pragma unroll
            for (int v = 0; v < 16; v++) av[v] = src[v * ROW_THREADS];
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
        store16_vec(accb + (size_t)u * n + (size_t)row * 256 + 16 * lo, acc0);
        store16_vec(accb + ((size_t)a.ext + u) * n + (size_t)row * 256 + 16 * lo, acc1);
    }
}
