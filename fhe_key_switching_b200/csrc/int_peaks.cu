// int_peaks.cu -- integer throughput probes: the measured denominators of the integer-ALU
// roofline that the benchmark reports (a measurement aid; the pages have no counterpart).
//
// Every probe kernel runs 8 independent dependency chains per thread, 256 threads per block,
// and counts the operations of its chains (one PTX instruction each, except the ChaCha12
// probe, which counts the op model's 608 int32 operations per block).  The chains mix two or
// three registers non-linearly so that no step can be folded into its neighbour.  The
// elapsed time of one launch (CUDA events on the launching stream) gives operations per
// second; divided by SMs x SM clock it gives operations per SM per clock, the per-pipe rate.
#include <cuda_runtime.h>

#include <cstdio>

#include "../../include/ckks_ks.h"
#include "chacha.cuh"

namespace {

constexpr int PROBE_THREADS = 256;
constexpr int PROBE_CHAINS = 8;
constexpr int PROBE_UNROLL = 4;

__device__ __forceinline__ u32 op_add(u32 a, u32 b) {
    u32 d;
    asm("add.u32 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
template <int LUT>
__device__ __forceinline__ u32 op_lop3(u32 a, u32 b, u32 c) {
    u32 d;
    asm("lop3.b32 %0, %1, %2, %3, %4;" : "=r"(d) : "r"(a), "r"(b), "r"(c), "n"(LUT));
    return d;
}
template <int S>
__device__ __forceinline__ u32 op_shf(u32 lo, u32 hi) {
    u32 d;
    asm("shf.l.wrap.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(lo), "r"(hi), "n"(S));
    return d;
}
__device__ __forceinline__ u32 op_mad(u32 a, u32 b, u32 c) {
    u32 d;
    asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ u32 op_madhi(u32 a, u32 b, u32 c) {
    u32 d;
    asm("mad.hi.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ u64 op_madwide(u32 a, u32 b, u64 c) {
    u64 d;
    asm("mad.wide.u32 %0, %1, %2, %3;" : "=l"(d) : "r"(a), "r"(b), "l"(c));
    return d;
}

// Operations per chain step (ChaCha12: per block, the op model's count).
__host__ __device__ constexpr int probe_ops_per_step(int op) {
    return op == CKKS_PROBE_IMAD_WIDE ? 1 : op == CKKS_PROBE_CHACHA12 ? 608 : 2;
}

template <int OP>
__global__ void __launch_bounds__(PROBE_THREADS) k_int_probe(u32 *sink, int iters, u32 seed) {
    const u32 tid = blockIdx.x * PROBE_THREADS + threadIdx.x;
    u32 a[PROBE_CHAINS], b[PROBE_CHAINS], c[PROBE_CHAINS];
    u64 w[PROBE_CHAINS];
#pragma unroll
    for (int k = 0; k < PROBE_CHAINS; k++) {
        a[k] = tid * 0x9E3779B9u + seed + 17u * k;
        b[k] = (tid ^ 0x85EBCA6Bu) + 31u * k + 1u;
        c[k] = seed * 0xC2B2AE35u + 101u * k + 3u;
        w[k] = ((u64)b[k] << 32) | a[k];
    }
    if (OP == CKKS_PROBE_CHACHA12) {
        ChachaKey key;
#pragma unroll
        for (int i = 0; i < 8; i++) key.k[i] = seed * (2u * i + 1u) + tid;
        u32 acc = 0;
        for (int it = 0; it < iters; it++) {
            u32 o[16];
            chacha12_block(key, (u32)it, tid, seed, 7u, o);
#pragma unroll
            for (int i = 0; i < 16; i++) acc ^= o[i];
        }
        sink[tid] = acc;
    } else {
        for (int it = 0; it < iters; it++) {
#pragma unroll
            for (int r = 0; r < PROBE_UNROLL; r++) {
#pragma unroll
                for (int k = 0; k < PROBE_CHAINS; k++) {
                    if (OP == CKKS_PROBE_IADD) {
                        a[k] = op_add(a[k], b[k]);
                        b[k] = op_add(b[k], a[k]);
                    } else if (OP == CKKS_PROBE_LOP3) {
                        a[k] = op_lop3<0x96>(a[k], b[k], c[k]);     // a ^ b ^ c
                        b[k] = op_lop3<0xE8>(b[k], c[k], a[k]);     // majority(b, c, a)
                    } else if (OP == CKKS_PROBE_SHF) {
                        a[k] = op_shf<7>(a[k], b[k]);
                        b[k] = op_shf<13>(b[k], a[k]);
                    } else if (OP == CKKS_PROBE_IMAD) {
                        a[k] = op_mad(a[k], b[k], c[k]);
                        b[k] = op_mad(b[k], a[k], c[k]);
                    } else if (OP == CKKS_PROBE_IMAD_HI) {
                        a[k] = op_madhi(a[k], b[k], c[k]);
                        b[k] = op_madhi(b[k], a[k], c[k]);
                    } else if (OP == CKKS_PROBE_IMAD_WIDE) {
                        w[k] = op_madwide((u32)w[k], c[k], w[k]);
                    } else if (OP == CKKS_PROBE_MIX) {              // one logic op and one multiply-add
                        a[k] = op_lop3<0x96>(a[k], b[k], c[k]);
                        b[k] = op_mad(b[k], a[k], c[k]);
                    }
                }
            }
        }
        u32 s = 0;
#pragma unroll
        for (int k = 0; k < PROBE_CHAINS; k++) s ^= a[k] ^ b[k] ^ (u32)w[k] ^ (u32)(w[k] >> 32);
        sink[tid] = s;
    }
}

}  // namespace

extern "C" int ckks_int_probe(int op, int blocks, int iters, uint32_t *sink, ckks_stream_t stream, float *ms,
                              double *ops) {
    if (!sink || !ms || !ops || blocks < 1 || iters < 1 || op < 0 || op >= CKKS_PROBE_COUNT) return CKKS_ERR_ARG;
    if (((uintptr_t)sink & 15u) != 0) return CKKS_ERR_ALIGN;
    cudaEvent_t e0 = nullptr, e1 = nullptr;
    if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) {
        if (e0) cudaEventDestroy(e0);
        return CKKS_ERR_CUDA;
    }
    const u32 seed = 0x1234567u + (u32)op;
    cudaEventRecord(e0, stream);
    switch (op) {
#define CKKS_PROBE_CASE(OP) \
    case OP: k_int_probe<OP><<<blocks, PROBE_THREADS, 0, stream>>>(sink, iters, seed); break;
        CKKS_PROBE_CASE(CKKS_PROBE_IADD) CKKS_PROBE_CASE(CKKS_PROBE_LOP3) CKKS_PROBE_CASE(CKKS_PROBE_SHF)
        CKKS_PROBE_CASE(CKKS_PROBE_IMAD) CKKS_PROBE_CASE(CKKS_PROBE_IMAD_HI) CKKS_PROBE_CASE(CKKS_PROBE_IMAD_WIDE)
        CKKS_PROBE_CASE(CKKS_PROBE_MIX) CKKS_PROBE_CASE(CKKS_PROBE_CHACHA12)
#undef CKKS_PROBE_CASE
        default: break;
    }
    cudaEventRecord(e1, stream);
    int r = CKKS_OK;
    if (cudaGetLastError() != cudaSuccess || cudaEventSynchronize(e1) != cudaSuccess ||
        cudaEventElapsedTime(ms, e0, e1) != cudaSuccess)
        r = CKKS_ERR_CUDA;
    cudaEventDestroy(e0);
    cudaEventDestroy(e1);
    const double per_iter = op == CKKS_PROBE_CHACHA12 ? 1.0 : (double)PROBE_UNROLL * PROBE_CHAINS;
    *ops = (double)blocks * PROBE_THREADS * iters * per_iter * probe_ops_per_step(op);
    return r;
}
