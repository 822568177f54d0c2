// arith.cuh -- ciphertext-constant and ciphertext-ciphertext additions and constant products, the
// elementwise steps of polynomial evaluation on ciphertexts (EvalMod).
#pragma once
#include "ntt.cuh"

// Ciphertext-constant arithmetic over [n_comp][l+1] rows (row r has the prime of limb r mod (l+1)):
//   k_mul_const: out = in * [c]_q (every component); k_add_const: out = in + [c]_q on component 0
//   of every ciphertext ([n][2][l+1] rows: the even components), the odd components copied;
//   k_add: out = x + y.  cw: per limb (w, Shoup companion) of [c]_q_i.
struct ConstRns {
    tw_t w[64];
};

__global__ void k_mul_const(const u32 *in, u32 *out, ConstRns cw, const PrimeInfo *pinfo, int log_n, int level) {
    const int n = 1 << log_n;
    const int c4 = blockIdx.x * blockDim.x + threadIdx.x;
    if (4 * c4 >= n) return;
    const int r = blockIdx.y, i = r % (level + 1);
    if (!CKKS_SPAN(pinfo + i, 1, CKKS_DBG_CONST) || !CKKS_SPAN(in + (size_t)r * n + 4 * c4, 4, CKKS_DBG_CONST) ||
        !CKKS_SPAN(out + (size_t)r * n + 4 * c4, 4, CKKS_DBG_CONST))
        return;
    const u32 q = pinfo[i].q;
    const tw_t w = cw.w[i];
    const uint4 v = reinterpret_cast<const uint4 *>(in + (size_t)r * n)[c4];
    reinterpret_cast<uint4 *>(out + (size_t)r * n)[c4] =
        make_uint4(csub(shoup_mul(v.x, w.x, w.y, q), q), csub(shoup_mul(v.y, w.x, w.y, q), q),
                   csub(shoup_mul(v.z, w.x, w.y, q), q), csub(shoup_mul(v.w, w.x, w.y, q), q));
}

__global__ void k_add_const(const u32 *in, u32 *out, ConstRns cw, const PrimeInfo *pinfo, int log_n, int level) {
    const int n = 1 << log_n;
    const int c4 = blockIdx.x * blockDim.x + threadIdx.x;
    if (4 * c4 >= n) return;
    const int r = blockIdx.y, i = r % (level + 1);
    if (!CKKS_SPAN(pinfo + i, 1, CKKS_DBG_CONST) || !CKKS_SPAN(in + (size_t)r * n + 4 * c4, 4, CKKS_DBG_CONST) ||
        !CKKS_SPAN(out + (size_t)r * n + 4 * c4, 4, CKKS_DBG_CONST))
        return;
    const u32 q = pinfo[i].q;
    const u32 c = ((r / (level + 1)) & 1) == 0 ? cw.w[i].x : 0u;   // component 0 of each ciphertext
    const uint4 v = reinterpret_cast<const uint4 *>(in + (size_t)r * n)[c4];
    reinterpret_cast<uint4 *>(out + (size_t)r * n)[c4] =
        make_uint4(csub(v.x + c, q), csub(v.y + c, q), csub(v.z + c, q), csub(v.w + c, q));
}

__global__ void k_add(const u32 *x, const u32 *y, u32 *out, const PrimeInfo *pinfo, int log_n, int level) {
    const int n = 1 << log_n;
    const int c4 = blockIdx.x * blockDim.x + threadIdx.x;
    if (4 * c4 >= n) return;
    const int r = blockIdx.y, i = r % (level + 1);
    if (!CKKS_SPAN(pinfo + i, 1, CKKS_DBG_CONST) || !CKKS_SPAN(x + (size_t)r * n + 4 * c4, 4, CKKS_DBG_CONST) ||
        !CKKS_SPAN(y + (size_t)r * n + 4 * c4, 4, CKKS_DBG_CONST) ||
        !CKKS_SPAN(out + (size_t)r * n + 4 * c4, 4, CKKS_DBG_CONST))
        return;
    const u32 q = pinfo[i].q;
    const uint4 a = reinterpret_cast<const uint4 *>(x + (size_t)r * n)[c4];
    const uint4 b = reinterpret_cast<const uint4 *>(y + (size_t)r * n)[c4];
    reinterpret_cast<uint4 *>(out + (size_t)r * n)[c4] =
        make_uint4(csub(a.x + b.x, q), csub(a.y + b.y, q), csub(a.z + b.z, q), csub(a.w + b.w, q));
}
