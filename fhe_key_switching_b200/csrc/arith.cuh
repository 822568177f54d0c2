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

// Products with the monomial X^(N/2), which multiplies every slot by i.  In the evaluation domain
// X^(N/2) takes, at the root psi^(2 brv(k) + 1) of storage index k, the value
// psi^((2 brv(k) + 1) N/2) = w (-1)^brv(k) with w = psi^(N/2) (w^2 = -1); brv(k) is odd exactly
// when k >= N/2.  So the product is a multiplication by w on the first half of every limb and by
// -w on the second.  Rows are [n_comp][l+1] as in the kernels above; w4: (w, Shoup companion)
// per limb.
//   mode 0 (split):         out0 = x + y,   out1 = X^(N/2) (y - x)
//   mode 1 (recombination): out0 = x + X^(N/2) y
//   mode 2 (product):       out0 = X^(N/2) x
enum { MONO_SPLIT = 0, MONO_MERGE = 1, MONO_MUL = 2 };

__global__ void k_monomial_half(const u32 *x, const u32 *y, u32 *out0, u32 *out1, ConstRns w4,
                                const PrimeInfo *pinfo, int log_n, int level, int mode) {
    const int n = 1 << log_n;
    const int c4 = blockIdx.x * blockDim.x + threadIdx.x;
    if (4 * c4 >= n) return;
    const int r = blockIdx.y, i = r % (level + 1);
    const size_t off = (size_t)r * n + 4 * c4;
    if (!CKKS_SPAN(pinfo + i, 1, CKKS_DBG_CONST) || !CKKS_SPAN(x + off, 4, CKKS_DBG_CONST) ||
        !CKKS_SPAN(out0 + off, 4, CKKS_DBG_CONST) ||
        (mode != MONO_MUL && !CKKS_SPAN(y + off, 4, CKKS_DBG_CONST)) ||
        (mode == MONO_SPLIT && !CKKS_SPAN(out1 + off, 4, CKKS_DBG_CONST)))
        return;
    const u32 q = pinfo[i].q;
    const tw_t w = w4.w[i];
    const bool upper = 4 * c4 >= (n >> 1);
    // v * X^(N/2) at these four slots, v < 2q: canonical
    auto mono = [&](u32 v) {
        const u32 t = csub(shoup_mul(v, w.x, w.y, q), q);
        return upper && t != 0u ? q - t : t;
    };
    const uint4 a = *reinterpret_cast<const uint4 *>(x + off);
    if (mode == MONO_MUL) {
        *reinterpret_cast<uint4 *>(out0 + off) = make_uint4(mono(a.x), mono(a.y), mono(a.z), mono(a.w));
        return;
    }
    const uint4 b = *reinterpret_cast<const uint4 *>(y + off);
    if (mode == MONO_SPLIT) {
        *reinterpret_cast<uint4 *>(out0 + off) =
            make_uint4(csub(a.x + b.x, q), csub(a.y + b.y, q), csub(a.z + b.z, q), csub(a.w + b.w, q));
        *reinterpret_cast<uint4 *>(out1 + off) =
            make_uint4(mono(b.x + q - a.x), mono(b.y + q - a.y), mono(b.z + q - a.z), mono(b.w + q - a.w));
    } else {
        *reinterpret_cast<uint4 *>(out0 + off) = make_uint4(csub(a.x + mono(b.x), q), csub(a.y + mono(b.y), q),
                                                            csub(a.z + mono(b.z), q), csub(a.w + mono(b.w), q));
    }
}
