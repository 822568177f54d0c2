/*
 * ckks_ks.h -- C ABI of the B200 (sm_100a) RNS-CKKS hybrid key-switching library.
 *
 * What the library computes.  The Perseus write-up ("Perseus: A Full-Stack System for
 * Homomorphic Model Inference", ai4snews, Interpretation, 2nd paragraph) describes a 32-bit
 * RNS CKKS runtime whose key-switching keys store only their b half: the uniformly random
 * a half is regenerated inside the two kernels that use the key by a counter-mode ChaCha12
 * expander, halving key storage.  Key switching is the core of every rotation and
 * relinearisation.  The pages give no formulas; the operations below follow full-RNS CKKS
 * and fast base conversion (Cheon, Han, Kim, Kim, Song, SAC 2018) and hybrid key switching
 * with dnum gadget digits (Han, Ki, CT-RSA 2020), with the conventions listed here.
 *
 * Conventions (every entry point):
 *  - N = 2^log_n, 12 <= log_n <= 16.  Primes are NTT friendly (q = 1 mod 2N) and below 2^30.
 *  - Chain: ciphertext primes q_0..q_{n_q-1}, special primes p_0..p_{n_p-1}; "global limb
 *    index" t = 0..n_q-1 for q_t and n_q + i for p_i.  `level` l means l+1 active ciphertext
 *    limbs q_0..q_l.  The extended basis at level l is q_0..q_l, p_0..p_{n_p-1}
 *    (ext = l + 1 + n_p limbs, in that order).
 *  - Gadget digits: alpha = ceil(n_q / dnum) primes per digit; digit j holds q_{j*alpha} ..
 *    q_{min((j+1)*alpha, l+1)-1}; beta = ceil((l+1)/alpha) digits are active at level l.
 *  - Polynomials are uint32 [limb][N] row-major, residues canonical in [0, q) on input and
 *    output.  Evaluation ("NTT") domain: storage index k holds a(psi^(2*brv(k)+1)) with
 *    psi the primitive 2N-th root chosen as h^((q-1)/2N) for the smallest h >= 2 with
 *    psi^N = -1, brv the log_n-bit reversal.  Ciphertexts are [2][l+1][N], the tensor
 *    product is [3][l+1][N]; all in the evaluation domain.
 *  - Device pointers must be 16-byte aligned.  Outputs must not alias inputs unless the
 *    entry point says so, and the workspace must not overlap either; the key-switching, rescale
 *    and baby-step giant-step entry points check this and return CKKS_ERR_ARG.  The caller owns
 *    every buffer and the stream.
 *  - A context belongs to the device that was current when it was created; every entry point
 *    that takes a context returns CKKS_ERR_ARG when another device is current.
 *  - Every call is asynchronous on `stream`; nothing synchronises the device, nothing
 *    allocates device memory except ckks_ctx_create.  The workspace `ws` is caller-owned
 *    device memory of at least ckks_workspace_bytes(...) bytes; calls on different streams
 *    need different workspaces.
 *  - Return codes: CKKS_OK (0) or a negative CKKS_ERR_*; ckks_last_error() gives a message
 *    (thread-local).  No C++ exception crosses this boundary.
 */
#ifndef CKKS_KS_H
#define CKKS_KS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same underlying type as cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st *ckks_stream_t;

enum {
    CKKS_OK = 0,
    CKKS_ERR_ARG = -1,          /* null pointer or bad argument */
    CKKS_ERR_UNSUPPORTED = -2,  /* log_n outside 12..16, prime >= 2^30 or not 1 mod 2N, level > L ... */
    CKKS_ERR_ALIGN = -3,        /* a device pointer is not 16-byte aligned */
    CKKS_ERR_WORKSPACE = -4,    /* workspace smaller than ckks_workspace_bytes() */
    CKKS_ERR_CUDA = -5,         /* a CUDA call or kernel launch failed */
    CKKS_ERR_TIMEOUT = -6,      /* ckks_sync_status: stream still busy at the deadline */
    CKKS_ERR_BOUNDS = -7        /* ckks_sync_status, debug-bounds build only: an index check failed */
};

typedef struct ckks_ctx ckks_ctx; /* opaque; owns read-only device tables only */

/* Parameter set.  q: n_q ciphertext primes, p: n_p special primes (host arrays, copied).
 * dnum: number of gadget digits the keys of this context are generated with. */
typedef struct {
    uint32_t log_n, n_q, n_p, dnum;
    const uint32_t *q, *p;
} ckks_params;

/* Key-switching key (from a secret s' to s), evaluation domain, full chain.
 *  b:  device, [D][n_q+n_p][N], D = ceil(n_q/alpha) digits:
 *      b_j[t] = -a_j[t]*s[t] + e_j[t] + [t in digit j]*[P]_{q_t}*s'[t]   (mod t).
 *  a:  NULL (default): the a half is regenerated in-kernel (see ckks_chacha_expand);
 *      non-NULL: device [D][n_q+n_p][N] stored a half (ablation that reads it from HBM).
 *  seed, key_id: the ChaCha12 key and the first nonce word; key_id is 0 for the
 *      relinearisation key and the Galois element g for the rotation key of kappa_g. */
typedef struct {
    const uint32_t *b;
    const uint32_t *a;
    uint8_t seed[32];
    uint32_t key_id;
} ckks_evk;

/* Prime chain rule: scan x = 1 (mod 2N) downward from the largest such x below 2^30, keep
 * primes in order; the first n_p found are the special primes p_0 > p_1 > ..., the next n_q
 * the ciphertext primes q_0 > q_1 > ...  Host only; q_out/p_out are host arrays. */
int ckks_gen_primes(uint32_t log_n, uint32_t n_q, uint32_t n_p, uint32_t *q_out, uint32_t *p_out);

/* Builds the device tables (twiddles, base-conversion constants) for a parameter set on the
 * current CUDA device.  Synchronous.  The context may then be used from any stream. */
int ckks_ctx_create(const ckks_params *params, ckks_ctx **ctx_out);
void ckks_ctx_destroy(ckks_ctx *ctx);

/* Forward / inverse negacyclic NTT, in place, on n_limbs consecutive rows of `poly`; row r
 * uses the prime of global limb first_limb + r.  Forward: coefficients -> evaluation domain
 * as defined above (A[k] = sum_n a[n] psi^((2 brv(k)+1) n)); inverse: its exact inverse
 * (including the N^-1 scale). */
int ckks_ntt_fwd(ckks_ctx *ctx, uint32_t *poly, int first_limb, int n_limbs, ckks_stream_t stream);
int ckks_ntt_inv(ckks_ctx *ctx, uint32_t *poly, int first_limb, int n_limbs, ckks_stream_t stream);

/* Automorphism kappa_g (g odd, 0 < g < 2N) in the evaluation domain on n_limbs rows:
 * out[k] = in[k'] with 2 brv(k')+1 = (2 brv(k)+1) g mod 2N.  out must not alias in. */
int ckks_automorph(ckks_ctx *ctx, const uint32_t *in, uint32_t *out, int n_limbs, uint32_t galois,
                   ckks_stream_t stream);

/* ModUp (hybrid key switching): c [l+1][N] -> dtilde [beta][ext][N].  For each active digit
 * j, digit limbs keep their evaluation values; every other extended limb t receives
 * NTT_t(FastBConv(iNTT(digit j's limbs))) with the centred lift
 * y_i = [x_i (D_j/q_i)^-1]_{q_i} in (-q_i/2, q_i/2], out_t = sum_i y_i [D_j/q_i]_t mod t. */
int ckks_modup(ckks_ctx *ctx, const uint32_t *c, int level, uint32_t *dtilde, void *ws,
               size_t ws_bytes, ckks_stream_t stream);

/* Key inner product (the kernel that uses the key): acc [2][ext][N],
 * acc0[u] = sum_j dtilde_j[u] * b_j[t], acc1[u] = sum_j dtilde_j[u] * a_j[t] (mod t), t the
 * global limb of extended position u; a_j[t] regenerated by ChaCha12 unless evk->a is set. */
int ckks_inner_product(ckks_ctx *ctx, const uint32_t *dtilde, int level, const ckks_evk *evk,
                       uint32_t *acc, ckks_stream_t stream);

/* ModDown: acc [ext][N] -> out [l+1][N]; iNTT of the special limbs, centred FastBConv
 * P -> q_i, NTT, out_i = (acc_i - conv_i) [P^-1]_{q_i}. */
int ckks_moddown(ckks_ctx *ctx, const uint32_t *acc, int level, uint32_t *out, void *ws,
                 size_t ws_bytes, ckks_stream_t stream);

/* Key switching of one polynomial c [l+1][N]: out [2][l+1][N] = (ModDown(acc0), ModDown(acc1)). */
int ckks_keyswitch(ckks_ctx *ctx, const uint32_t *c, int level, const ckks_evk *evk, uint32_t *out,
                   void *ws, size_t ws_bytes, ckks_stream_t stream);

/* Rotation by the Galois element g: kappa_g on both components, key switching of
 * kappa_g(c1) with the key for kappa_g(s), kappa_g(c0) added to the first output component.
 * ct, out: [2][l+1][N]. */
int ckks_rotate(ckks_ctx *ctx, const uint32_t *ct, int level, uint32_t galois, const ckks_evk *evk,
                uint32_t *out, void *ws, size_t ws_bytes, ckks_stream_t stream);

/* Hoisted rotations: one ModUp of c1, then for each r the extended digits permuted by
 * kappa_{g_r}, the inner product with keys[r], ModDown and kappa_{g_r}(c0) added.
 * galois, keys: host arrays of n_rot entries; out: [n_rot][2][l+1][N].  (With the centred
 * lift, ModUp commutes with kappa_g, so each output equals ckks_rotate bit for bit.) */
int ckks_rotate_hoisted(ckks_ctx *ctx, const uint32_t *ct, int level, int n_rot,
                        const uint32_t *galois, const ckks_evk *keys, uint32_t *out, void *ws,
                        size_t ws_bytes, ckks_stream_t stream);

/* Hoisted rotations of several ciphertexts by the same n_rot rotations: ct [n_ct][2][l+1][N],
 * out [n_ct][n_rot][2][l+1][N]; output (u, r) equals ckks_rotate_hoisted of ciphertext u, rotation
 * r, bit for bit (and so ckks_rotate).  One ModUp per ciphertext, then one inner product and
 * ModDown launch over up to 64 (ciphertext, rotation) pairs, in which the pairs that use the same
 * key regenerate its a half once per group of up to 8 (the a half is regenerated inside the kernel
 * that uses the key: ai4snews write-up of Perseus, Interpretation, 2nd paragraph; hoisting several
 * rotations over one ModUp is Halevi and Shoup's).  1 <= n_rot <= 64; the workspace is
 * ckks_workspace_bytes(ctx, level, min(n_ct, 64 / n_rot) * n_rot).  Errors as for
 * ckks_rotate_hoisted, and CKKS_ERR_ARG for n_ct < 0, n_rot outside 0..64 and overlaps between
 * the input, the output and the workspace; n_ct = 0 or n_rot = 0 does nothing. */
int ckks_rotate_hoisted_batch(ckks_ctx *ctx, int n_ct, const uint32_t *ct, int level, int n_rot,
                              const uint32_t *galois, const ckks_evk *keys, uint32_t *out, void *ws,
                              size_t ws_bytes, ckks_stream_t stream);

/* Relinearisation: d [3][l+1][N] (decrypting under 1, s, s^2) -> out [2][l+1][N] =
 * (d0, d1) + keyswitch(d2) with the key for s^2. */
int ckks_relin(ckks_ctx *ctx, const uint32_t *d, int level, const ckks_evk *evk, uint32_t *out,
               void *ws, size_t ws_bytes, ckks_stream_t stream);

/* Tensor product of x = (x0, x1), y = (y0, y1) [2][l+1][N]: d [3][l+1][N] =
 * (x0 y0, x0 y1 + x1 y0, x1 y1) pointwise mod q_i. */
int ckks_tensor(ckks_ctx *ctx, const uint32_t *x, const uint32_t *y, int level, uint32_t *d,
                ckks_stream_t stream);

/* Batches of independent operations at one level, executed by the same kernels as one launch
 * per step (each launch covers all items, up to 64 at a time), which fills the GPU far better
 * than one operation at a time.  Item z's operands are contiguous: c [n][l+1][N],
 * ct/out [n][2][l+1][N], d [n][3][l+1][N], x, y [n][2][l+1][N]; keys and galois are host arrays
 * of n entries (items may share a key).  Each item's result equals the corresponding single
 * call bit for bit.  Workspace: ckks_workspace_bytes(ctx, level, n). */
int ckks_keyswitch_batch(ckks_ctx *ctx, int n, const uint32_t *c, int level, const ckks_evk *keys,
                         uint32_t *out, void *ws, size_t ws_bytes, ckks_stream_t stream);
int ckks_rotate_batch(ckks_ctx *ctx, int n, const uint32_t *ct, int level, const uint32_t *galois,
                      const ckks_evk *keys, uint32_t *out, void *ws, size_t ws_bytes, ckks_stream_t stream);
int ckks_relin_batch(ckks_ctx *ctx, int n, const uint32_t *d, int level, const ckks_evk *keys, uint32_t *out,
                     void *ws, size_t ws_bytes, ckks_stream_t stream);
int ckks_tensor_batch(ckks_ctx *ctx, int n, const uint32_t *x, const uint32_t *y, int level, uint32_t *d,
                      ckks_stream_t stream);

/* Rescale by the last active prime q_l (the RNS rescale of full-RNS CKKS, Cheon, Han, Kim,
 * Kim, Song, SAC 2018; the Perseus pages name no rescale of their own, and it follows the
 * tensor product and relinearisation of a multiplication):
 *   ct [2][l+1][N] at level l -> out [2][l][N] at level l-1, evaluation domain, canonical;
 *   per component with integer polynomial C over q_0..q_l, out = (C - [C]_{q_l}) / q_l mod
 *   q_0..q_{l-1}, with the centred residue [C]_{q_l} in (-q_l/2, q_l/2] (rounding to nearest);
 *   limb by limb: out_i = (c_i - NTT_i(lift(iNTT_l(c_l)))) [q_l^-1]_{q_i}.
 * The plaintext scale is divided by q_l.  level >= 1.  Batched: ct [n][2][l+1][N],
 * out [n][2][l][N].  Workspace: ckks_workspace_bytes(ctx, level, n).  out must not overlap ct
 * (CKKS_ERR_ARG).  Errors as for the other calls: CKKS_ERR_ARG for a null pointer, n < 0 or
 * level < 1; CKKS_ERR_UNSUPPORTED for a level above the chain; CKKS_ERR_ALIGN for pointers not
 * 16-byte aligned; CKKS_ERR_WORKSPACE for a short workspace. */
int ckks_rescale(ckks_ctx *ctx, const uint32_t *ct, int level, uint32_t *out, void *ws, size_t ws_bytes,
                 ckks_stream_t stream);
int ckks_rescale_batch(ckks_ctx *ctx, int n, const uint32_t *ct, int level, uint32_t *out, void *ws,
                       size_t ws_bytes, ckks_stream_t stream);

/* Baby-step giant-step linear transform with double hoisting (Bossuat, Mouchet,
 * Troncoso-Pastoriza, Hubaux, "Efficient Bootstrapping for Approximate Homomorphic Encryption
 * with Non-Sparse Keys", Eurocrypt 2021, Sec. 6; the split into baby and giant steps is Halevi
 * and Shoup's).  The Perseus pages do not describe it; it is the linear-transform step that the
 * hoisted rotation keys of a CoeffToSlot level serve.
 *   out = sum_j rot_{G_j}( sum_k pt[j][k] * rot_{B_k}(ct) )
 * computed as: one ModUp of c1; for every baby k with B_k != 1 the hoisted inner product with
 * kappa_{B_k} applied to the extended digits, kept in the extended basis PQ as
 * X_k = (acc0_k + P kappa_{B_k}(c0), acc1_k) (X_k = (P c0, P c1) for B_k = 1); for every giant j
 * the sum V_j = sum_k pt[j][k] X_k in PQ and one ModDown of it; then each partial rotated by
 * ckks_rotate's path (none for G_j = 1) and the partials added.
 *   ct, out: [2][l+1][N] (device, evaluation domain; out must not overlap ct);
 *   baby_galois[n_baby], giant_galois[n_giant]: host arrays of odd elements in (0, 2N), 1 meaning
 *     no rotation; baby_keys, giant_keys: host arrays of the same lengths (entries for element 1
 *     are not read);
 *   pt: [n_giant][n_baby][ext][N] (device) canonical evaluation-domain plaintexts over the
 *     extended basis q_0..q_l, p_0..p_{k-1}, ext = l+1+k (the caller pre-rotates the diagonal of
 *     index (j, k) by -G_j in the slots, as usual for baby-step giant-step);
 *   1 <= n_baby, n_giant <= 64; workspace: ckks_bsgs_workspace_bytes(ctx, level, n_baby, n_giant)
 *     (0 for arguments out of range).
 * Errors: CKKS_ERR_ARG (null pointer, counts out of range, even Galois element, overlap),
 * CKKS_ERR_UNSUPPORTED (level), CKKS_ERR_ALIGN, CKKS_ERR_WORKSPACE. */
size_t ckks_bsgs_workspace_bytes(ckks_ctx *ctx, int level, int n_baby, int n_giant);
int ckks_bsgs(ckks_ctx *ctx, const uint32_t *ct, int level, int n_baby, const uint32_t *baby_galois,
              const ckks_evk *baby_keys, int n_giant, const uint32_t *giant_galois, const ckks_evk *giant_keys,
              const uint32_t *pt, uint32_t *out, void *ws, size_t ws_bytes, ckks_stream_t stream);

/* CKKS encoding of N/2 complex slots into a plaintext (the pages give no encoder; this is the
 * canonical embedding of full-RNS CKKS): m is the real integer polynomial with
 * m(zeta^(5^j)) ~ scale * z_j, zeta = exp(i pi / N), j < N/2, computed on the host in double
 * precision by the inverse of the slot DFT (radix-2 stages, then bit reversal) and rounded half
 * away from zero; then reduced into q_0..q_level (and p_0..p_(k-1) when with_special != 0, the
 * extended basis that ckks_bsgs's plaintexts use) and transformed to the evaluation domain on the
 * GPU.  re, im: host arrays of N/2 doubles (the call copies them before returning);
 * out: device [(level+1) (+ n_p)][N], canonical; ws: device, >= 8 N bytes (the coefficients);
 * scale > 0.  The caller keeps |scale * t| well below 2^62 and below half the basis' modulus.
 * Integer coefficients are decided in double precision, so another correct encoder may differ by
 * one in a rare coefficient whose scaled value lies within rounding error of a half-integer.
 * Errors: CKKS_ERR_ARG (null, scale, overlap), CKKS_ERR_UNSUPPORTED (level), CKKS_ERR_ALIGN,
 * CKKS_ERR_WORKSPACE, CKKS_ERR_CUDA. */
int ckks_encode(ckks_ctx *ctx, const double *re, const double *im, double scale, int level, int with_special,
                uint32_t *out, void *ws, size_t ws_bytes, ckks_stream_t stream);

/* ModRaise, the first step of CKKS bootstrapping (Cheon, Han, Kim, Kim, Song, Eurocrypt 2018;
 * the pages give no construction): a ciphertext at level 0, ct [2][1][N] (evaluation domain mod
 * q_0), is read as integer polynomials with centred coefficients in (-q_0/2, q_0/2] and reduced
 * into q_0..q_level: out [2][level+1][N], evaluation domain, canonical.  Per component: inverse
 * NTT mod q_0, centred lift, NTT in every limb.  It decrypts to m + q_0 I with a small integer
 * polynomial I, which the bootstrapping's modular reduction then removes.
 * Workspace: 2 N words (ws_bytes >= 8 N).  out must not overlap ct, and ws neither
 * (CKKS_ERR_ARG); other errors as for the key-switching calls. */
int ckks_modraise(ckks_ctx *ctx, const uint32_t *ct, int level, uint32_t *out, void *ws, size_t ws_bytes,
                  ckks_stream_t stream);

/* Ciphertext arithmetic for polynomial evaluation (EvalMod).  All in the evaluation domain over
 * q_0..q_level, canonical; out may equal the input (elementwise).
 *  ckks_mul_const: every component of ct [n_comp][l+1][N] times the integer v (reduced mod q_i;
 *    the plaintext scale is unchanged, the slots are multiplied by v);
 *  ckks_add_const: ct [2][l+1][N] plus the constant polynomial v on component 0 (the slots gain
 *    v / scale);
 *  ckks_add: x + y, both [n_comp][l+1][N].
 * n_comp in 1..3; errors as for the other calls. */
int ckks_mul_const(ckks_ctx *ctx, const uint32_t *ct, int n_comp, int level, long long v, uint32_t *out,
                   ckks_stream_t stream);
int ckks_add_const(ckks_ctx *ctx, const uint32_t *ct, int level, long long v, uint32_t *out, ckks_stream_t stream);
int ckks_add(ckks_ctx *ctx, const uint32_t *x, const uint32_t *y, int n_comp, int level, uint32_t *out,
             ckks_stream_t stream);

/* EvalMod, the modular reduction of CKKS bootstrapping (Cheon, Han, Kim, Kim, Song, Eurocrypt
 * 2018; the pages give no construction): for a ciphertext whose slots hold real x with
 * |x| small, out's slots approximate sin(2 pi x) / (2 pi), which equals x - round(x) near the
 * integers.  Fixed sequence (every constant an integer by std::llround, half away from zero, of
 * an IEEE double product; the nominal scale S tracked in double):
 *   theta = (2 pi / 2^r)(x - 1/4): ct * llround(c1 q_l), rescale, + llround(-(c1/4) S);
 *   u = theta^2 (tensor, relinearisation, rescale; S_u = S^2 / q_l);
 *   cos(theta) = sum_{k<=d} (-1)^k u^k / (2k)! by Horner: p = u * llround(a_d q_l), rescale,
 *     + llround(a_(d-1) S_u), then d - 1 times p = p * u (u dropped to p's level), + llround(a_k S_p);
 *   r double angles: p = 2 p^2 - 1 (square, relinearisation, rescale, * 2, + llround(-S_p));
 *   out = p * llround(q_l / (2 pi)), rescale.
 * It consumes d + r + 3 levels: *out_level = level - d - r - 3, *out_scale = the tracked scale of
 * out.  ct: [2][level+1][N]; out: room for 2 (level+1) N words, of which the first
 * 2 (*out_level+1) N hold the result as [2][*out_level+1][N]; relin_key: the key for s^2
 * (key_id 0); ws: ckks_evalmod_workspace_bytes(ctx, level)
 * bytes.  r in 0..16, d in 1..16.  Errors: CKKS_ERR_ARG (null, ranges, scale, overlap),
 * CKKS_ERR_UNSUPPORTED (level below d + r + 3 or above the chain), CKKS_ERR_ALIGN,
 * CKKS_ERR_WORKSPACE. */
size_t ckks_evalmod_workspace_bytes(const ckks_ctx *ctx, int level);
int ckks_evalmod(ckks_ctx *ctx, const uint32_t *ct, int level, double scale, int r, int d, const ckks_evk *relin_key,
                 uint32_t *out, int *out_level, double *out_scale, void *ws, size_t ws_bytes, ckks_stream_t stream);

/* The same EvalMod on n ciphertexts at one level and scale (1 <= n <= 64; bootstrapping applies it
 * to the real and the imaginary halves): ct [n][2][level+1][N]; out: room for n 2 (level+1) N
 * words, of which the first n 2 (*out_level+1) N hold the results as [n][2][*out_level+1][N];
 * ws: ckks_evalmod_batch_workspace_bytes(ctx, level, n) bytes (0 for n or level out of range).
 * Every step runs once for the whole batch (the batched tensor, relinearisation and rescale
 * calls; the items' relinearisations share the one key's regenerated a half).  Each item's
 * result equals ckks_evalmod on that item alone, bit for bit.  Errors as ckks_evalmod, and
 * CKKS_ERR_ARG for n out of range. */
size_t ckks_evalmod_batch_workspace_bytes(const ckks_ctx *ctx, int level, int n);
int ckks_evalmod_batch(ckks_ctx *ctx, int n, const uint32_t *ct, int level, double scale, int r, int d,
                       const ckks_evk *relin_key, uint32_t *out, int *out_level, double *out_scale, void *ws,
                       size_t ws_bytes, ckks_stream_t stream);

/* Product with the monomial X^(N/2): every slot is multiplied by i, since each slot root
 * zeta^(5^j) raised to N/2 is i (5^j = 1 mod 4).  Bootstrapping uses it to take the imaginary half of
 * CoeffToSlot's output and to put it back (Cheon, Han, Kim, Kim, Song, Eurocrypt 2018; the pages give
 * no construction).  In the evaluation domain it is a multiplication by w = psi^(N/2) on the first
 * N/2 entries of every limb and by -w on the rest.  ct, out: [n_comp][level+1][N] (out may equal
 * ct), n_comp in 1..3; errors as for ckks_add, and CKKS_ERR_ALIGN. */
int ckks_mul_i(ckks_ctx *ctx, const uint32_t *ct, int n_comp, int level, uint32_t *out, ckks_stream_t stream);

/* One level of a slot DFT for ckks_bootstrap: the arguments of one ckks_bsgs call (host arrays of
 * n_baby and n_giant entries; pt on the device, [n_giant][n_baby][l+1+k][N] at the level the
 * transform runs at, encoded at scale q_l so that the rescale after it keeps the scale). */
typedef struct {
    int n_baby;
    const uint32_t *baby_galois;
    const ckks_evk *baby_keys;
    int n_giant;
    const uint32_t *giant_galois;
    const ckks_evk *giant_keys;
    const uint32_t *pt;
} ckks_bsgs_level;

/* What ckks_bootstrap runs: ModRaise to top_level; n_c2s CoeffToSlot levels at top_level,
 * top_level - 1, ...; EvalMod of degree 2 d with r double angles (d + r + 3 levels); n_s2c
 * SlotToCoeff levels.  conj_key switches kappa_(2N-1)(s) -> s, relin_key s^2 -> s (key_id 0).  The
 * CoeffToSlot diagonals carry the factor 1/2 of the split into real and imaginary halves. */
typedef struct {
    int top_level;
    int n_c2s;
    const ckks_bsgs_level *c2s;
    int n_s2c;
    const ckks_bsgs_level *s2c;
    const ckks_evk *conj_key;
    const ckks_evk *relin_key;
    int r, d;
} ckks_bootstrap_plan;

/* CKKS bootstrapping (Cheon, Han, Kim, Kim, Song, Eurocrypt 2018; the linear maps as levels of the
 * slot DFT, Chen, Chillotti, Song, Eurocrypt 2019; the pages name bootstrapping and its cost but give
 * no construction): a ciphertext at level 0, ct [2][1][N], is raised to top_level (its plaintext
 * becomes m + q_0 I); CoeffToSlot (each level one ckks_bsgs and one ckks_rescale) leaves the slots
 * holding the raised coefficients over q_0, in bit-reversed order, at scale q_0; one conjugation
 * splits them into the real half z + conj(z) and the imaginary half X^(N/2) (conj(z) - z); EvalMod
 * (ckks_evalmod_batch on both halves) replaces each value x by sin(2 pi x) / (2 pi), which removes
 * I; the halves are recombined as real + X^(N/2) imag; SlotToCoeff moves the values back into the
 * coefficients.  The output decrypts to m (the input's message), scaled by *out_ratio: it decodes
 * at the input's scale times *out_ratio.  It is exact where m is small against q_0, up to the
 * approximation of EvalMod and the noise of the steps.
 *   out: [2][*out_level+1][N] with *out_level = top_level - n_c2s - (d + r + 3) - n_s2c;
 *   ws: ckks_bootstrap_workspace_bytes(ctx, plan) bytes (0 for a plan out of range).
 * Errors: CKKS_ERR_ARG (null pointers, level counts outside 1..16, r outside 0..16, d outside 1..16,
 * overlaps between the input, the output, the workspace and the plaintexts, and every error of the
 * ckks_bsgs calls), CKKS_ERR_UNSUPPORTED (top_level above the chain or below the levels consumed),
 * CKKS_ERR_ALIGN, CKKS_ERR_WORKSPACE. */
size_t ckks_bootstrap_workspace_bytes(ckks_ctx *ctx, const ckks_bootstrap_plan *plan);
int ckks_bootstrap(ckks_ctx *ctx, const uint32_t *ct, const ckks_bootstrap_plan *plan, uint32_t *out, int *out_level,
                   double *out_ratio, void *ws, size_t ws_bytes, ckks_stream_t stream);

/* Base-conversion engine (the results are the same residues either way; the bits of every
 * entry point's output are identical):
 *  CKKS_BCONV_TENSOR: the conversion as an exact 8-bit contraction on the tensor cores
 *    (tcgen05.mma kind::i8, sm_100a): inputs split into bytes along K with the byte shifts folded
 *    into the constants, 4 byte columns per target summed with shifts 0, 8, 16, 24 in the
 *    epilogue.  Groups of more than 15 primes use the CUDA cores;
 *  CKKS_BCONV_CUDA_CORES: 32 x 32 -> 64-bit multiply-adds on the CUDA cores;
 *  CKKS_BCONV_AUTO (default): the tensor cores for launches large enough to give each block of
 *    the tensor-core kernel at least 4 tiles of 128 coefficients, the CUDA cores otherwise.
 * The mode applies to later calls on the context; it is not synchronised with calls in flight
 * from other threads.  CKKS_ERR_ARG for an unknown mode. */
enum { CKKS_BCONV_CUDA_CORES = 0, CKKS_BCONV_TENSOR = 1, CKKS_BCONV_AUTO = 2 };
int ckks_set_bconv_mode(ckks_ctx *ctx, int mode);

/* The key's regenerated uniform half for one (digit, global limb): out [N] (device),
 * out[n] = w mod q_t with w = (x[2m] | x[2m+1] << 32), m = n mod 8, x = ChaCha12 block
 * (RFC 8439 state: key = seed as 8 LE words, counter = n/8, nonce = (key_id, digit, limb)). */
int ckks_chacha_expand(ckks_ctx *ctx, const uint8_t seed[32], uint32_t key_id, int digit, int limb,
                       uint32_t *out, ckks_stream_t stream);

/* Key switching without any device allocation, for callers that must not allocate device
 * memory themselves: code that runs inside a host framework which owns every device
 * allocation (a serving runtime with its own memory pool that forbids third-party cudaMalloc),
 * or a latency-critical loop where a cudaMalloc, which may synchronise the device, is not
 * acceptable.  Same operation and output as ckks_keyswitch; the workspace is a fixed array in
 * the library's device memory (CKKS_NOALLOC_SCRATCH_BYTES, present on every GPU that loads the
 * library until the process exits) instead of a caller buffer.
 *  - Returns CKKS_ERR_WORKSPACE when ckks_workspace_bytes(ctx, level, 1) exceeds that size
 *    (N=2^12 and N=2^14 parameter sets fit; N=2^16 with 36+12 primes does not).
 *  - ckks_ctx_create looks up the array's device address on the context's device and keeps it
 *    in the context, so the entry point itself makes no set-up call.  A device reset
 *    invalidates the address together with the context's tables: create a new context after it.
 *    Like every entry point, it returns CKKS_ERR_ARG when the current device is not the
 *    context's.
 *  - Every call on a device shares the one array: calls that may overlap on the GPU (different
 *    streams, or different host threads) race on it; serialise them.  Nothing in the array
 *    needs to start at zero, so the previous call's contents are harmless.
 *  - Allocates nothing: no cudaMalloc, no cudaFree.
 * (This entry point is an engineering addition; the pages describe nothing like it.) */
#define CKKS_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)
int ckks_keyswitch_noalloc(ckks_ctx *ctx, const uint32_t *c, int level, const ckks_evk *evk,
                           uint32_t *out, ckks_stream_t stream);

/* Workspace bytes for keyswitch/rotate/relin/modup/moddown at `level`; n > 1: a batch of n
 * items, or rotate_hoisted with n rotations (batches run in chunks of 64, so n is capped at 64). */
size_t ckks_workspace_bytes(const ckks_ctx *ctx, int level, int n);

/* Waits for `stream` with a deadline (polling, no device-side wait): CKKS_OK when the
 * stream is idle and no CUDA error is pending, CKKS_ERR_TIMEOUT at the deadline,
 * CKKS_ERR_CUDA on an asynchronous error.  With a context, it then reads (and clears) the
 * context's device error word: kernels whose waits are bounded (the shared-memory pipeline of
 * ckks_bsgs) record an expired wait there and return early, and ckks_sync_status reports it as
 * CKKS_ERR_TIMEOUT; the results of the calls since the previous check are then invalid, and the
 * context stays usable.  In the debug-bounds build it last reads (and clears) the index-check
 * record and returns CKKS_ERR_BOUNDS when a check failed since the previous clear. */
int ckks_sync_status(ckks_ctx *ctx, ckks_stream_t stream, int timeout_ms);

/* Self-test of the failure path of bounded device waits (no counterpart in the pages):
 * launches one block that waits on an mbarrier that never completes, so its bounded wait
 * expires after about one second and sets the context's device error word; the next
 * ckks_sync_status on `stream` returns CKKS_ERR_TIMEOUT and clears it, and the context stays
 * usable.  Nothing faults or hangs. */
int ckks_selftest_wait_expiry(ckks_ctx *ctx, ckks_stream_t stream);

/* Self-test of the CUDA-error path (no counterpart in the pages): launches a kernel with an
 * invalid configuration (2048 threads per block), which the CUDA runtime rejects on the host
 * before anything reaches the GPU, and returns what every entry point returns after a failed
 * launch: CKKS_ERR_CUDA, with the runtime's message in ckks_last_error().  The error is not
 * sticky: the context and the stream stay usable. */
int ckks_selftest_launch_error(ckks_ctx *ctx, ckks_stream_t stream);

/* Debug-bounds build (a checking aid; the pages have no counterpart).  The same sources compiled
 * with -DCKKS_DEBUG_BOUNDS (`python fhe_key_switching_b200/build.py --debug` writes
 * libckks_ks_debug.so beside the release library) give every kernel index checks: before each
 * group of global-memory accesses it checks that the group's span lies inside one region of the
 * running call -- the caller's buffers, sized from the call's arguments as this header states
 * (a workspace by the ws_bytes passed), the keys ([D][n_q+n_p][N] words per half), and the
 * context's device tables.  A failed check is counted in a device record that keeps the first
 * failure's site, address and size, and the accesses of that group are skipped (loads read 0), so
 * a wrong index is reported and no memory outside the call's buffers is touched.  Shared memory is
 * filled with a poison word at the start of each kernel that stages data in it, so that a read of
 * a word never written gives a wrong result.  Calls may run on several streams at once: each
 * call's regions stay in the table until its stream has run the call's last launch.  The
 * release build has no checks and the same results; the integer-throughput probe is not
 * instrumented.
 *   ckks_debug_bounds_enabled: 1 in the debug-bounds build, 0 otherwise.
 *   ckks_debug_bounds_report: waits for the current device, then stores the number of failed
 *     checks since the last clear and the first failure's site (see ckks_debug_bounds_site_name),
 *     address and size (each pointer but count may be NULL); clear != 0 empties the record.
 *     CKKS_ERR_UNSUPPORTED in the release build.
 *   ckks_debug_bounds_site_name: the name of a check site ("unknown" outside the list).
 *   ckks_selftest_bounds: enqueues on `stream` one check of the 4 bytes after the context's
 *     device error word (a region of its own), which fails and is recorded at site "selftest";
 *     nothing is read or written.  CKKS_ERR_UNSUPPORTED in the release build. */
int ckks_debug_bounds_enabled(void);
int ckks_debug_bounds_report(uint64_t *count, int *site, uint64_t *addr, uint64_t *bytes, int clear);
const char *ckks_debug_bounds_site_name(int site);
int ckks_selftest_bounds(ckks_ctx *ctx, ckks_stream_t stream);

/* Kernel timing.  Between ckks_prof_begin and ckks_prof_end, every launch of the kernel named
 * `kernel` ("ip_row", "bconv", "ntt_col_fwd", "ntt_col_inv", "ntt_row_fwd", "ntt_row_inv",
 * "row_combine", "tensor", "bsgs_combine") made through `ctx` is bracketed by CUDA events recorded on its
 * launching stream; up to max_launches launches are recorded (the events are created by
 * ckks_prof_begin, outside any timed region).  ckks_prof_end synchronises on the last event and
 * returns the number of recorded launches and their summed device time in milliseconds.
 * Not thread-safe: one profiling session per context at a time. */
int ckks_prof_begin(ckks_ctx *ctx, const char *kernel, int max_launches);
int ckks_prof_end(ckks_ctx *ctx, int *launches, double *total_ms);

/* Integer throughput probe (a measurement aid; the pages have no counterpart).  Launches one
 * kernel of `blocks` blocks x 256 threads on `stream`, each thread running 8 independent
 * dependency chains of the operation `op` for `iters` iterations, and waits for it.
 *   CKKS_PROBE_IADD       add.u32              CKKS_PROBE_IMAD       mad.lo.u32
 *   CKKS_PROBE_LOP3       lop3.b32             CKKS_PROBE_IMAD_HI    mad.hi.u32
 *   CKKS_PROBE_SHF        shf.l.wrap.b32       CKKS_PROBE_IMAD_WIDE  mad.wide.u32 (64-bit sum)
 *   CKKS_PROBE_MIX        alternating lop3.b32 and mad.lo.u32
 *   CKKS_PROBE_CHACHA12   the library's ChaCha12 block function, counted as 608 int32
 *                         operations per block (the op model's unit cost)
 * sink: device, blocks * 256 words (written, 16-byte aligned).  *ms: the launch's elapsed time
 * (CUDA events on `stream`); *ops: the operations it executed.  Returns CKKS_ERR_ARG for a bad
 * argument, CKKS_ERR_CUDA when the launch fails.  Synchronous; not for use inside a capture. */
enum {
    CKKS_PROBE_IADD = 0, CKKS_PROBE_LOP3, CKKS_PROBE_SHF, CKKS_PROBE_IMAD, CKKS_PROBE_IMAD_HI,
    CKKS_PROBE_IMAD_WIDE, CKKS_PROBE_MIX, CKKS_PROBE_CHACHA12, CKKS_PROBE_COUNT
};
int ckks_int_probe(int op, int blocks, int iters, uint32_t *sink, ckks_stream_t stream, float *ms,
                   double *ops);

/* Message of the last error on this thread ("" if none). */
const char *ckks_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* CKKS_KS_H */
