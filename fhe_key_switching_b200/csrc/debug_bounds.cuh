// debug_bounds.cuh -- the index checks of the debug-bounds build (compiled with -DCKKS_DEBUG_BOUNDS).
//
// Before each group of global-memory accesses a kernel checks the span the group touches (from
// its lowest to its highest address) against a table of regions that the host fills for the
// running call: the caller's buffers, sized from the call's arguments (a workspace by the size the
// caller passed), the keys, and the context's tables.  A span outside every region is counted in
// a device record that keeps the first failure's site and address, and the group's accesses are
// skipped (loads give 0), so that a wrong index is reported instead of reading or writing memory
// the call does not own.  Checks whose span is the same for the whole block (a table row chosen
// by blockIdx) make the block return at once.  Shared memory is filled with a poison word at the
// start of every kernel that stages data there, so that a read before the write shows up as a
// wrong result.
//
// In the release build every check is the constant true and the poison is empty, so both leave
// the kernels' code unchanged.
#pragma once
#include <cstddef>
#include <cstdint>

// Check sites (the record's site field; ckks_debug_bounds_site_name gives the names).
#define CKKS_DBG_SITES(X)                                                                          \
    X(SELFTEST, "selftest")                                                                        \
    X(NTT_TABLES, "ntt: prime record / twiddle row / scale")                                       \
    X(NTT_IN, "ntt: input")                                                                        \
    X(NTT_OUT, "ntt: output")                                                                      \
    X(CHACHA_OUT, "chacha_expand: output")                                                         \
    X(BCONV_TABLES, "bconv: constants / prime records")                                            \
    X(BCONV_IN, "bconv: input rows")                                                               \
    X(BCONV_OUT, "bconv: output rows")                                                             \
    X(IP_TABLES, "inner_product: prime record")                                                    \
    X(IP_IN, "inner_product: extended digit")                                                      \
    X(IP_KEY, "inner_product: key")                                                                \
    X(IP_OUT, "inner_product: accumulators")                                                       \
    X(TENSOR, "tensor: operands / output")                                                         \
    X(AUTOMORPH, "automorph: input / output")                                                      \
    X(ENCODE, "encode: coefficients / output")                                                     \
    X(COPY_DIGIT, "copy_digit_limbs: input / output")                                              \
    X(IPROW_TABLES, "ip_row: prime record / twiddle row")                                          \
    X(IPROW_X, "ip_row: column-pass rows")                                                         \
    X(IPROW_CDIG, "ip_row: digit limbs")                                                           \
    X(IPROW_KEY, "ip_row: key")                                                                    \
    X(IPROW_OUT, "ip_row: accumulators")                                                           \
    X(COMBINE_TABLES, "row_combine: prime record / twiddle row / P^-1")                            \
    X(COMBINE_IN, "row_combine: conversions / accumulators")                                       \
    X(COMBINE_ADD, "row_combine: added polynomial")                                                \
    X(COMBINE_OUT, "row_combine: output")                                                          \
    X(BSGS_TABLES, "bsgs_combine: prime record / [P]_q")                                           \
    X(BSGS_PT, "bsgs_combine: plaintext chunk")                                                    \
    X(BSGS_IN, "bsgs_combine: ciphertext / baby accumulators")                                     \
    X(BSGS_V, "bsgs_combine: giant sums")                                                          \
    X(SUM, "sum_parts: inputs / output")                                                           \
    X(TC_TABLES, "bconv_tc: constants / prime records")                                            \
    X(TC_IN, "bconv_tc: input rows")                                                               \
    X(TC_OUT, "bconv_tc: output")                                                                  \
    X(CONST, "const arithmetic: inputs / output")                                                  \
    X(ERR_WORD, "device error word")

enum CkksDbgSite {
    CKKS_DBG_NONE = 0,
#define CKKS_DBG_ENUM(id, name) CKKS_DBG_##id,
    CKKS_DBG_SITES(CKKS_DBG_ENUM)
#undef CKKS_DBG_ENUM
    CKKS_DBG_N_SITES
};

#ifdef CKKS_DEBUG_BOUNDS

constexpr int CKKS_DBG_MAX_REGIONS = 512;
constexpr unsigned CKKS_DBG_POISON_WORD = 0xA5A5A5A5u;

struct CkksDbgRegion {
    unsigned long long lo, hi;                 // bytes [lo, hi)
};
struct CkksDbgRecord {
    unsigned long long count;                  // failed checks since the last clear
    unsigned long long site, addr, bytes;      // the first of them
};

static __device__ CkksDbgRegion g_dbg_regions[CKKS_DBG_MAX_REGIONS];
static __device__ int g_dbg_n_regions;
static __device__ CkksDbgRecord g_dbg_record;

// true when [p, p + bytes) lies inside one registered region; otherwise counts the failure
__device__ __noinline__ bool ckks_dbg_span(const void *p, unsigned long long bytes, int site) {
    const unsigned long long lo = (unsigned long long)p, hi = lo + bytes;
    const int nr = *(volatile int *)&g_dbg_n_regions;
    if (hi >= lo)
        for (int i = 0; i < nr && i < CKKS_DBG_MAX_REGIONS; i++)
            if (lo >= g_dbg_regions[i].lo && hi <= g_dbg_regions[i].hi) return true;
    if (atomicAdd(&g_dbg_record.count, 1ull) == 0ull) {
        g_dbg_record.site = (unsigned long long)site;
        g_dbg_record.addr = lo;
        g_dbg_record.bytes = bytes;
    }
    return false;
}

// every thread of the block: fill `bytes` of shared memory at p with the poison word
__device__ __forceinline__ void ckks_dbg_poison(void *p, size_t bytes) {
    unsigned *w = (unsigned *)p;
    for (size_t i = threadIdx.x; i < bytes / 4; i += blockDim.x) w[i] = CKKS_DBG_POISON_WORD;
    __syncthreads();
}

__device__ __forceinline__ unsigned ckks_dbg_dynamic_smem_bytes() {
    unsigned b;
    asm volatile("mov.u32 %0, %%dynamic_smem_size;" : "=r"(b));
    return b;
}

// [p, p + count elements of *p) inside a registered region
#define CKKS_SPAN(p, count, site) ckks_dbg_span((p), (unsigned long long)(count) * sizeof(*(p)), (site))
// [lo, hi] (both element pointers, inclusive) inside one registered region
#define CKKS_SPAN2(lo, hi, site) \
    ckks_dbg_span((lo), (unsigned long long)((const char *)((hi) + 1) - (const char *)(lo)), (site))
#define CKKS_POISON(p, bytes) ckks_dbg_poison((p), (bytes))
#define CKKS_POISON_DYNAMIC(p) ckks_dbg_poison((p), ckks_dbg_dynamic_smem_bytes())

// The host's region slots reach the device through this kernel, launched on the registering
// call's stream before its first launch: it writes that call's slots only and raises the table
// length with atomicMax, so that calls on other streams never see their own slots shrink away.
constexpr int CKKS_DBG_PUBLISH_MAX = 64;
struct CkksDbgPublish {
    int n;
    int slot[CKKS_DBG_PUBLISH_MAX];
    CkksDbgRegion r[CKKS_DBG_PUBLISH_MAX];
};
__global__ void k_dbg_publish(CkksDbgPublish p) {
    const int i = threadIdx.x;
    if (i < p.n && p.slot[i] >= 0 && p.slot[i] < CKKS_DBG_MAX_REGIONS) {
        g_dbg_regions[p.slot[i]] = p.r[i];
        __threadfence();
        atomicMax(&g_dbg_n_regions, p.slot[i] + 1);
    }
}

// Self-test of the record: checks the 4 bytes after a word the host registered as a region of its
// own (a cudaMalloc'd word: no other allocation starts before the next 256-byte boundary), so the
// check fails; nothing is read or written.
__global__ void k_bounds_probe(const int *word) { (void)CKKS_SPAN(word + 1, 1, CKKS_DBG_SELFTEST); }

#else

#define CKKS_SPAN(p, count, site) true
#define CKKS_SPAN2(lo, hi, site) true
#define CKKS_POISON(p, bytes) ((void)0)
#define CKKS_POISON_DYNAMIC(p) ((void)0)

#endif
