// Definitions shared by the tensor-core attention kernels (bf16, head_dim 128, 128-row query blocks): tile geometry,
// the argument block, bounded mbarrier waits, work items and their key lists, the polynomial 2^x and the MMA form
// whose A operand comes from tensor memory. The kernels are attn_dense.cuh (dense steps, with or without the block
// masses) and attn_sparse.cuh (retained lists).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace losa {

constexpr int kTcRows = 128;      // R = C = 128
constexpr int kTcDim = 128;       // head_dim
constexpr int kTcThreads = 384;
constexpr uint32_t kTileBytes = kTcRows * kTcDim * 2;   // 32 KB: one 128 x 128 bf16 tile
constexpr uint32_t kBoxBytes = kTileBytes / 2;         // 16 KB: one 128-row x 64-column TMA box
constexpr unsigned long long kDrainLimitNs = 2000000000ull;  // bound of the exit-path waits
constexpr int kMaxMassBlocks = 1024;                   // key blocks per flush of the dense kernel's mass phase

struct TcArgs {
    int H, N, Np, nq, nk, n_items;  // nk: 128-key tiles per head (Np / 128)
    int nkb;                        // key blocks of the selection (Np / C): nk for C = 128, 4 * nk for C = 32
    float scale_log2;              // logit scale times log2(e)
    const int32_t* indptr;         // null: dense list 0..nk-1
    const int32_t* kv_idx;
    const int32_t* order;          // null: ascending item ids
    __nv_bfloat16* o;
    float* lse;                    // may be null
    float* mass;                   // [H*nq][nk], WITH_MASS only
    unsigned long long wait_limit_ns;
};

// Bounded wait on a barrier phase; records a timeout in the device error word.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, unsigned long long limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 63u) == 0 && global_timer_ns() - t0 > limit_ns) {
            atomicOr(&g_device_error, kDevErrTimeout);
            return false;
        }
    }
}

// Warp-uniform variant: all lanes poll, the warp agrees on the outcome.
__device__ __forceinline__ bool wait_bounded_warp(uint32_t bar, uint32_t parity, unsigned long long limit_ns) {
    const bool ok = wait_bounded(bar, parity, limit_ns);
    return __all_sync(0xffffffffu, ok);
}

struct ItemInfo {
    int id, h, qb, begin;
    int count;  // list entries (key blocks); every block for a dense call
    int tiles;  // forward 128-key tiles: ceil(count / SUB) for a list, nk for a dense call
};

// Item of CTA round `round` (false past the end of the work order).
__device__ __forceinline__ bool item_of_round(const TcArgs& a, int round, ItemInfo& it) {
    const int G = gridDim.x, b = blockIdx.x;
    const long long w = (long long)round * G + ((round & 1) ? (G - 1 - b) : b);
    if (w >= a.n_items) return false;
    it.id = a.order ? a.order[w] : (int)w;
    if (it.id < 0 || it.id >= a.n_items) {  // not a permutation of the items: report it and skip the entry
        atomicOr(&g_device_error, kDevErrBadData);
        it.id = 0;
        it.h = it.qb = it.begin = it.count = it.tiles = 0;
        return true;
    }
    it.h = it.id / a.nq;
    it.qb = it.id - it.h * a.nq;
    if (a.indptr) {
        it.begin = a.indptr[it.id];
        it.count = a.indptr[it.id + 1] - it.begin;
        it.tiles = (it.count + (a.nkb / a.nk) - 1) / (a.nkb / a.nk);
    } else {
        it.begin = 0;
        it.count = a.nkb;
        it.tiles = a.nk;
    }
    return true;
}

// 2^x on the FMA/ALU pipes, to take part of the load off the exp unit, for weights that are rounded to bf16 (relative
// step 2^-8) right after. Cody-Waite split x = n + f with n = round(x) (the 1.5 * 2^23 shift leaves n in the low
// mantissa bits) and f in [-1/2, 1/2]; 2^f by a degree-3 polynomial whose coefficients minimise the maximum relative
// error on that interval (fitted by Lawson's iteratively reweighted least squares; max relative error 7.5e-5 in fp32
// Horner form); n is added to the exponent field. Valid for x <= 126; inputs below -125 are clamped there
// (2^-125 ~ 2.4e-38), so callers that need exact zeros (masked keys) use ex2_approx instead. Works on a pair of fp32
// values with packed f32x2 arithmetic (the integer exponent update stays scalar).
constexpr float kExp2D0 = 0.9999280571937561f, kExp2D1 = 0.6932609677314758f, kExp2D2 = 0.2426111251115799f,
                kExp2D3 = 0.0551716685295105f;
__device__ __forceinline__ void exp2_poly2_d3(uint64_t xx, float& r0, float& r1) {
    float x0, x1;
    f2_unpack(xx, x0, x1);
    xx = f2_pack(fmaxf(x0, -125.0f), fmaxf(x1, -125.0f));
    const uint64_t t = f2_add(xx, f2_pack(12582912.0f, 12582912.0f));
    const uint64_t n = f2_add(t, f2_pack(-12582912.0f, -12582912.0f));
    const uint64_t f = f2_fma(n, f2_pack(-1.0f, -1.0f), xx);
    uint64_t p = f2_fma(f2_pack(kExp2D3, kExp2D3), f, f2_pack(kExp2D2, kExp2D2));
    p = f2_fma(p, f, f2_pack(kExp2D1, kExp2D1));
    p = f2_fma(p, f, f2_pack(kExp2D0, kExp2D0));
    float p0, p1, t0, t1;
    f2_unpack(p, p0, p1);
    f2_unpack(t, t0, t1);
    r0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
    r1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

// The two fp32 values a bf16 pair from pack_bf16x2 holds (low half first), exactly, as a packed fp32 pair. The
// attention kernels add them up per row: O is divided by the sum of the weights P V was given (the bf16-rounded P),
// which makes O a convex combination of V rows again, so the rounding of a dominant weight cancels; the exact fp32
// sum gives the log-sum-exp.
__device__ __forceinline__ uint64_t bf16x2_to_f2(uint32_t w) {
    return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// D[tmem] (+)= A[tmem] * B[smem desc]^T: the A operand (P) is read from tensor memory.
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
        ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

}  // namespace losa
