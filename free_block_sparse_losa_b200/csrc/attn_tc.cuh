// Definitions shared by the tensor-core attention kernels (bf16, head_dim 128, 128-row query blocks): tile geometry,
// the argument block, bounded mbarrier waits, work items and their key lists, the bf16 pair unpacking and the MMA form
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
    float* mass_part;              // one-pass masses: per-CTA scratch of [nkb][128] fp32 partial sums (else null)
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
