// Tensor-core (tcgen05 / TMEM / TMA) attention kernel for bf16 inputs, head_dim 128, 128 x 128 blocks.
//
// attn_tc_kernel<WITH_MASS> processes work items = (head, 128-row query block):
//   forward phase — online-softmax attention against a list of 128-key blocks: the full list 0..nk-1 for a dense
//                   step (LoSA page, Motivation Summary: A = softmax(Q K^T / sqrt(d))) or the frozen retained list for
//                   later steps (Methodology Summary, "Sparse attention with a frozen pattern": the softmax
//                   denominator covers the retained keys only). Writes O (bf16) and the row log-sum-exp.
//   mass phase    — (WITH_MASS) recomputes S = Q K^T for every key block and sums 2^(s*c - lse2) with the forward
//                   phase's exact log-sum-exp, still in registers, into one value per (query block, key block), then
//                   divides by the block's real rows (Motivation Summary: block attention mass M(i, j)). The
//                   probability matrix is never stored.
//
// Persistent grid, one CTA (384 threads) per SM, split into two independent LANES that share the SM's tensor core
// and TMA unit. Lane x owns 96 KB of shared memory (Q, K and V tiles), 256 TMEM columns (S/P and O, 128 each) and
// three roles: a TMA producer thread (warp 2x), an MMA issuer thread (warp 2x + 1) and a softmax warpgroup (warps
// 4 + 4x .. 7 + 4x; thread t owns query row t = TMEM lane t). Lane x takes rounds x, x + 2, x + 4, ... of the CTA's
// items; CTA b's round r is item r*G + b (r even) or r*G + G - 1 - b (r odd) of the work order, a snake over the
// longest-first order. Inside a lane, tile t flows QK^T -> softmax -> P V -> next QK^T; the other lane fills the
// tensor core meanwhile, and two softmax warps per SM sub-partition hide each other's latencies.
//
// S = Q K^T lands in the lane's S/P columns; the softmax writes P = 2^(s*c - m*c) as packed bf16 into the first 64
// of them and the MMA computes O += P V with P read from TMEM (V is an MN-major shared-memory operand). O is
// rescaled in place only when a row's running max grows by more than 2^8 (the final division by the sum taken
// against the same reference keeps this exact).
//
// Every wait is bounded in time; on expiry the kernel records LOSA_ERR_TIMEOUT in the device error word, waits for its
// own copies and MMAs in flight, frees TMEM and exits.
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
constexpr int kMaxMassBlocks = 1024;                   // nk limit of the mass phase (partial-sum buffer)

// Per-lane shared memory (from a 1024-aligned base): Q, K, V tiles, then (mass) 4 x 1024 fp32 partial sums.
constexpr uint32_t kLaneQ = 0, kLaneK = kTileBytes, kLaneV = 2 * kTileBytes;
constexpr uint32_t kLaneTiles = 3 * kTileBytes;                         // 96 KB
constexpr uint32_t kPartBytes = 4 * kMaxMassBlocks * 4;                 // 16 KB
constexpr uint32_t kBarBytes = 256;                                     // per lane
template <bool M>
constexpr uint32_t tc_smem_bytes() {
    return 2 * kLaneTiles + (M ? 2 * kPartBytes : 0) + 2 * kBarBytes + 1024;  // + alignment slack
}

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

// Block index of list entry e (clamped; the producer reports out-of-range entries).
__device__ __forceinline__ int list_block(const TcArgs& a, const ItemInfo& it, int e) {
    const int j = a.kv_idx[it.begin + e];
    return (j < 0) ? 0 : (j >= a.nkb ? a.nkb - 1 : j);
}

// Real keys in each 32-key quarter of forward tile t, packed 8 bits per quarter. A quarter with no list entry (the
// tail of a C = 32 list) has none; the ragged end of the sequence cuts the last block.
template <int SUB>
__device__ __forceinline__ uint32_t quarter_keys(const TcArgs& a, const ItemInfo& it, int t) {
    uint32_t kv = 0;
    if (SUB == 1 || !a.indptr) {
        const int j128 = a.indptr ? list_block(a, it, t) : t;
        const int kvalid = a.N - j128 * 128;
#pragma unroll
        for (int g = 0; g < 4; ++g) kv |= (uint32_t)min(32, max(0, kvalid - 32 * g)) << (8 * g);
    } else {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const int e = SUB * t + g;
            if (e < it.count) kv |= (uint32_t)min(32, max(0, a.N - list_block(a, it, e) * 32)) << (8 * g);
        }
    }
    return kv;
}


// 2^x on the FMA/ALU pipes, to take part of the load off the exp unit. Cody-Waite split x = n + f with n = round(x)
// (the 1.5 * 2^23 shift leaves n in the low mantissa bits) and f in [-1/2, 1/2]; 2^f by a degree-4 polynomial whose
// coefficients minimise the maximum relative error on that interval (fitted by Lawson's iteratively reweighted least
// squares; max relative error 2.7e-6 evaluated in fp32 Horner form); n is added to the exponent field. Valid for
// x <= 126; inputs below -125 are clamped there (2^-125 ~ 2.4e-38), so callers that need exact zeros (masked keys)
// use ex2_approx instead.
constexpr float kExp2C0 = 0.9999992847442627f, kExp2C1 = 0.6931217908859253f, kExp2C2 = 0.240247443318367f,
                kExp2C3 = 0.05591785907745361f, kExp2C4 = 0.009570102207362652f;
__device__ __forceinline__ float exp2_poly(float x) {
    x = fmaxf(x, -125.0f);
    const float t = x + 12582912.0f;
    const float f = x - (t - 12582912.0f);
    float p = fmaf(kExp2C4, f, kExp2C3);
    p = fmaf(p, f, kExp2C2);
    p = fmaf(p, f, kExp2C1);
    p = fmaf(p, f, kExp2C0);
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// exp2_poly on a pair of fp32 values with packed f32x2 arithmetic (the integer exponent update stays scalar).
__device__ __forceinline__ void exp2_poly2(uint64_t xx, float& r0, float& r1) {
    float x0, x1;
    f2_unpack(xx, x0, x1);
    xx = f2_pack(fmaxf(x0, -125.0f), fmaxf(x1, -125.0f));
    const uint64_t t = f2_add(xx, f2_pack(12582912.0f, 12582912.0f));
    const uint64_t n = f2_add(t, f2_pack(-12582912.0f, -12582912.0f));
    const uint64_t f = f2_fma(n, f2_pack(-1.0f, -1.0f), xx);
    uint64_t p = f2_fma(f2_pack(kExp2C4, kExp2C4), f, f2_pack(kExp2C3, kExp2C3));
    p = f2_fma(p, f, f2_pack(kExp2C2, kExp2C2));
    p = f2_fma(p, f, f2_pack(kExp2C1, kExp2C1));
    p = f2_fma(p, f, f2_pack(kExp2C0, kExp2C0));
    float p0, p1, t0, t1;
    f2_unpack(p, p0, p1);
    f2_unpack(t, t0, t1);
    r0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
    r1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
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

// Barrier slots of one lane (8 bytes each). Counts: P_FULL, O_FREE, S_FREE, PART take 128 arrivals, the rest 1.
enum : uint32_t {
    L_Q_FULL = 0, L_Q_EMPTY, L_K_FULL, L_K_EMPTY, L_V_FULL, L_V_EMPTY, L_S_FULL, L_P_FULL, L_PV_DONE, L_O_FREE,
    L_S_FREE, L_PART, L_PART2, L_MMA_DONE, L_COUNT
};

// SUB = key blocks per 128-key tile: 1 for C = 128, 4 for C = 32 (tmK32 / tmV32: 32-row boxes for gathering a list's
// 32-key blocks into the quarters of a tile).
template <bool WITH_MASS, int SUB>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmK32,
                   const __grid_constant__ CUtensorMap tmV32, const TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const base_ptr = smem_raw + (base - raw);
    const uint32_t part_off = 2 * kLaneTiles;
    const uint32_t bar_off = part_off + (WITH_MASS ? 2 * kPartBytes : 0);
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + bar_off + 2 * kBarBytes - 16);

    const int warp = threadIdx.x >> 5;
    const uint32_t lane = lane_id();
    // lane x: producer warp 2x, MMA warp 2x + 1, softmax warps 4 + 4x .. 7 + 4x
    const uint32_t x = (warp < 4) ? (uint32_t)(warp >> 1) : (uint32_t)((warp - 4) >> 2);
    const uint32_t bar0 = base + bar_off + x * kBarBytes;
    auto BAR = [&](uint32_t s) { return bar0 + 8u * s; };
    const uint32_t sQ = base + x * kLaneTiles + kLaneQ;
    const uint32_t sK = base + x * kLaneTiles + kLaneK;
    const uint32_t sV = base + x * kLaneTiles + kLaneV;

    if (threadIdx.x < 2) {  // thread 0 initialises lane 0's barriers, thread 1 lane 1's
        const uint32_t b0 = base + bar_off + threadIdx.x * kBarBytes;
        for (uint32_t s = 0; s < L_COUNT; ++s) {
            const bool wide = (s == L_P_FULL || s == L_O_FREE || s == L_S_FREE || s == L_PART || s == L_PART2);
            mbar_init(b0 + 8u * s, wide ? 128u : 1u);
        }
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), 512);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        if (SUB > 1) {
            tma_prefetch_desc(&tmK32);
            tma_prefetch_desc(&tmV32);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
    const uint32_t tS = tmem + x * 256u;        // lane's S/P columns
    const uint32_t tO = tS + 128u;              // lane's O columns
    const unsigned long long lim = a.wait_limit_ns;
    const int mass_tiles = WITH_MASS ? a.nk : 0;

    if (warp < 4 && (warp & 1) == 0) {
        // ------------------------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            const uint64_t pol_q = l2_policy_evict_first();
            const uint64_t pol_kv = l2_policy_evict_last();
            uint32_t nq = 0, nk_ld = 0, nv_ld = 0;
            bool ok = true;
            ItemInfo it;
            for (int r = (int)x; ok && item_of_round(a, r, it); r += 2) {
                if (it.count <= 0) {
                    if (a.indptr) atomicOr(&g_device_error, kDevErrBadData);
                    continue;
                }
                if (!(ok = wait_bounded(BAR(L_Q_EMPTY), (nq & 1u) ^ 1u, lim))) break;
                const int32_t qrow = it.h * a.Np + it.qb * kTcRows;
                mbar_arrive_expect_tx(BAR(L_Q_FULL), kTileBytes);
                tma_load_2d_hint(sQ, &tmQ, 0, qrow, BAR(L_Q_FULL), pol_q);
                tma_load_2d_hint(sQ + kBoxBytes, &tmQ, 64, qrow, BAR(L_Q_FULL), pol_q);
                ++nq;
                const int total = it.tiles + mass_tiles;
                for (int t = 0; t < total; ++t) {
                    const bool fwd = t < it.tiles;
                    const bool gather = fwd && SUB > 1 && a.indptr;  // C = 32 list: four 32-row blocks per tile
                    int32_t krow = 0;
                    if (!gather) {
                        const int j = fwd ? (a.indptr ? list_block(a, it, t) : t) : t - it.tiles;
                        krow = it.h * a.Np + j * kTcRows;
                    }
                    if (fwd && a.indptr) {
                        for (int e = SUB * t; e < SUB * t + SUB && e < it.count; ++e) {
                            const int jr = a.kv_idx[it.begin + e];
                            if (jr < 0 || jr >= a.nkb) atomicOr(&g_device_error, kDevErrBadData);
                        }
                    }
                    if (!(ok = wait_bounded(BAR(L_K_EMPTY), (nk_ld & 1u) ^ 1u, lim))) break;
                    mbar_arrive_expect_tx(BAR(L_K_FULL), kTileBytes);
                    if (!gather) {
                        tma_load_2d_hint(sK, &tmK, 0, krow, BAR(L_K_FULL), pol_kv);
                        tma_load_2d_hint(sK + kBoxBytes, &tmK, 64, krow, BAR(L_K_FULL), pol_kv);
                    } else {
#pragma unroll
                        for (int g = 0; g < SUB; ++g) {
                            // a missing quarter reloads the tile's first block (finite data, masked to P = 0)
                            const int e = SUB * t + g < it.count ? SUB * t + g : SUB * t;
                            const int32_t r32 = it.h * a.Np + list_block(a, it, e) * 32;
                            tma_load_2d_hint(sK + g * 4096u, &tmK32, 0, r32, BAR(L_K_FULL), pol_kv);
                            tma_load_2d_hint(sK + kBoxBytes + g * 4096u, &tmK32, 64, r32, BAR(L_K_FULL), pol_kv);
                        }
                    }
                    ++nk_ld;
                    if (fwd) {
                        if (!(ok = wait_bounded(BAR(L_V_EMPTY), (nv_ld & 1u) ^ 1u, lim))) break;
                        mbar_arrive_expect_tx(BAR(L_V_FULL), kTileBytes);
                        if (!gather) {
                            tma_load_2d_hint(sV, &tmV, 0, krow, BAR(L_V_FULL), pol_kv);
                            tma_load_2d_hint(sV + kBoxBytes, &tmV, 64, krow, BAR(L_V_FULL), pol_kv);
                        } else {
#pragma unroll
                            for (int g = 0; g < SUB; ++g) {
                                const int e = SUB * t + g < it.count ? SUB * t + g : SUB * t;
                                const int32_t r32 = it.h * a.Np + list_block(a, it, e) * 32;
                                tma_load_2d_hint(sV + g * 4096u, &tmV32, 0, r32, BAR(L_V_FULL), pol_kv);
                                tma_load_2d_hint(sV + kBoxBytes + g * 4096u, &tmV32, 64, r32, BAR(L_V_FULL), pol_kv);
                            }
                        }
                        ++nv_ld;
                    }
                }
            }
            // Drain: every copy this thread issued lands before the CTA may exit.
            if (nq) wait_bounded(BAR(L_Q_FULL), (nq - 1) & 1u, kDrainLimitNs);
            if (nk_ld) wait_bounded(BAR(L_K_FULL), (nk_ld - 1) & 1u, kDrainLimitNs);
            if (nv_ld) wait_bounded(BAR(L_V_FULL), (nv_ld - 1) & 1u, kDrainLimitNs);
        }
        __syncwarp();
    } else if (warp < 4) {
        // ------------------------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdQK = idesc_bf16_f32(128, 128, false, false);
            constexpr uint32_t kIdPV = idesc_bf16_f32(128, 128, false, true);
            uint32_t nq = 0, nk_use = 0, nv_use = 0, n_pv = 0, n_sfree = 0, n_items = 0;
            bool ok = true;
            ItemInfo it;
            for (int r = (int)x; ok && item_of_round(a, r, it); r += 2) {
                if (it.count <= 0) continue;
                if (!(ok = wait_bounded(BAR(L_Q_FULL), nq & 1u, lim))) break;
                ++nq;
                const int total = it.tiles + mass_tiles;
                for (int t = 0; t < total; ++t) {
                    const bool fwd = t < it.tiles;
                    if (!(ok = wait_bounded(BAR(L_K_FULL), nk_use & 1u, lim))) break;
                    // The S/P columns are free once the previous tile's P V (forward) or S read (mass) completed.
                    if (t > 0 && t <= it.tiles) {
                        if (!(ok = wait_bounded(BAR(L_PV_DONE), (n_pv - 1) & 1u, lim))) break;
                    } else if (t > it.tiles) {
                        if (!(ok = wait_bounded(BAR(L_S_FREE), (n_sfree - 1) & 1u, lim))) break;
                    } else if (n_items > 0) {
                        // first tile of an item: the previous item's last S/P use must be over
                        if (!(ok = (mass_tiles ? wait_bounded(BAR(L_S_FREE), (n_sfree - 1) & 1u, lim)
                                               : wait_bounded(BAR(L_PV_DONE), (n_pv - 1) & 1u, lim))))
                            break;
                    }
                    tc_fence_after();
#pragma unroll
                    for (uint32_t kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3u) * 32u;
                        tc_mma_ss(tS, smem_desc(sQ + off, 16, 1024), smem_desc(sK + off, 16, 1024), kIdQK,
                                  kk ? 1u : 0u);
                    }
                    tc_commit(BAR(L_S_FULL));
                    tc_commit(BAR(L_K_EMPTY));
                    ++nk_use;
                    if (t == total - 1) tc_commit(BAR(L_Q_EMPTY));
                    if (fwd) {
                        if (!(ok = wait_bounded(BAR(L_P_FULL), n_pv & 1u, lim))) break;
                        if (!(ok = wait_bounded(BAR(L_V_FULL), nv_use & 1u, lim))) break;
                        if (t == 0 && !(ok = wait_bounded(BAR(L_O_FREE), (n_items & 1u) ^ 1u, lim))) break;
                        tc_fence_after();
#pragma unroll
                        for (uint32_t kk = 0; kk < 8; ++kk) {
                            const uint64_t db = smem_desc(sV + kk * 2048u, kBoxBytes, 1024);
                            tc_mma_ts(tO, tS + kk * 8u, db, kIdPV, (t == 0 && kk == 0) ? 0u : 1u);
                        }
                        tc_commit(BAR(L_V_EMPTY));
                        tc_commit(BAR(L_PV_DONE));
                        ++nv_use;
                        ++n_pv;
                    } else {
                        ++n_sfree;  // the softmax frees S after reading it; the wait happens before the next QK
                    }
                }
                ++n_items;
            }
            tc_commit(BAR(L_MMA_DONE));
            wait_bounded(BAR(L_MMA_DONE), 0, kDrainLimitNs);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------------------- softmax / epilogue
        const uint32_t wl = (uint32_t)warp & 3u;
        const int row = (int)(wl * 32u + lane);
        const uint32_t lane_off = (wl * 32u) << 16;
        const float c = a.scale_log2;
        float* const part = reinterpret_cast<float*>(base_ptr + part_off + x * kPartBytes);
        uint32_t n_s = 0, n_pv = 0, n_items = 0, n_chunks = 0;
        bool ok = true;
        ItemInfo it;
        for (int r = (int)x; ok && item_of_round(a, r, it); r += 2) {
            if (it.count <= 0) continue;
            const int qrow = it.qb * kTcRows + row;
            const size_t grow = (size_t)it.h * a.Np + qrow;
            float m_raw = -INFINITY, l_run = 0.0f;
            uint32_t kvn = quarter_keys<SUB>(a, it, 0);
            for (int t = 0; t < it.tiles; ++t) {
                const uint32_t kv4 = kvn;  // real keys per 32-column quarter of this tile
                if (t + 1 < it.tiles) kvn = quarter_keys<SUB>(a, it, t + 1);  // prefetched one tile ahead
                const bool full = kv4 == 0x20202020u;
                if (!(ok = wait_bounded_warp(BAR(L_S_FULL), n_s & 1u, lim))) break;
                ++n_s;
                tc_fence_after();
                // Pass 1: the tile's row max over all 128 columns (only columns 0..31 stay live afterwards).
                float s0[32];
                float tmax;
                {
                    float s[128];
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch)
                        tmem_ld32(tS + lane_off + ch * 32u, *reinterpret_cast<uint32_t(*)[32]>(&s[ch * 32]));
                    tmem_wait_ld();
                    if (!full) {  // keys past the sequence end, or quarters without a listed block, do not exist
#pragma unroll
                        for (int cc = 0; cc < 128; ++cc)
                            if ((uint32_t)(cc & 31) >= ((kv4 >> (8 * (cc >> 5))) & 255u)) s[cc] = -INFINITY;
                    }
                    float mx[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) mx[e] = fmax3(s[e], s[8 + e], s[16 + e]);
#pragma unroll
                    for (int cc = 24; cc < 128; cc += 16)
#pragma unroll
                        for (int e = 0; e < 8; ++e) mx[e] = fmax3(mx[e], s[cc + e], s[cc + 8 + e]);
                    tmax = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], fmax3(mx[5], mx[6], mx[7])));
#pragma unroll
                    for (int e = 0; e < 32; ++e) s0[e] = s[e];
                }
                // Reference max: raised only when the tile max exceeds it by more than 2^8 in the exp2 domain.
                const bool need = (t == 0) || (tmax - m_raw) * c > 8.0f;
                const float alpha = (t > 0 && need && tmax != -INFINITY) ? ex2_approx((m_raw - tmax) * c) : 1.0f;
                // A tile without any real key (only possible for a listed block that is all padding) keeps a finite
                // reference so that its weights come out as exact zeros.
                if (need) m_raw = (tmax == -INFINITY) ? (t == 0 ? 0.0f : m_raw) : tmax;
                const float neg_mc = -m_raw * c;
                // Pass 2, 32 columns at a time, the next chunk's TMEM load in flight during this chunk's math:
                // P = 2^(s*c - m*c) as bf16 pairs written behind the read position (columns 16*ch .. 16*ch + 15
                // hold keys 32*ch .. 32*ch + 31).
                uint64_t l2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
                float rb[2][32];
#pragma unroll
                for (int ch = 0; ch < 4; ++ch) {
                    if (ch < 3)
                        tmem_ld32(tS + lane_off + (ch + 1) * 32u, *reinterpret_cast<uint32_t(*)[32]>(&rb[(ch + 1) & 1][0]));
                    const float* r = (ch == 0) ? s0 : rb[ch & 1];
                    uint32_t pw[16];
                    if (full) {
                        // three pairs in eight on the FMA pipe (packed polynomial), the rest on the exp unit
                        const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(neg_mc, neg_mc);
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            const uint64_t xx = f2_fma(f2_pack(r[2 * e], r[2 * e + 1]), c2, nm2);
                            float p0, p1;
                            if ((e & 7) >= 5) {
                                exp2_poly2(xx, p0, p1);
                            } else {
                                float x0, x1;
                                f2_unpack(xx, x0, x1);
                                p0 = ex2_approx(x0);
                                p1 = ex2_approx(x1);
                            }
                            pw[e] = pack_bf16x2(p0, p1);
                            l2[e & 1] = f2_add(l2[e & 1], f2_pack(p0, p1));
                        }
                    } else {
#pragma unroll
                        const int kq = (int)((kv4 >> (8 * ch)) & 255u);  // chunk ch is quarter ch
                        for (int e = 0; e < 16; ++e) {
                            const float p0 = (2 * e < kq) ? ex2_approx(fmaf(r[2 * e], c, neg_mc)) : 0.0f;
                            const float p1 = (2 * e + 1 < kq) ? ex2_approx(fmaf(r[2 * e + 1], c, neg_mc)) : 0.0f;
                            pw[e] = pack_bf16x2(p0, p1);
                            l2[e & 1] = f2_add(l2[e & 1], f2_pack(p0, p1));
                        }
                    }
                    tmem_st16(tS + lane_off + ch * 16u, pw);
                    if (ch < 3) tmem_wait_ld_regs(rb[(ch + 1) & 1]);
                }
                float la, lb, lc, ld;
                f2_unpack(l2[0], la, lb);
                f2_unpack(l2[1], lc, ld);
                l_run = l_run * alpha + ((la + lb) + (lc + ld));
                // O (complete: this tile's S was computed after the previous P V finished) is rescaled before the
                // P V of this tile may start.
                if (t > 0 && __any_sync(0xffffffffu, need)) {
#pragma unroll
                    for (int ch = 0; ch < 4; ++ch) {
                        uint32_t ov[32];
                        tmem_ld32(tO + lane_off + ch * 32u, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                        tmem_st32(tO + lane_off + ch * 32u, ov);
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(BAR(L_P_FULL));
            }
            if (!ok) break;
            // Epilogue: O / l -> bf16 rows and lse; O's columns are then free for the next item.
            if (!(ok = wait_bounded_warp(BAR(L_PV_DONE), (n_pv + it.tiles - 1) & 1u, lim))) break;
            n_pv += it.tiles;
            tc_fence_after();
            const float inv_l = 1.0f / l_run;
            const float lse2 = m_raw * c + lg2_approx(l_run);
            uint4* dst = reinterpret_cast<uint4*>(a.o + grow * kTcDim);
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
                uint32_t ov[32];
                tmem_ld32(tO + lane_off + ch * 32u, ov);
                tmem_wait_ld();
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(ov[q4 * 8 + 0]) * inv_l, __uint_as_float(ov[q4 * 8 + 1]) * inv_l);
                    v.y = pack_bf16x2(__uint_as_float(ov[q4 * 8 + 2]) * inv_l, __uint_as_float(ov[q4 * 8 + 3]) * inv_l);
                    v.z = pack_bf16x2(__uint_as_float(ov[q4 * 8 + 4]) * inv_l, __uint_as_float(ov[q4 * 8 + 5]) * inv_l);
                    v.w = pack_bf16x2(__uint_as_float(ov[q4 * 8 + 6]) * inv_l, __uint_as_float(ov[q4 * 8 + 7]) * inv_l);
                    dst[ch * 4 + q4] = v;
                }
            }
            tc_fence_before();
            mbar_arrive(BAR(L_O_FREE));
            if (a.lse) a.lse[grow] = lse2 * 0.6931471805599453f;

            if (WITH_MASS) {
                // Mass phase: p = 2^(s*c - lse2) summed per key block (SUB blocks per tile) for real rows and keys.
                // The per-warp partials are flushed to M every kMaxMassBlocks blocks: all 128 threads arrive on PART
                // once their partials are written, combine the four warps in fixed order, then arrive on PART2 before
                // the buffer is written again.
                const bool qvalid = qrow < a.N;
                const float neg_lse2 = qvalid ? -lse2 : 0.0f;
                const uint64_t c2 = f2_pack(c, c), nl2 = f2_pack(neg_lse2, neg_lse2);
                const float inv_rows = 1.0f / (float)min(kTcRows, a.N - it.qb * kTcRows);
                float* mrow = a.mass + (size_t)it.id * a.nkb;
                constexpr int kChunkTiles = kMaxMassBlocks / SUB;
                for (int t0 = 0; ok && t0 < a.nk; t0 += kChunkTiles) {
                    const int t1 = min(a.nk, t0 + kChunkTiles);
                    for (int t = t0; t < t1; ++t) {
                        if (!(ok = wait_bounded_warp(BAR(L_S_FULL), n_s & 1u, lim))) break;
                        ++n_s;
                        tc_fence_after();
                        float s[128];
#pragma unroll
                        for (int ch = 0; ch < 4; ++ch)
                            tmem_ld32(tS + lane_off + ch * 32u, *reinterpret_cast<uint32_t(*)[32]>(&s[ch * 32]));
                        tmem_wait_ld();
                        tc_fence_before();
                        mbar_arrive(BAR(L_S_FREE));
                        const int kvalid = a.N - t * kTcRows;
                        // acc[2 * g + (e & 1)]: two packed accumulators per 32-key quarter g
                        uint64_t acc[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[i] = f2_pack(0.f, 0.f);
                        if (kvalid >= kTcRows) {
                            // seven pairs in sixteen on the FMA pipe (packed polynomial), the rest on the exp unit
#pragma unroll
                            for (int e = 0; e < 64; ++e) {
                                const uint64_t xx = f2_fma(f2_pack(s[2 * e], s[2 * e + 1]), c2, nl2);
                                float p0, p1;
                                if ((e & 15) >= 9) {
                                    exp2_poly2(xx, p0, p1);
                                } else {
                                    float x0, x1;
                                    f2_unpack(xx, x0, x1);
                                    p0 = ex2_approx(x0);
                                    p1 = ex2_approx(x1);
                                }
                                acc[2 * (e >> 4) + (e & 1)] = f2_add(acc[2 * (e >> 4) + (e & 1)], f2_pack(p0, p1));
                            }
                        } else {
#pragma unroll
                            for (int e = 0; e < 64; ++e) {
                                const float p0 = (2 * e < kvalid) ? ex2_approx(fmaf(s[2 * e], c, neg_lse2)) : 0.0f;
                                const float p1 = (2 * e + 1 < kvalid) ? ex2_approx(fmaf(s[2 * e + 1], c, neg_lse2)) : 0.0f;
                                acc[2 * (e >> 4) + (e & 1)] = f2_add(acc[2 * (e >> 4) + (e & 1)], f2_pack(p0, p1));
                            }
                        }
                        float q[4];
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            float x0, x1, x2, x3;
                            f2_unpack(acc[2 * g], x0, x1);
                            f2_unpack(acc[2 * g + 1], x2, x3);
                            q[g] = qvalid ? (x0 + x1) + (x2 + x3) : 0.0f;
                        }
                        if (SUB == 1) {
                            float sum = (q[0] + q[1]) + (q[2] + q[3]);
#pragma unroll
                            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                            if (lane == 0) part[wl * kMaxMassBlocks + (t - t0)] = sum;
                        } else {
#pragma unroll
                            for (int g = 0; g < 4; ++g) {
#pragma unroll
                                for (int o = 16; o > 0; o >>= 1) q[g] += __shfl_xor_sync(0xffffffffu, q[g], o);
                            }
                            if (lane < 4) {
                                const float mine = lane == 0 ? q[0] : (lane == 1 ? q[1] : (lane == 2 ? q[2] : q[3]));
                                part[wl * kMaxMassBlocks + (t - t0) * SUB + lane] = mine;
                            }
                        }
                    }
                    if (!ok) break;
                    mbar_arrive(BAR(L_PART));
                    if (!(ok = wait_bounded_warp(BAR(L_PART), n_chunks & 1u, lim))) break;
                    const int b0 = t0 * SUB, b1 = min(a.nkb, t1 * SUB);
                    for (int jj = b0 + row; jj < b1; jj += 128) {
                        const int o = jj - b0;
                        mrow[jj] = ((part[o] + part[kMaxMassBlocks + o]) +
                                    (part[2 * kMaxMassBlocks + o] + part[3 * kMaxMassBlocks + o])) * inv_rows;
                    }
                    mbar_arrive(BAR(L_PART2));
                    if (!(ok = wait_bounded_warp(BAR(L_PART2), n_chunks & 1u, lim))) break;
                    ++n_chunks;
                }
                if (!ok) break;
            }
            ++n_items;
        }
    }
    // Teardown: every role has left its loop (normally or after a bounded wait ran out).
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace losa
