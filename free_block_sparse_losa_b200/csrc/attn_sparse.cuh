// Sparse-step tensor-core kernel (bf16, head_dim 128, 128-row query blocks): attn_sparse_kernel<SUB>.
//
// Online-softmax attention of each work item = (head, 128-row query block) against its retained list of key blocks
// (LoSA page, Methodology Summary, "Sparse attention with a frozen pattern": the softmax denominator covers the
// retained keys only), SUB key blocks per 128-key tile (1 for C = 128, 4 for C = 32). Writes O (bf16) and the row
// log-sum-exp.
//
// One persistent CTA per SM walks one stream of items (CTA b takes rounds r = 0, 1, 2, ...: item r*G + b for even r,
// r*G + G - 1 - b for odd r, a snake over the longest-first work order). The tiles of all its items form one
// sequence n = 0, 1, 2, ... through a software pipeline:
//   warp 3   reads the work order and the lists ahead of time into a four-entry ring of item records in shared
//            memory (head, query block, list start and length, tiles, key validity of the first tile), so that no
//            role waits on dependent global loads at an item boundary.
//   warp 0   TMA: Q double-buffered (the next item's Q arrives during this item), K in a three-stage ring.
//   warp 2   TMA: V in a two-stage ring (a V slot waiting for its P V never holds back K), and the O stores.
//            In both producer warps every TMA box of a tile is issued by its own lane: one thread's TMA loads are
//            served one after another at about 30 bytes per clock, which would cap a 32 KB tile at ~1100 clocks.
//   warp 1   MMA: per tile S_n = Q K^T (128 x 128, N = 128, both operands in shared memory; the item's Q slot is
//            released after its last Q K^T) into S buffer n & 1, and O += P V of tile n - 1 (P from TMEM buffer
//            (n - 1) & 1).
//   warps 4..11  softmax in two warpgroups that split each tile's keys (warps 4..7 keys 0..63, warps 8..11 keys
//            64..127; thread t owns query row t = TMEM lane t). A group reads the whole of S_n (the other half only
//            for its row max, which then needs no exchange: the max is exact, so both groups agree on it). The groups share one running max, keep their own partial sums and write their
//            half of P.
// TMEM: S_0 columns 0..127, S_1 128..255, O 256..383, P_0 384..447, P_1 448..511 (bf16 pairs). With two S buffers
// the Q K^T of tile n + 1 runs while the softmax still reads tile n. Buffer n & 1 was last read for tile n - 2, and
// the MMA issuer has waited for that tile's P (stored after the read) before it issues Q K^T of tile n, so no separate
// release is needed. With two P buffers the softmax stores P_n while P V of tile n - 1 still runs: P buffer n & 1 was
// last read by P V of tile n - 2, which the in-order tensor pipe completed before S_n. O is rescaled in place only
// when a row's running max grows by more than 2^8 (the final division by the sum taken against the same reference
// keeps this exact), after P V of tile n - 1; each group rescales its own 64 columns of O.
// Registers: the producer / MMA warpgroup drops to 56 per thread and the softmax warpgroups rise to 224 (setmaxnreg).
// Epilogue, deferred until the next item's first P is stored (the item's last P V has usually completed by then):
// the two groups add their partial row sums through shared memory (a group writes its next sums only after both
// have read these: it first waits for its next item's last P V, and that item's first P V waited for both groups to
// release O after reading them), write O / l in bf16, 128-byte swizzled, into the V slot the item's last P V has
// released, and go on. The V producer stores the two 64-column boxes with TMA before it
// refills that slot. Row stores from registers would put 32 rows into every warp-wide store; waiting for the TMA
// store would stall the softmax warps.
// Every wait is bounded in time (LOSA_ERR_TIMEOUT in the device error word, then a clean exit).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "attn_tc.cuh"

namespace losa {

constexpr uint32_t kSpQ = 0;                              // 2 Q tiles
constexpr uint32_t kSpK = 2 * kTileBytes;                 // 3 K tiles
constexpr uint32_t kSpV = 5 * kTileBytes;                 // 2 V tiles (the second use: O staging)
constexpr uint32_t kSpBar = 7 * kTileBytes;               // 48 barrier slots; the last holds the TMEM address
constexpr uint32_t kSpRing = kSpBar + 384;                // 4 item records of 32 bytes
constexpr uint32_t kSpXsum = kSpRing + 4 * 32;            // [2 groups][128 rows] (exact, rounded) partial row sums
constexpr uint32_t kSpSmem = kSpXsum + 2 * 128 * 8;       // 231936 bytes: needs a 1024-aligned dynamic base
constexpr int kSpKStages = 3;
constexpr uint32_t kSpRingSlots = 4;
static_assert(kSpSmem <= 232448, "shared memory");

enum : uint32_t {
    S_Q_FULL0 = 0, S_Q_EMPTY0 = 2, S_K_FULL0 = 4, S_K_EMPTY0 = 7, S_V_FULL0 = 10, S_V_EMPTY0 = 12, S_S_FULL0 = 14,
    S_P_FULL0 = 16, S_PV_DONE0 = 18, S_SUM_X = 20, S_O_FREE, S_STAGED0, S_IT_FULL0 = S_STAGED0 + 2,
    S_IT_EMPTY0 = S_IT_FULL0 + kSpRingSlots, S_MMA_DONE = S_IT_EMPTY0 + kSpRingSlots, S_COUNT
};
constexpr int kSpThreads = 384;  // 12 warps: 0 Q/K TMA, 1 MMA, 2 V TMA, 3 work order, 4..11 softmax
static_assert(S_COUNT <= 47, "barrier slots");

struct SpItem {
    int id, h, qb, begin, count, tiles;
    uint32_t kv4;  // real keys per 32-key quarter of the first tile
    int end;       // 1: past the end of this CTA's work
};
static_assert(sizeof(SpItem) == 32, "item record");

// List entry e of an item as a block index (clamped; out-of-range entries are reported by the work-order reader).
__device__ __forceinline__ int sp_block(const TcArgs& a, const SpItem& it, int e) {
    const int j = a.kv_idx[it.begin + e];
    return (j < 0) ? 0 : (j >= a.nkb ? a.nkb - 1 : j);
}

// Loads tile t of an item into dst, one 16 KB (C = 128) or 4 KB (C = 32) box per lane; lane 0 posts the expected
// bytes first. Called by all lanes of the producer warp.
template <int SUB>
__device__ __forceinline__ void sp_load_tile(const TcArgs& a, const SpItem& it, int t, uint32_t dst,
                                             const CUtensorMap* tm, const CUtensorMap* tm32, uint32_t bar,
                                             uint64_t pol, uint32_t lane) {
    if (lane == 0) mbar_arrive_expect_tx(bar, kTileBytes);
    __syncwarp();
    if (SUB == 1) {
        if (lane < 2) {
            const int32_t krow = it.h * a.Np + sp_block(a, it, t) * kTcRows;
            tma_load_2d_hint(dst + lane * kBoxBytes, tm, 64 * (int)lane, krow, bar, pol);
        }
    } else if (lane < 2 * SUB) {
        const int g = (int)(lane >> 1), hx = (int)(lane & 1u);
        // a missing quarter reloads the tile's first block (finite data, masked to P = 0)
        const int e = SUB * t + g < it.count ? SUB * t + g : SUB * t;
        const int32_t r32 = it.h * a.Np + sp_block(a, it, e) * 32;
        tma_load_2d_hint(dst + hx * kBoxBytes + g * 4096u, tm32, 64 * hx, r32, bar, pol);
    }
}

// Real keys in each 32-key quarter of tile t of a list item, packed 8 bits per quarter. A quarter with no list entry
// (the tail of a C = 32 list) has none; the ragged end of the sequence cuts the last block.
template <int SUB>
__device__ __forceinline__ uint32_t sp_quarter_keys(const TcArgs& a, const SpItem& it, int t) {
    uint32_t kv = 0;
    if (SUB == 1) {
        const int kvalid = a.N - sp_block(a, it, t) * 128;
#pragma unroll
        for (int g = 0; g < 4; ++g) kv |= (uint32_t)min(32, max(0, kvalid - 32 * g)) << (8 * g);
    } else {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            const int e = SUB * t + g;
            if (e < it.count) kv |= (uint32_t)min(32, max(0, a.N - sp_block(a, it, e) * 32)) << (8 * g);
        }
    }
    return kv;
}

template <int SUB>
__global__ void __launch_bounds__(kSpThreads, 1)
    attn_sparse_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmK32,
                       const __grid_constant__ CUtensorMap tmV32, const __grid_constant__ CUtensorMap tmO,
                       const TcArgs a) {
    extern __shared__ __align__(1024) uint8_t sp_smem[];
    const uint32_t base = smem_addr(sp_smem);
    if (base & 1023u) {  // the 128-byte-swizzled tiles need a 1024-aligned base; report instead of overrunning
        if (threadIdx.x == 0) atomicOr(&g_device_error, kDevErrBadData);
        return;
    }
    const uint32_t bar0 = base + kSpBar;
    auto BAR = [&](uint32_t s) { return bar0 + 8u * s; };
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(sp_smem + kSpBar + 47 * 8);
    SpItem* const ring = reinterpret_cast<SpItem*>(sp_smem + kSpRing);
    float2* const xsum = reinterpret_cast<float2*>(sp_smem + kSpXsum);  // [2 groups][128 rows]: exact, rounded

    const int warp = threadIdx.x >> 5;
    const uint32_t lane = lane_id();
    if (threadIdx.x == 0) {
        for (uint32_t s = 0; s < S_COUNT; ++s) {
            uint32_t cnt = 1;
            if (s == S_P_FULL0 || s == S_P_FULL0 + 1 || s == S_SUM_X || s == S_O_FREE || s == S_STAGED0 ||
                s == S_STAGED0 + 1)
                cnt = 256;
            else if (s >= S_IT_EMPTY0 && s < S_IT_EMPTY0 + kSpRingSlots)
                cnt = 3 + 256;  // Q/K producer, V producer, MMA issuer, 256 softmax threads
            mbar_init(BAR(s), cnt);
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
        tma_prefetch_desc(&tmO);
        if (SUB > 1) {
            tma_prefetch_desc(&tmK32);
            tma_prefetch_desc(&tmV32);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
    const uint32_t tS = tmem, tO = tmem + 256u, tP = tmem + 384u;
    const unsigned long long lim = a.wait_limit_ns;

    // Item record of round r from the ring (false on a timeout). mode 0: one thread waits and arrives; 1: the whole
    // warp waits and every lane arrives; 2: the whole warp waits and lane 0 arrives for it.
    auto next_item = [&](int r, SpItem& it, int mode) -> bool {
        const uint32_t sl = (uint32_t)r & (kSpRingSlots - 1);
        const uint32_t par = ((uint32_t)r / kSpRingSlots) & 1u;
        const bool ok = mode ? wait_bounded_warp(BAR(S_IT_FULL0 + sl), par, lim)
                             : wait_bounded(BAR(S_IT_FULL0 + sl), par, lim);
        if (!ok) return false;
        const volatile SpItem* src = &ring[sl];
        it.id = src->id;
        it.h = src->h;
        it.qb = src->qb;
        it.begin = src->begin;
        it.count = src->count;
        it.tiles = src->tiles;
        it.kv4 = src->kv4;
        it.end = src->end;
        if (mode != 2 || lane == 0) mbar_arrive(BAR(S_IT_EMPTY0 + sl));
        return true;
    };

    // Registers: the producer / MMA warpgroup needs few, the softmax warpgroups many. Each warpgroup reaches one
    // setmaxnreg; the split uses exactly the 384 x 168 registers the block is launched with (128 x 56 + 256 x 224).
    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
        if (warp == 3) {
            // ------------------------------------------------------------------------- work-order reader (lane 0)
            if (lane == 0) {
                uint32_t bad = 0;
                for (int r = 0;; ++r) {
                    const uint32_t sl = (uint32_t)r & (kSpRingSlots - 1);
                    if (!wait_bounded(BAR(S_IT_EMPTY0 + sl), (((uint32_t)r / kSpRingSlots) & 1u) ^ 1u, lim)) break;
                    ItemInfo ii;
                    const bool has = item_of_round(a, r, ii);
                    SpItem it;
                    it.end = has ? 0 : 1;
                    it.id = has ? ii.id : 0;
                    it.h = has ? ii.h : 0;
                    it.qb = has ? ii.qb : 0;
                    it.begin = has ? ii.begin : 0;
                    it.count = has ? ii.count : 0;
                    it.tiles = has ? ii.tiles : 0;
                    it.kv4 = 0;
                    if (has) {
                        if (it.count <= 0) bad = 1;
                        for (int e = 0; e < it.count; ++e) {
                            const int j = a.kv_idx[it.begin + e];
                            bad |= (j < 0 || j >= a.nkb) ? 1u : 0u;
                        }
                        if (it.count > 0) it.kv4 = sp_quarter_keys<SUB>(a, it, 0);
                    }
                    volatile SpItem* dst = &ring[sl];
                    dst->id = it.id;
                    dst->h = it.h;
                    dst->qb = it.qb;
                    dst->begin = it.begin;
                    dst->count = it.count;
                    dst->tiles = it.tiles;
                    dst->kv4 = it.kv4;
                    dst->end = it.end;
                    mbar_arrive(BAR(S_IT_FULL0 + sl));
                    if (!has) break;
                }
                if (bad) atomicOr(&g_device_error, kDevErrBadData);
            }
            __syncwarp();
        } else if (warp == 0) {
            // ----------------------------------------------------------------- TMA producer: Q and K (whole warp)
            const uint64_t pol_q = l2_policy_evict_first();
            const uint64_t pol_kv = l2_policy_evict_last();
            uint32_t nq = 0, nk = 0;
            bool ok = true;
            SpItem it;
            for (int r = 0; ok && (ok = next_item(r, it, 2)) && !it.end; ++r) {
                if (it.count <= 0) continue;
                const uint32_t qs = nq & 1u;
                if (!(ok = wait_bounded_warp(BAR(S_Q_EMPTY0 + qs), ((nq >> 1) & 1u) ^ 1u, lim))) break;
                const int32_t qrow = it.h * a.Np + it.qb * kTcRows;
                if (lane == 0) mbar_arrive_expect_tx(BAR(S_Q_FULL0 + qs), kTileBytes);
                __syncwarp();
                if (lane < 2)
                    tma_load_2d_hint(base + kSpQ + qs * kTileBytes + lane * kBoxBytes, &tmQ, 64 * (int)lane, qrow,
                                     BAR(S_Q_FULL0 + qs), pol_q);
                ++nq;
                for (int t = 0; t < it.tiles; ++t) {
                    const uint32_t ks = nk % kSpKStages;
                    if (!(ok = wait_bounded_warp(BAR(S_K_EMPTY0 + ks), ((nk / kSpKStages) & 1u) ^ 1u, lim))) break;
                    sp_load_tile<SUB>(a, it, t, base + kSpK + ks * kTileBytes, &tmK, &tmK32, BAR(S_K_FULL0 + ks), pol_kv,
                                      lane);
                    ++nk;
                }
            }
            for (uint32_t i = 1; i <= 2 && i <= nq; ++i) {
                const uint32_t n = nq - i;
                wait_bounded(BAR(S_Q_FULL0 + (n & 1u)), (n >> 1) & 1u, kDrainLimitNs);
            }
            for (uint32_t i = 1; i <= kSpKStages && i <= nk; ++i) {
                const uint32_t n = nk - i;
                wait_bounded(BAR(S_K_FULL0 + n % kSpKStages), (n / kSpKStages) & 1u, kDrainLimitNs);
            }
            __syncwarp();
        } else if (warp == 2) {
            // ------------------------------------------------------------- TMA producer: V and the O stores (whole warp)
            // A V slot whose last tile closed an item holds that item's staged O when it is wanted again: its two
            // 64-column boxes are stored (one lane each) and read out before the slot is refilled. Other slots come back
            // through V_EMPTY from the MMA.
            const uint64_t pol_kv = l2_policy_evict_last();
            uint32_t nv = 0;
            uint32_t empty_cnt[2] = {0u, 0u}, staged_cnt[2] = {0u, 0u};
            bool fin[2] = {false, false};
            int32_t fin_row[2] = {0, 0};
            bool ok = true;
            auto flush = [&](uint32_t sl) -> bool {
                if (!wait_bounded_warp(BAR(S_STAGED0 + sl), staged_cnt[sl] & 1u, lim)) return false;
                ++staged_cnt[sl];
                if (lane < 2) {
                    tma_store_2d(&tmO, base + kSpV + sl * kTileBytes + lane * kBoxBytes, 64 * (int)lane, fin_row[sl]);
                    bulk_commit_group();
                    bulk_wait_read_all();
                }
                __syncwarp();
                fin[sl] = false;
                return true;
            };
            SpItem it;
            for (int r = 0; ok && (ok = next_item(r, it, 2)) && !it.end; ++r) {
                if (it.count <= 0) continue;
                for (int t = 0; t < it.tiles; ++t) {
                    const uint32_t vs = nv & 1u;
                    if (nv >= 2) {
                        if (fin[vs]) {
                            if (!(ok = flush(vs))) break;
                        } else {
                            if (!(ok = wait_bounded_warp(BAR(S_V_EMPTY0 + vs), empty_cnt[vs] & 1u, lim))) break;
                            ++empty_cnt[vs];
                        }
                    }
                    sp_load_tile<SUB>(a, it, t, base + kSpV + vs * kTileBytes, &tmV, &tmV32, BAR(S_V_FULL0 + vs), pol_kv,
                                      lane);
                    fin[vs] = (t == it.tiles - 1);
                    fin_row[vs] = it.h * a.Np + it.qb * kTcRows;
                    ++nv;
                }
            }
            // the last one or two items' O, oldest slot first
            for (uint32_t k = 0; ok && k < 2; ++k) {
                const uint32_t sl = (nv + k) & 1u;
                if (fin[sl]) ok = flush(sl);
            }
            if (lane < 2) bulk_wait_all();  // the O stores have landed before the CTA exits
            for (uint32_t i = 1; i <= 2 && i <= nv; ++i) {
                const uint32_t n = nv - i;
                wait_bounded(BAR(S_V_FULL0 + (n & 1u)), (n >> 1) & 1u, kDrainLimitNs);
            }
            __syncwarp();
        } else if (warp == 1) {
            // ------------------------------------------------------------------------------------- MMA issuer
            if (lane == 0) {
                constexpr uint32_t kIdQK = idesc_bf16_f32(128, 128, false, false);
                constexpr uint32_t kIdPV = idesc_bf16_f32(128, 128, false, true);
                constexpr uint32_t kSlot = kTileBytes >> 4;  // descriptor step between ring slots
                const uint64_t dQ0 = smem_desc(base + kSpQ, 16, 1024), dK0 = smem_desc(base + kSpK, 16, 1024);
                const uint64_t dV0 = smem_desc(base + kSpV, kBoxBytes, 1024);
                uint32_t nq = 0, n = 0, n_items = 0;
                // the tile whose P V is still to be issued: sequence number, first / last tile of its item, item index
                bool pend = false, pend_first = false, pend_last = false;
                uint32_t pend_n = 0, pend_item = 0;
                bool ok = true;
                auto issue_pv = [&]() -> bool {
                    const uint32_t b = pend_n & 1u;
                    if (!wait_bounded(BAR(S_P_FULL0 + b), (pend_n >> 1) & 1u, lim)) return false;
                    if (!wait_bounded(BAR(S_V_FULL0 + b), (pend_n >> 1) & 1u, lim)) return false;
                    if (pend_first && pend_item > 0 && !wait_bounded(BAR(S_O_FREE), (pend_item - 1) & 1u, lim))
                        return false;
                    tc_fence_after();
                    const uint64_t dV = dV0 + b * kSlot;
    #pragma unroll
                    for (uint32_t kk = 0; kk < 8; ++kk)
                        tc_mma_ts(tO, tP + b * 64u + kk * 8u, dV + kk * 128u, kIdPV, (pend_first && kk == 0) ? 0u : 1u);
                    // an item's last V slot comes back through the O staging: the V producer stores the item's O from it
                    // before refilling it
                    if (!pend_last) tc_commit(BAR(S_V_EMPTY0 + b));
                    tc_commit(BAR(S_PV_DONE0 + b));
                    pend = false;
                    return true;
                };
                SpItem it;
                for (int r = 0; ok && (ok = next_item(r, it, 0)) && !it.end; ++r) {
                    if (it.count <= 0) continue;
                    const uint32_t qs = nq & 1u;
                    if (!(ok = wait_bounded(BAR(S_Q_FULL0 + qs), (nq >> 1) & 1u, lim))) break;
                    ++nq;
                    const uint64_t dQ = dQ0 + qs * kSlot;
                    for (int t = 0; t < it.tiles; ++t, ++n) {
                        const uint32_t ks = n % kSpKStages;
                        const uint32_t b = n & 1u;
                        // S buffer b was read for tile n - 2, whose P this thread has already waited for
                        if (!(ok = wait_bounded(BAR(S_K_FULL0 + ks), (n / kSpKStages) & 1u, lim))) break;
                        tc_fence_after();
                        const uint64_t dK = dK0 + ks * kSlot;
    #pragma unroll
                        for (uint32_t kk = 0; kk < 8; ++kk) {
                            const uint32_t off = ((kk >> 2) * kBoxBytes + (kk & 3u) * 32u) >> 4;
                            tc_mma_ss(tS + b * 128u, dQ + off, dK + off, kIdQK, kk ? 1u : 0u);
                        }
                        tc_commit(BAR(S_S_FULL0 + b));
                        tc_commit(BAR(S_K_EMPTY0 + ks));
                        if (t == it.tiles - 1) tc_commit(BAR(S_Q_EMPTY0 + qs));  // the item's last read of its Q slot
                        // the previous tile's P V goes behind this QK^T in the tensor pipe
                        if (pend && !(ok = issue_pv())) break;
                        pend = true;
                        pend_first = (t == 0);
                        pend_last = (t == it.tiles - 1);
                        pend_n = n;
                        pend_item = n_items;
                    }
                    ++n_items;
                }
                if (ok && pend) issue_pv();
                tc_commit(BAR(S_MMA_DONE));
                wait_bounded(BAR(S_MMA_DONE), 0, kDrainLimitNs);
            }
            __syncwarp();
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory");
        // --------------------------------------------------------------------------- softmax warpgroups
        const uint32_t grp = (uint32_t)(warp - 4) >> 2;  // keys 64 * grp .. 64 * grp + 63 of every tile
        const uint32_t wl = (uint32_t)warp & 3u;
        const int row = (int)(wl * 32u + lane);
        const uint32_t lane_off = (wl * 32u) << 16;
        const float c = a.scale_log2;
        uint32_t n = 0, n_epi = 0;
        bool ok = true;
        // An item's epilogue waits until the next item's first P is stored: by then the item's last P V has
        // completed, where an immediate epilogue would sit waiting for it.
        bool pend = false;
        size_t pd_grow = 0;
        float pd_m = 0.0f, pd_l = 0.0f, pd_lr = 0.0f;
        uint32_t pd_nl = 0;
        auto epilogue = [&]() -> bool {
            const uint32_t bl = pd_nl & 1u;
            if (!wait_bounded_warp(BAR(S_PV_DONE0 + bl), (pd_nl >> 1) & 1u, lim)) return false;  // the item's last P V
            // Full row sum: each group writes its partial sums into shared memory. Both groups read the previous
            // epilogue's sums before they released O; the wait above covers this item's first P V, which waited for
            // that release.
            xsum[grp * 128u + (uint32_t)row] = make_float2(pd_l, pd_lr);
            mbar_arrive(BAR(S_SUM_X));
            if (!wait_bounded_warp(BAR(S_SUM_X), n_epi & 1u, lim)) return false;
            const float2 other = xsum[(grp ^ 1u) * 128u + (uint32_t)row];
            const float l_all = pd_l + other.x;
            const float inv_l = 1.0f / (pd_lr + other.y);
            tc_fence_after();
            uint32_t ov[2][32];
            tmem_ld32(tO + grp * 64u + lane_off, ov[0]);
            tmem_ld32(tO + grp * 64u + lane_off + 32u, ov[1]);
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(BAR(S_O_FREE));  // the next item's first P V may overwrite O
            // O / l in bf16, 128-byte swizzled, into this group's box of the released V slot
            const uint32_t stage = base + kSpV + bl * kTileBytes + grp * kBoxBytes;
    #pragma unroll
            for (int ch = 0; ch < 2; ++ch)
    #pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const uint32_t j = (uint32_t)(ch * 4 + q4);  // 16-byte chunk of this row's 128 bytes
                    uint32_t w[4];
    #pragma unroll
                    for (int k2 = 0; k2 < 4; ++k2)
                        w[k2] = pack_bf16x2(__uint_as_float(ov[ch][q4 * 8 + 2 * k2]) * inv_l,
                                            __uint_as_float(ov[ch][q4 * 8 + 2 * k2 + 1]) * inv_l);
                    st_shared_v4(stage + (uint32_t)row * 128u + ((j ^ ((uint32_t)row & 7u)) << 4), w[0], w[1], w[2],
                                 w[3]);
                }
            fence_proxy_async_smem();
            mbar_arrive(BAR(S_STAGED0 + bl));  // the V producer stores the slot before it loads into it again
            if (a.lse && grp == 0) a.lse[pd_grow] = (pd_m * c + lg2_approx(l_all)) * 0.6931471805599453f;
            ++n_epi;
            return true;
        };
        SpItem it;
        for (int r = 0; ok && (ok = next_item(r, it, 1)) && !it.end; ++r) {
            if (it.count <= 0) continue;
            const size_t grow = (size_t)it.h * a.Np + it.qb * kTcRows + row;
            float m_raw = -INFINITY, l_run = 0.0f, lr_run = 0.0f;  // exact and bf16-rounded row sums
            uint32_t kvn = it.kv4;
            for (int t = 0; t < it.tiles; ++t, ++n) {
                const uint32_t kv4 = kvn;  // real keys per 32-column quarter of this tile
                if (t + 1 < it.tiles) kvn = sp_quarter_keys<SUB>(a, it, t + 1);  // prefetched one tile ahead
                const uint32_t kq0 = (kv4 >> (16 * grp)) & 255u, kq1 = (kv4 >> (16 * grp + 8)) & 255u;
                const bool full = kq0 == 32u && kq1 == 32u;
                const uint32_t b = n & 1u;
                const uint32_t tSb = tS + b * 128u;
                if (!(ok = wait_bounded_warp(BAR(S_S_FULL0 + b), (n >> 1) & 1u, lim))) break;
                tc_fence_after();
                // The row max over the whole tile without a cross-group exchange: the other group's 64 columns are
                // read first and only their maximum is kept (max is exact, so both groups get the same value).
                float omax;
                {
                    const uint32_t oq0 = (kv4 >> (16 * (grp ^ 1u))) & 255u, oq1 = (kv4 >> (16 * (grp ^ 1u) + 8)) & 255u;
                    float o[64];
                    tmem_ld32(tSb + (grp ^ 1u) * 64u + lane_off, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
                    tmem_ld32(tSb + (grp ^ 1u) * 64u + lane_off + 32u, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
                    tmem_wait_ld();
                    if (oq0 != 32u || oq1 != 32u) {
    #pragma unroll
                        for (int cc = 0; cc < 64; ++cc)
                            if ((uint32_t)(cc & 31) >= (cc < 32 ? oq0 : oq1)) o[cc] = -INFINITY;
                    }
                    float mx[8];
    #pragma unroll
                    for (int e = 0; e < 8; ++e) mx[e] = fmax3(o[e], o[8 + e], o[16 + e]);
    #pragma unroll
                    for (int cc = 24; cc < 64; cc += 16)
    #pragma unroll
                        for (int e = 0; e < 8; ++e) mx[e] = fmax3(mx[e], o[cc + e], o[cc + 8 + e]);
                    omax = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], fmax3(mx[5], mx[6], mx[7])));
                }
                float s[64];
                tmem_ld32(tSb + grp * 64u + lane_off, *reinterpret_cast<uint32_t(*)[32]>(&s[0]));
                tmem_ld32(tSb + grp * 64u + lane_off + 32u, *reinterpret_cast<uint32_t(*)[32]>(&s[32]));
                tmem_wait_ld();
                if (!full) {  // keys past the sequence end, or quarters without a listed block, do not exist
    #pragma unroll
                    for (int cc = 0; cc < 64; ++cc)
                        if ((uint32_t)(cc & 31) >= (cc < 32 ? kq0 : kq1)) s[cc] = -INFINITY;
                }
                float tmax;
                {
                    float mx[8];
    #pragma unroll
                    for (int e = 0; e < 8; ++e) mx[e] = fmax3(s[e], s[8 + e], s[16 + e]);
    #pragma unroll
                    for (int cc = 24; cc < 64; cc += 16)
    #pragma unroll
                        for (int e = 0; e < 8; ++e) mx[e] = fmax3(mx[e], s[cc + e], s[cc + 8 + e]);
                    tmax = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], fmax3(mx[5], mx[6], mx[7])));
                }
                tmax = fmaxf(tmax, omax);  // the tile max over all 128 columns
                // Reference max: raised only when the tile max exceeds it by more than 2^8 in the exp2 domain. A row
                // that has seen no real key yet keeps a finite reference so that its weights are exact zeros.
                const bool need = (t == 0) || (tmax - m_raw) * c > 8.0f;
                const float alpha = (t > 0 && need && tmax != -INFINITY) ? ex2_approx((m_raw - tmax) * c) : 1.0f;
                if (need) m_raw = (tmax == -INFINITY) ? (t == 0 ? 0.0f : m_raw) : tmax;
                const float neg_mc = -m_raw * c;
                uint32_t pw[32];
                uint64_t l2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)}, r2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
                if (full) {
                    const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(neg_mc, neg_mc);
    #pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const uint64_t xx = f2_fma(f2_pack(s[2 * e], s[2 * e + 1]), c2, nm2);
                        float x0, x1;
                        f2_unpack(xx, x0, x1);
                        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                        pw[e] = pack_bf16x2(p0, p1);
                        l2[e & 1] = f2_add(l2[e & 1], f2_pack(p0, p1));
                        r2[e & 1] = f2_add(r2[e & 1], bf16x2_to_f2(pw[e]));
                    }
                } else {
    #pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const float p0 = (s[2 * e] != -INFINITY) ? ex2_approx(fmaf(s[2 * e], c, neg_mc)) : 0.0f;
                        const float p1 = (s[2 * e + 1] != -INFINITY) ? ex2_approx(fmaf(s[2 * e + 1], c, neg_mc)) : 0.0f;
                        pw[e] = pack_bf16x2(p0, p1);
                        l2[e & 1] = f2_add(l2[e & 1], f2_pack(p0, p1));
                        r2[e & 1] = f2_add(r2[e & 1], bf16x2_to_f2(pw[e]));
                    }
                }
                float la, lb, lc, ld;
                f2_unpack(l2[0], la, lb);
                f2_unpack(l2[1], lc, ld);
                l_run = l_run * alpha + ((la + lb) + (lc + ld));
                f2_unpack(r2[0], la, lb);
                f2_unpack(r2[1], lc, ld);
                lr_run = lr_run * alpha + ((la + lb) + (lc + ld));
                // P buffer b was last read by P V of tile n - 2, which the tensor pipe completed before S_n (in order)
                // this group rescales its 64 columns of O (once P V of tile n - 1 has added to them) before this tile's
                // P V may add to them
                if (t > 0 && __any_sync(0xffffffffu, need)) {
                    if (!(ok = wait_bounded_warp(BAR(S_PV_DONE0 + (b ^ 1u)), ((n - 1) >> 1) & 1u, lim))) break;
                    tc_fence_after();
    #pragma unroll
                    for (int ch = 0; ch < 2; ++ch) {
                        uint32_t ov[32];
                        tmem_ld32(tO + grp * 64u + lane_off + ch * 32u, ov);
                        tmem_wait_ld();
    #pragma unroll
                        for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                        tmem_st32(tO + grp * 64u + lane_off + ch * 32u, ov);
                    }
                }
                tmem_st32(tP + b * 64u + grp * 32u + lane_off, pw);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(BAR(S_P_FULL0 + b));
                // the previous item's epilogue, now that this item's first tile is out of the way
                if (t == 0 && pend) {
                    if (!(ok = epilogue())) break;
                    pend = false;
                }
            }
            if (!ok) break;
            pend = true;
            pd_grow = grow;
            pd_m = m_raw;
            pd_l = l_run;
            pd_lr = lr_run;
            pd_nl = n - 1;
        }
        if (ok && pend) epilogue();
    }
    // Teardown: every role has left its loop (normally or after a bounded wait ran out).
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace losa
