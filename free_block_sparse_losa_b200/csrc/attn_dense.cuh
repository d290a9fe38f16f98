// Dense-step tensor-core kernel (bf16, head_dim 128, 128-row query blocks): attn_dense_kernel<WITH_MASS, SUB, ONE_PASS>.
//
// The dense forward (LoSA page, Motivation Summary: A = softmax(Q K^T / sqrt(d)) and O = A V) and, with WITH_MASS, the
// exact block masses of the construction step (Motivation Summary: M(i, j) = sum of A over query block i and key
// block j; Methodology Summary: the masses are exact because construction coincides with a dense step), with SUB key
// blocks per 128 keys (1 for C = 128, 4 for C = 32).
//
// Shape of the work: one CTA per SM, one query block (item) at a time; keys are consumed in tiles of 256.
//   S = Q K^T is one 128 x 256 tcgen05.mma tile (8 instructions of K = 16): N = 256 reads each Q fragment once for
//   256 keys and needs half the instructions per key. TMEM holds S (columns 0..255), O (256..383) and P (384..511,
//   bf16 pairs),
//   so S is free as soon as the softmax has read it: the next QK^T overlaps this tile's softmax and P V.
//   Two softmax warpgroups (warps 4..7 and 8..11) split the 256 columns; thread t of each owns query row t (TMEM lane
//   t). Each also reads the other group's half of S, for the row max only: the max is exact, so both groups reach the
//   same running max without an exchange. They keep their own partial row sums, rescale their own half of O, and
//   write their own half of P. P V runs as two groups of eight
//   N = 128 instructions (keys 0..127 and 128..255) with P read from TMEM and V from shared memory (MN-major).
//   Warp 0 issues the TMA loads of Q (once per item) and K (single-buffered), warp 2 those of V (double-buffered),
//   64 KB per 256-key tile; each box of a tile comes from its own lane. Warp 1 issues the MMAs and owns TMEM.
//   One-pass masses (ONE_PASS): every forward tile's exact per-block sums of its weights, brought to a per-row anchor
//   max, are stored to a [SMs][nk][128] fp32 workspace; once the item's rows have their final max and sum, eight
//   warps reduce them to M with one factor per row (passed through shared memory).
//   Two-pass masses (mass phase: same item, Q still in shared memory, lse exact in registers): S is recomputed for
//   every 256-key tile and each warpgroup sums 2^(s*c - lse2) over its 128 columns per key block; per-warp partials
//   go to the idle V buffer and are flushed to M every 1024 blocks.
// Registers: the producer / MMA warpgroup drops to 56 per thread and the softmax warpgroups rise to 224 (setmaxnreg), so
// the softmax's 128 S values, 64 P words and sums stay in registers.
// Every wait is bounded in time (LOSA_ERR_TIMEOUT in the device error word, then a clean exit).
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "attn_tc.cuh"

namespace losa {

constexpr uint32_t kDnQ = 0;                       // Q tile, 32 KB
constexpr uint32_t kDnK = 32768;                   // K tile of 256 keys, 64 KB: [d-half][256 rows][128 B]
constexpr uint32_t kDnV = 98304;                   // V tiles, 2 x 64 KB, same layout; buffer 0 doubles as mass partials
constexpr uint32_t kDnBar = 98304 + 2 * 65536;     // barriers, TMEM slot
constexpr uint32_t kDnXchg = kDnBar + 256;         // [2 groups][128] (exact, rounded) fp32 partial row sums
constexpr uint32_t kDnFsc = kDnXchg + 2 * 128 * 8;   // [128] fp32 row factors of the one-pass mass reduction
constexpr uint32_t kDnSmem = kDnFsc + 128 * 4;       // 232192 bytes: needs a 1024-aligned dynamic base
static_assert(kDnSmem <= 232448, "shared memory");
// One-pass masses: a row's stored block sums stay relative to its anchor max m0 while the running max stays within
// 2^kAnchorSpan of it (so no stored sum can overflow); past that the row re-anchors and rescales what it stored.
constexpr float kAnchorSpan = 60.0f;

enum : uint32_t {
    D_Q_FULL = 0, D_Q_EMPTY, D_K_FULL, D_K_EMPTY, D_V_FULL0, D_V_FULL1, D_V_EMPTY0, D_V_EMPTY1, D_S_FULL, D_S_FREE,
    D_P_FULL, D_PV_DONE, D_O_FREE, D_SUM_X, D_PART, D_PART2, D_MASS_DONE, D_MMA_DONE, D_COUNT
};

template <bool WITH_MASS, int SUB, bool ONE_PASS = false>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_dense_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV, const TcArgs a) {
    extern __shared__ __align__(1024) uint8_t dn_smem[];
    const uint32_t base = smem_addr(dn_smem);
    if (base & 1023u) {  // the 128-byte-swizzled tiles need a 1024-aligned base; report instead of overrunning
        if (threadIdx.x == 0) atomicOr(&g_device_error, kDevErrBadData);
        return;
    }
    uint8_t* const base_ptr = dn_smem;
    const uint32_t bar0 = base + kDnBar;
    auto BAR = [&](uint32_t s) { return bar0 + 8u * s; };
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + kDnBar + D_COUNT * 8);
    float2* const xsum = reinterpret_cast<float2*>(base_ptr + kDnXchg);         // [2 groups][128]
    float* const part = reinterpret_cast<float*>(base_ptr + kDnV);              // [4 row groups][1024 blocks]
    float* const fsc = reinterpret_cast<float*>(base_ptr + kDnFsc);             // [128] one-pass row factors

    const int warp = threadIdx.x >> 5;
    const uint32_t lane = lane_id();
    if (threadIdx.x == 0) {
        for (uint32_t s = 0; s < D_COUNT; ++s) {
            const bool wide = s == D_S_FREE || s == D_P_FULL || s == D_O_FREE || s == D_SUM_X ||
                              s == D_PART || s == D_PART2 || s == D_MASS_DONE;
            mbar_init(BAR(s), wide ? 256u : 1u);
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
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
    const uint32_t tS = tmem, tO = tmem + 256u, tP = tmem + 384u;
    const unsigned long long lim = a.wait_limit_ns;
    const int T = (a.nk + 1) / 2;  // 256-key tiles per head
    const int mass_tiles = (WITH_MASS && !ONE_PASS) ? T : 0;  // the two-pass form recomputes every tile
    const int G = gridDim.x;

    // Registers: the producer / MMA warpgroup needs few, the softmax warpgroups many. Each warpgroup reaches one
    // setmaxnreg; the split uses exactly the 384 x 168 registers the block is launched with (128 x 56 + 256 x 224).
    if (warp < 4) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
        if (warp == 0) {
            // ------------------------------------------------------------- TMA producer: Q and K (whole warp)
            // Every 16 KB box of a tile is issued by its own lane (lane 0 posts the expected bytes first): one thread's
            // TMA loads are served one after another at about 30 bytes per clock, too slow for 64 KB per tile.
            const uint64_t pol_q = l2_policy_evict_first();
            const uint64_t pol_kv = l2_policy_evict_last();
            const uint32_t dh = lane >> 1, rh = lane & 1u;  // box of lane < 4: column half dh, row half rh
            uint32_t nq = 0, nk_ld = 0;
            bool ok = true;
            for (int w = blockIdx.x; ok && w < a.n_items; w += G) {
                const int h = w / a.nq, qb = w - h * a.nq;
                if (!(ok = wait_bounded_warp(BAR(D_Q_EMPTY), (nq & 1u) ^ 1u, lim))) break;
                const int32_t qrow = h * a.Np + qb * kTcRows;
                if (lane == 0) mbar_arrive_expect_tx(BAR(D_Q_FULL), kTileBytes);
                __syncwarp();
                if (lane < 2) tma_load_2d_hint(base + kDnQ + lane * kBoxBytes, &tmQ, 64 * (int)lane, qrow, BAR(D_Q_FULL), pol_q);
                ++nq;
                for (int t = 0; t < T + mass_tiles; ++t) {
                    const int32_t krow = h * a.Np + (t < T ? t : t - T) * 256;  // rows past the head are masked
                    if (!(ok = wait_bounded_warp(BAR(D_K_EMPTY), (nk_ld & 1u) ^ 1u, lim))) break;
                    if (lane == 0) mbar_arrive_expect_tx(BAR(D_K_FULL), 2 * kTileBytes);
                    __syncwarp();
                    if (lane < 4)
                        tma_load_2d_hint(base + kDnK + dh * 32768u + rh * 16384u, &tmK, 64 * (int)dh, krow + 128 * (int)rh,
                                         BAR(D_K_FULL), pol_kv);
                    ++nk_ld;
                }
            }
            if (nq) wait_bounded(BAR(D_Q_FULL), (nq - 1) & 1u, kDrainLimitNs);
            if (nk_ld) wait_bounded(BAR(D_K_FULL), (nk_ld - 1) & 1u, kDrainLimitNs);
            __syncwarp();
        } else if (warp == 2) {
            // ------------------------------------------------------------------- TMA producer: V (whole warp)
            const uint64_t pol_kv = l2_policy_evict_last();
            const uint32_t dh = lane >> 1, rh = lane & 1u;
            uint32_t nv_ld = 0, n_it = 0;
            bool ok = true;
            for (int w = blockIdx.x; ok && w < a.n_items; w += G) {
                const int h = w / a.nq;
                for (int t = 0; t < T; ++t) {
                    const int32_t krow = h * a.Np + t * 256;
                    const uint32_t vb = nv_ld & 1u;
                    if (!(ok = wait_bounded_warp(BAR(D_V_EMPTY0 + vb), ((nv_ld >> 1) & 1u) ^ 1u, lim))) break;
                    if (lane == 0) mbar_arrive_expect_tx(BAR(D_V_FULL0 + vb), 2 * kTileBytes);
                    __syncwarp();
                    if (lane < 4)
                        tma_load_2d_hint(base + kDnV + vb * 65536u + dh * 32768u + rh * 16384u, &tmV, 64 * (int)dh,
                                         krow + 128 * (int)rh, BAR(D_V_FULL0 + vb), pol_kv);
                    ++nv_ld;
                }
                // The mass phase reuses V buffer 0 for partial sums: before loading the next item's V, wait until the
                // softmax has flushed this item's last chunk. MASS_DONE completes once per item, so its phase cannot be
                // confused with a later one: the next item's needs this warp's next V loads.
                if (WITH_MASS && !ONE_PASS && ok && !(ok = wait_bounded_warp(BAR(D_MASS_DONE), n_it & 1u, lim))) break;
                ++n_it;
            }
            for (uint32_t vb = 0; vb < 2; ++vb) {
                const uint32_t n = (nv_ld + 1u - vb) >> 1;
                if (n) wait_bounded(BAR(D_V_FULL0 + vb), (n - 1) & 1u, kDrainLimitNs);
            }
            __syncwarp();
        } else if (warp == 1) {
            // ------------------------------------------------------------------------------------ MMA issuer
            if (lane == 0) {
                constexpr uint32_t kIdQK = idesc_bf16_f32(128, 256, false, false);
                constexpr uint32_t kIdPV = idesc_bf16_f32(128, 128, false, true);
                uint32_t nq = 0, n_qk = 0, nk_use = 0, n_pv = 0, n_items = 0;
                bool ok = true;
                auto issue_pv = [&](int t) -> bool {
                    const uint32_t vb = n_pv & 1u;
                    if (!wait_bounded(BAR(D_P_FULL), n_pv & 1u, lim)) return false;
                    if (!wait_bounded(BAR(D_V_FULL0 + vb), (n_pv >> 1) & 1u, lim)) return false;
                    if (t == 0 && !wait_bounded(BAR(D_O_FREE), (n_items & 1u) ^ 1u, lim)) return false;
                    tc_fence_after();
                    const uint32_t vbase = base + kDnV + vb * 65536u;
    #pragma unroll
                    for (uint32_t h2 = 0; h2 < 2; ++h2)
    #pragma unroll
                        for (uint32_t kk = 0; kk < 8; ++kk)
                            tc_mma_ts(tO, tP + h2 * 64u + kk * 8u, smem_desc(vbase + h2 * 16384u + kk * 2048u, 32768, 1024),
                                      kIdPV, (t == 0 && h2 == 0 && kk == 0) ? 0u : 1u);
                    tc_commit(BAR(D_V_EMPTY0 + vb));
                    tc_commit(BAR(D_PV_DONE));
                    ++n_pv;
                    return true;
                };
                for (int w = blockIdx.x; ok && w < a.n_items; w += G) {
                    if (!(ok = wait_bounded(BAR(D_Q_FULL), nq & 1u, lim))) break;
                    ++nq;
                    for (int t = 0; t < T + mass_tiles; ++t) {
                        if (!(ok = wait_bounded(BAR(D_K_FULL), nk_use & 1u, lim))) break;
                        if (n_qk > 0 && !(ok = wait_bounded(BAR(D_S_FREE), (n_qk - 1) & 1u, lim))) break;
                        tc_fence_after();
    #pragma unroll
                        for (uint32_t kk = 0; kk < 8; ++kk) {
                            const uint32_t qo = (kk >> 2) * kBoxBytes + (kk & 3u) * 32u;
                            const uint32_t ko = (kk >> 2) * 32768u + (kk & 3u) * 32u;
                            tc_mma_ss(tS, smem_desc(base + kDnQ + qo, 16, 1024), smem_desc(base + kDnK + ko, 16, 1024), kIdQK,
                                      kk ? 1u : 0u);
                        }
                        tc_commit(BAR(D_S_FULL));
                        tc_commit(BAR(D_K_EMPTY));
                        ++nk_use;
                        ++n_qk;
                        if (t == T + mass_tiles - 1) tc_commit(BAR(D_Q_EMPTY));
                        // P V of the previous forward tile goes behind this QK^T in the tensor pipe.
                        if (t >= 1 && t <= T && !(ok = issue_pv(t - 1))) break;
                    }
                    if (ok && mass_tiles == 0 && !(ok = issue_pv(T - 1))) break;
                    ++n_items;
                }
                tc_commit(BAR(D_MMA_DONE));
                wait_bounded(BAR(D_MMA_DONE), 0, kDrainLimitNs);
            }
            __syncwarp();
        } else if (warp == 3) {
            // idle: gives up its registers with the rest of its warpgroup
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 224;" ::: "memory");
        // --------------------------------------------------------------------------- softmax warpgroups
        const uint32_t grp = (uint32_t)(warp - 4) >> 2;  // column half: keys 128 * grp .. 128 * grp + 127 of a tile
        const uint32_t wl = (uint32_t)warp & 3u;
        const int row = (int)(wl * 32u + lane);
        const uint32_t lane_off = (wl * 32u) << 16;
        const uint32_t tSg = tS + grp * 128u, tPg = tP + grp * 64u, tOg = tO + grp * 64u;
        const float c = a.scale_log2;
        uint32_t n_s = 0, n_pv = 0, n_items = 0, n_chunks = 0;
        bool ok = true;
        for (int w = blockIdx.x; ok && w < a.n_items; w += G) {
            const int h = w / a.nq, qb = w - h * a.nq;
            const int qrow = qb * kTcRows + row;
            const size_t grow = (size_t)h * a.Np + qrow;
            float m_raw = -INFINITY, l_run = 0.0f, lr_run = 0.0f;  // exact and bf16-rounded row sums
            // one-pass masses: this row's anchor max and the factor from the current reference max to it
            float m0 = 0.0f, fac = 1.0f;
            float* const pslot = ONE_PASS ? a.mass_part + (size_t)blockIdx.x * a.nkb * kTcRows : nullptr;
            for (int t = 0; t < T; ++t) {
                const int kvalid = a.N - (2 * t + (int)grp) * 128;  // real keys in this group's 128 columns
                const bool full = kvalid >= 128;
                if (!(ok = wait_bounded_warp(BAR(D_S_FULL), n_s & 1u, lim))) break;
                ++n_s;
                tc_fence_after();
                // The row max over the whole tile without a cross-group exchange: the other group's 128 columns are
                // read first, 64 at a time, and only their maximum is kept (max is exact, so both groups agree).
                float omax = -INFINITY;
                {
                    const int ovalid = a.N - (2 * t + (int)(1u - grp)) * 128;  // real keys in the other group's columns
                    const uint32_t tSo = tS + (1u - grp) * 128u;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh) {
                        float o[64];
                        tmem_ld32(tSo + lane_off + hh * 64u, *reinterpret_cast<uint32_t(*)[32]>(&o[0]));
                        tmem_ld32(tSo + lane_off + hh * 64u + 32u, *reinterpret_cast<uint32_t(*)[32]>(&o[32]));
                        tmem_wait_ld();
                        if (ovalid < 128) {
#pragma unroll
                            for (int cc = 0; cc < 64; ++cc)
                                if (hh * 64 + cc >= ovalid) o[cc] = -INFINITY;
                        }
                        float mx[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) mx[e] = fmax3(o[e], o[8 + e], o[16 + e]);
#pragma unroll
                        for (int cc = 24; cc < 64; cc += 16)
#pragma unroll
                            for (int e = 0; e < 8; ++e) mx[e] = fmax3(mx[e], o[cc + e], o[cc + 8 + e]);
                        omax = fmaxf(omax, fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], fmax3(mx[5], mx[6], mx[7]))));
                    }
                }
                // This group's own 128 columns; S is released once both groups have read all of it, so the next QK^T
                // runs under this tile's exponentials.
                float s[128];
#pragma unroll
                for (int ch = 0; ch < 4; ++ch)
                    tmem_ld32(tSg + lane_off + ch * 32u, *reinterpret_cast<uint32_t(*)[32]>(&s[ch * 32]));
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(BAR(D_S_FREE));
                if (!full) {
#pragma unroll
                    for (int cc = 0; cc < 128; ++cc)
                        if (cc >= kvalid) s[cc] = -INFINITY;
                }
                float tmax;
                {
                    float mx[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) mx[e] = fmax3(s[e], s[8 + e], s[16 + e]);
#pragma unroll
                    for (int cc = 24; cc < 128; cc += 16)
#pragma unroll
                        for (int e = 0; e < 8; ++e) mx[e] = fmax3(mx[e], s[cc + e], s[cc + 8 + e]);
                    tmax = fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], fmax3(mx[5], mx[6], mx[7])));
                }
                tmax = fmaxf(tmax, omax);  // the tile max over all 256 columns
                const bool need = (t == 0) || (tmax - m_raw) * c > 8.0f;
                const float alpha = (t > 0 && need) ? ex2_approx((m_raw - tmax) * c) : 1.0f;
                if (need) m_raw = tmax;
                const float neg_mc = -m_raw * c;
                // P for this group's 128 columns, from registers, held until the P unit is free. The one-pass mass
                // with 32-key blocks keeps the exact sums per 32 columns (lq), the others per pair parity (l2).
                constexpr bool kQuarters = ONE_PASS && SUB > 1;
                uint32_t pw[64];
                uint64_t l2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)}, r2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
                uint64_t lq[kQuarters ? 8 : 1];
#pragma unroll
                for (int i = 0; i < (kQuarters ? 8 : 1); ++i) lq[i] = f2_pack(0.f, 0.f);
                if (full) {
                    const uint64_t c2 = f2_pack(c, c), nm2 = f2_pack(neg_mc, neg_mc);
#pragma unroll
                    for (int e = 0; e < 64; ++e) {
                        const uint64_t xx = f2_fma(f2_pack(s[2 * e], s[2 * e + 1]), c2, nm2);
                        float x0, x1;
                        f2_unpack(xx, x0, x1);
                        const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                        pw[e] = pack_bf16x2(p0, p1);
                        if constexpr (kQuarters)
                            lq[2 * (e >> 4) + (e & 1)] = f2_add(lq[2 * (e >> 4) + (e & 1)], f2_pack(p0, p1));
                        else
                            l2[e & 1] = f2_add(l2[e & 1], f2_pack(p0, p1));
                        r2[e & 1] = f2_add(r2[e & 1], bf16x2_to_f2(pw[e]));
                    }
                } else {
#pragma unroll
                    for (int e = 0; e < 64; ++e) {
                        const float p0 = (2 * e < kvalid) ? ex2_approx(fmaf(s[2 * e], c, neg_mc)) : 0.0f;
                        const float p1 = (2 * e + 1 < kvalid) ? ex2_approx(fmaf(s[2 * e + 1], c, neg_mc)) : 0.0f;
                        pw[e] = pack_bf16x2(p0, p1);
                        if constexpr (kQuarters)
                            lq[2 * (e >> 4) + (e & 1)] = f2_add(lq[2 * (e >> 4) + (e & 1)], f2_pack(p0, p1));
                        else
                            l2[e & 1] = f2_add(l2[e & 1], f2_pack(p0, p1));
                        r2[e & 1] = f2_add(r2[e & 1], bf16x2_to_f2(pw[e]));
                    }
                }
                float qs[kQuarters ? 4 : 1];  // exact sums of the 32-column quarters
                if constexpr (kQuarters) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        float x0, x1, x2, x3;
                        f2_unpack(lq[2 * g], x0, x1);
                        f2_unpack(lq[2 * g + 1], x2, x3);
                        qs[g] = (x0 + x1) + (x2 + x3);
                    }
                }
                float la, lb, lc, ld;
                f2_unpack(l2[0], la, lb);
                f2_unpack(l2[1], lc, ld);
                float tsum;  // exact sum of this tile's 128 columns
                if constexpr (kQuarters)
                    tsum = (qs[0] + qs[1]) + (qs[2] + qs[3]);
                else
                    tsum = (la + lb) + (lc + ld);
                l_run = l_run * alpha + tsum;
                f2_unpack(r2[0], la, lb);
                f2_unpack(r2[1], lc, ld);
                lr_run = lr_run * alpha + ((la + lb) + (lc + ld));
                if constexpr (ONE_PASS) {
                    // This tile's block sums of 2^(s c - m0 c), for the reduction at the item's end. The reference
                    // max only grows; past 2^kAnchorSpan above the anchor the row re-anchors first (rare).
                    if (t == 0) {
                        m0 = m_raw;
                        fac = 1.0f;
                    } else if (need) {
                        if ((m_raw - m0) * c > kAnchorSpan) {
                            const float r = ex2_approx((m0 - m_raw) * c);
                            for (int tt = 0; tt < t; ++tt)
                                for (int g = 0; g < SUB; ++g) {
                                    const int j = (2 * tt + (int)grp) * SUB + g;
                                    if (j < a.nkb) pslot[(size_t)j * kTcRows + row] *= r;
                                }
                            m0 = m_raw;
                            fac = 1.0f;
                        } else {
                            fac = ex2_approx((m_raw - m0) * c);
                        }
                    }
                    if constexpr (kQuarters) {
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const int j = (2 * t + (int)grp) * SUB + g;
                            if (j < a.nkb) pslot[(size_t)j * kTcRows + row] = qs[g] * fac;
                        }
                    } else {
                        const int j = 2 * t + (int)grp;
                        if (j < a.nkb) pslot[(size_t)j * kTcRows + row] = tsum * fac;
                    }
                }
                // The previous P V must be done before its P is overwritten and before O is rescaled.
                if (t > 0) {
                    if (!(ok = wait_bounded_warp(BAR(D_PV_DONE), n_pv & 1u, lim))) break;
                    ++n_pv;
                    tc_fence_after();
                    if (__any_sync(0xffffffffu, need)) {
#pragma unroll
                        for (int ch = 0; ch < 2; ++ch) {
                            uint32_t ov[32];
                            tmem_ld32(tOg + lane_off + ch * 32u, ov);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                            tmem_st32(tOg + lane_off + ch * 32u, ov);
                        }
                    }
                }
                tmem_st32(tPg + lane_off, *reinterpret_cast<uint32_t(*)[32]>(&pw[0]));
                tmem_st32(tPg + lane_off + 32u, *reinterpret_cast<uint32_t(*)[32]>(&pw[32]));
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(BAR(D_P_FULL));
            }
            if (!ok) break;
            // Epilogue: full row sums from both groups, O / l for this group's 64 columns, lse. A group writes the
            // sums of the next item only after that item's first P V, or its mass phase, has needed both groups'
            // arrivals after they read these (P_FULL, PART), so one buffer serves every item.
            if (!(ok = wait_bounded_warp(BAR(D_PV_DONE), n_pv & 1u, lim))) break;
            ++n_pv;
            tc_fence_after();
            xsum[grp * 128u + row] = make_float2(l_run, lr_run);
            mbar_arrive(BAR(D_SUM_X));
            if (!(ok = wait_bounded_warp(BAR(D_SUM_X), n_items & 1u, lim))) break;
            const float2 other = xsum[(1u - grp) * 128u + row];
            const float l_all = l_run + other.x;
            const float inv_l = 1.0f / (lr_run + other.y);
            const float lse2 = m_raw * c + lg2_approx(l_all);
            uint4* dst = reinterpret_cast<uint4*>(a.o + grow * kTcDim + grp * 64u);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) {
                uint32_t ov[32];
                tmem_ld32(tOg + lane_off + ch * 32u, ov);
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
            mbar_arrive(BAR(D_O_FREE));
            if (a.lse && grp == 0) a.lse[grow] = lse2 * 0.6931471805599453f;

            if constexpr (ONE_PASS) {
                // M(i, j) = sum over the block's rows of (stored sum) * 2^(m0 c - m c) / l, divided by its real rows.
                // Every row's sums were stored before the row-sum exchange above; the factors go through shared
                // memory; the next item overwrites both only after every warp has passed PART2.
                if (grp == 0) fsc[row] = (qrow < a.N) ? ex2_approx((m0 - m_raw) * c) / l_all : 0.0f;
                mbar_arrive(BAR(D_PART));
                if (!(ok = wait_bounded_warp(BAR(D_PART), n_items & 1u, lim))) break;
                const float inv_rows = 1.0f / (float)min(kTcRows, a.N - qb * kTcRows);
                float* mrow = a.mass + (size_t)w * a.nkb;
                const float4 f4 = reinterpret_cast<const float4*>(fsc)[lane];
                for (int j = warp - 4; j < a.nkb; j += 8) {
                    const float4 v4 = reinterpret_cast<const float4*>(pslot + (size_t)j * kTcRows)[lane];
                    float sum = (v4.x * f4.x + v4.y * f4.y) + (v4.z * f4.z + v4.w * f4.w);
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                    if (lane == 0) mrow[j] = sum * inv_rows;
                }
                mbar_arrive(BAR(D_PART2));
                if (!(ok = wait_bounded_warp(BAR(D_PART2), n_items & 1u, lim))) break;
            }

            if (WITH_MASS && !ONE_PASS) {
                // Mass phase: 2^(s*c - lse2) summed per key block of this group's columns, for real rows and keys.
                const bool qvalid = qrow < a.N;
                const float neg_lse2 = qvalid ? -lse2 : 0.0f;
                const uint64_t c2 = f2_pack(c, c), nl2 = f2_pack(neg_lse2, neg_lse2);
                const float inv_rows = 1.0f / (float)min(kTcRows, a.N - qb * kTcRows);
                float* mrow = a.mass + (size_t)w * a.nkb;
                constexpr int kChunkTiles = kMaxMassBlocks / (2 * SUB);  // 256-key tiles per flush of 1024 blocks
                for (int t0 = 0; ok && t0 < T; t0 += kChunkTiles) {
                    const int t1 = min(T, t0 + kChunkTiles);
                    for (int t = t0; t < t1; ++t) {
                        if (!(ok = wait_bounded_warp(BAR(D_S_FULL), n_s & 1u, lim))) break;
                        ++n_s;
                        tc_fence_after();
                        float s[128];
#pragma unroll
                        for (int ch = 0; ch < 4; ++ch)
                            tmem_ld32(tSg + lane_off + ch * 32u, *reinterpret_cast<uint32_t(*)[32]>(&s[ch * 32]));
                        tmem_wait_ld();
                        tc_fence_before();
                        mbar_arrive(BAR(D_S_FREE));
                        const int kvalid = a.N - (2 * t + (int)grp) * 128;
                        uint64_t acc[8];
#pragma unroll
                        for (int i = 0; i < 8; ++i) acc[i] = f2_pack(0.f, 0.f);
                        if (kvalid >= 128) {
#pragma unroll
                            for (int e = 0; e < 64; ++e) {
                                const uint64_t xx = f2_fma(f2_pack(s[2 * e], s[2 * e + 1]), c2, nl2);
                                float x0, x1;
                                f2_unpack(xx, x0, x1);
                                const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
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
                        // block index (within the chunk) of this group's first block in tile t
                        const int jb0 = ((t - t0) * 2 + (int)grp) * SUB;
                        if (SUB == 1) {
                            float sum = (q[0] + q[1]) + (q[2] + q[3]);
#pragma unroll
                            for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                            if (lane == 0) part[wl * kMaxMassBlocks + jb0] = sum;
                        } else {
#pragma unroll
                            for (int g = 0; g < 4; ++g) {
#pragma unroll
                                for (int o = 16; o > 0; o >>= 1) q[g] += __shfl_xor_sync(0xffffffffu, q[g], o);
                            }
                            if (lane < 4) {
                                const float mine = lane == 0 ? q[0] : (lane == 1 ? q[1] : (lane == 2 ? q[2] : q[3]));
                                part[wl * kMaxMassBlocks + jb0 + lane] = mine;
                            }
                        }
                    }
                    if (!ok) break;
                    mbar_arrive(BAR(D_PART));
                    if (!(ok = wait_bounded_warp(BAR(D_PART), n_chunks & 1u, lim))) break;
                    const int b0 = t0 * 2 * SUB, b1 = min(a.nkb, t1 * 2 * SUB);
                    for (int jj = b0 + (int)grp * 128 + row; jj < b1; jj += 256) {
                        const int o = jj - b0;
                        mrow[jj] = ((part[o] + part[kMaxMassBlocks + o]) +
                                    (part[2 * kMaxMassBlocks + o] + part[3 * kMaxMassBlocks + o])) * inv_rows;
                    }
                    mbar_arrive(BAR(D_PART2));
                    if (!(ok = wait_bounded_warp(BAR(D_PART2), n_chunks & 1u, lim))) break;
                    ++n_chunks;
                }
                if (!ok) break;
                mbar_arrive(BAR(D_MASS_DONE));  // every chunk of this item is flushed: V buffer 0 is free again
            }
            ++n_items;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, 512);
}

}  // namespace losa
