// Tensor-core (tcgen05 / TMEM / TMA) attention kernels for bf16 inputs, head_dim 128, 128 x 128 blocks.
//
// One kernel template, two modes:
//   Fwd  — online-softmax attention of one 128-row query block against a list of 128-key blocks: the full list
//          0..nk-1 for the dense step (LoSA page, Motivation Summary: A = softmax(Q K^T / sqrt(d))), or the frozen
//          retained list for the sparse steps (Methodology Summary, "Sparse attention with a frozen pattern":
//          the softmax denominator covers the retained keys only). Writes O (bf16) and the row log-sum-exp.
//   Mass — recomputes S = Q K^T for every key block and sums exp(s - lse) with the forward pass's log-sum-exp into
//          one value per (query block, key block), divided by the block's real rows (Motivation Summary: block
//          attention mass M(i, j)). The probability matrix is never written to memory.
//
// Persistent grid (one CTA per SM). CTA b takes work items b, 2G-1-b, 2G+b, ... of the item order (a snake over
// the longest-first order balances list lengths across CTAs). Warp roles inside a CTA (256 threads):
//   warp 0       TMA producer: Q tile once per item, K/V tiles into a 2-stage ring.
//   warp 1       MMA issuer (one thread): S = Q K^T into one of two TMEM S buffers, then O += P V into TMEM.
//                Also owns the TMEM allocation.
//   warps 4..7   softmax / epilogue: thread t owns query row t (TMEM lane t). Reads S from TMEM, keeps the running
//                max and sum in registers, writes P (bf16) to shared memory in the 128-byte-swizzled K-major layout
//                the tensor core reads, and rescales O in TMEM only when a row's max grows by more than 2^8 (the
//                final division by the row sum makes the choice of reference max exact). Epilogue: O / l -> bf16.
// Every wait is bounded in time; on expiry the kernel records LOSA_ERR_TIMEOUT in the device error word, waits for
// its own copies and MMAs in flight, frees TMEM and exits.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>
#include "ptx.cuh"

namespace losa {

enum class TcMode : int { Fwd = 0, Mass = 1 };

constexpr int kTcRows = 128;      // R = C = 128
constexpr int kTcDim = 128;       // head_dim
constexpr int kTcThreads = 256;
constexpr uint32_t kTileBytes = kTcRows * kTcDim * 2;   // 32 KB: one 128 x 128 bf16 tile
constexpr uint32_t kBoxBytes = kTileBytes / 2;         // 16 KB: one 128-row x 64-column TMA box

// Shared-memory map (offsets from a 1024-byte-aligned base).
constexpr uint32_t kOffQ = 0;
constexpr uint32_t kOffK = kOffQ + kTileBytes;            // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kTileBytes;        // 2 stages (Fwd)
constexpr uint32_t kOffP = kOffV + 2 * kTileBytes;        // Fwd
constexpr uint32_t kOffPart = kOffV;                      // Mass: 2 x [4][1024] fp32 partial sums (nk <= 1024)
constexpr uint32_t kPartFloats = 4 * 1024;
constexpr uint32_t kFwdBarOff = kOffP + kTileBytes;
constexpr uint32_t kMassBarOff = kOffPart + 2 * kPartFloats * 4;
constexpr uint32_t kBarBytes = 256;
constexpr uint32_t tc_smem_bytes(TcMode m) {
    return (m == TcMode::Fwd ? kFwdBarOff : kMassBarOff) + kBarBytes + 1024;  // + alignment slack
}

// Barrier slots (8 bytes each).
enum : uint32_t {
    B_Q_FULL = 0, B_Q_EMPTY = 1, B_K_FULL = 2, B_K_EMPTY = 4, B_V_FULL = 6, B_V_EMPTY = 8, B_S_FULL = 10,
    B_S_FREE = 12, B_P_FULL = 14, B_O_READY = 15, B_O_FREE = 16, B_MMA_DONE = 17, B_PART = 18, B_COUNT = 19
};

struct TcArgs {
    int H, N, Np, nq, nk, n_items;
    float scale_log2;              // logit scale times log2(e)
    const int32_t* indptr;         // null: dense list 0..nk-1
    const int32_t* kv_idx;
    const int32_t* order;          // null: ascending item ids
    __nv_bfloat16* o;              // Fwd output
    float* lse;                    // Fwd: output (may be null); Mass: input
    float* mass;                   // Mass output [n_items... H*nq][nk]
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
    int id, h, qb, begin, count;
};

__device__ __forceinline__ bool next_item(const TcArgs& a, int round, ItemInfo& it) {
    const int G = gridDim.x, b = blockIdx.x;
    const long long w = (long long)round * G + ((round & 1) ? (G - 1 - b) : b);
    if (w >= a.n_items) return false;
    it.id = a.order ? a.order[w] : (int)w;
    it.h = it.id / a.nq;
    it.qb = it.id - it.h * a.nq;
    if (a.indptr) {
        it.begin = a.indptr[it.id];
        it.count = a.indptr[it.id + 1] - it.begin;
    } else {
        it.begin = 0;
        it.count = a.nk;
    }
    return true;
}

__device__ __forceinline__ int tile_block(const TcArgs& a, const ItemInfo& it, int t) {
    if (!a.indptr) return t;
    const int j = a.kv_idx[it.begin + t];
    return (j < 0) ? 0 : (j >= a.nk ? a.nk - 1 : j);  // out-of-range indices are reported by the producer
}

template <TcMode MODE>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_addr(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    uint8_t* const base_ptr = smem_raw + (base - raw);
    const uint32_t bar0 = base + (MODE == TcMode::Fwd ? kFwdBarOff : kMassBarOff);
    uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(base_ptr + (bar0 - base) + B_COUNT * 8);
    auto BAR = [&](uint32_t slot) { return bar0 + slot * 8u; };
    constexpr uint32_t kTmemCols = (MODE == TcMode::Fwd) ? 512u : 256u;

    const int warp = threadIdx.x >> 5;
    const uint32_t lane = lane_id();

    if (threadIdx.x == 0) {
        mbar_init(BAR(B_Q_FULL), 1);
        mbar_init(BAR(B_Q_EMPTY), 1);
        for (int s = 0; s < 2; ++s) {
            mbar_init(BAR(B_K_FULL + s), 1);
            mbar_init(BAR(B_K_EMPTY + s), 1);
            mbar_init(BAR(B_V_FULL + s), 1);
            mbar_init(BAR(B_V_EMPTY + s), 1);
            mbar_init(BAR(B_S_FULL + s), 1);
            mbar_init(BAR(B_S_FREE + s), 128);
        }
        mbar_init(BAR(B_P_FULL), 128);
        mbar_init(BAR(B_O_READY), 1);
        mbar_init(BAR(B_O_FREE), 128);
        mbar_init(BAR(B_MMA_DONE), 1);
        mbar_init(BAR(B_PART), 128);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(smem_addr(tmem_slot), kTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        if (MODE == TcMode::Fwd) tma_prefetch_desc(&tmV);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const unsigned long long lim = a.wait_limit_ns;

    if (warp == 0) {
        // ------------------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t kc = 0, nq_loads = 0;
            uint32_t nk_loads[2] = {0u, 0u}, nv_loads[2] = {0u, 0u};
            bool ok = true;
            ItemInfo it;
            for (int round = 0; ok && next_item(a, round, it); ++round) {
                if (it.count <= 0) {
                    if (a.indptr) atomicOr(&g_device_error, kDevErrBadData);
                    continue;
                }
                if (!(ok = wait_bounded(BAR(B_Q_EMPTY), (nq_loads & 1u) ^ 1u, lim))) break;
                const int32_t qrow = it.h * a.Np + it.qb * kTcRows;
                mbar_arrive_expect_tx(BAR(B_Q_FULL), kTileBytes);
                tma_load_2d(base + kOffQ, &tmQ, 0, qrow, BAR(B_Q_FULL));
                tma_load_2d(base + kOffQ + kBoxBytes, &tmQ, 64, qrow, BAR(B_Q_FULL));
                ++nq_loads;
                for (int t = 0; t < it.count; ++t, ++kc) {
                    if (a.indptr) {
                        const int jr = a.kv_idx[it.begin + t];
                        if (jr < 0 || jr >= a.nk) atomicOr(&g_device_error, kDevErrBadData);
                    }
                    const int32_t krow = it.h * a.Np + tile_block(a, it, t) * kTcRows;
                    const uint32_t s = kc & 1u, ph = (kc >> 1) & 1u;
                    if (!(ok = wait_bounded(BAR(B_K_EMPTY + s), ph ^ 1u, lim))) break;
                    mbar_arrive_expect_tx(BAR(B_K_FULL + s), kTileBytes);
                    tma_load_2d(base + kOffK + s * kTileBytes, &tmK, 0, krow, BAR(B_K_FULL + s));
                    tma_load_2d(base + kOffK + s * kTileBytes + kBoxBytes, &tmK, 64, krow, BAR(B_K_FULL + s));
                    ++nk_loads[s];
                    if (MODE == TcMode::Fwd) {
                        if (!(ok = wait_bounded(BAR(B_V_EMPTY + s), ph ^ 1u, lim))) break;
                        mbar_arrive_expect_tx(BAR(B_V_FULL + s), kTileBytes);
                        tma_load_2d(base + kOffV + s * kTileBytes, &tmV, 0, krow, BAR(B_V_FULL + s));
                        tma_load_2d(base + kOffV + s * kTileBytes + kBoxBytes, &tmV, 64, krow, BAR(B_V_FULL + s));
                        ++nv_loads[s];
                    }
                }
            }
            // Drain: wait until every copy this thread issued has landed (they complete on their own).
            if (nq_loads) wait_bounded(BAR(B_Q_FULL), (nq_loads - 1) & 1u, lim);
            for (uint32_t s = 0; s < 2; ++s) {
                if (nk_loads[s]) wait_bounded(BAR(B_K_FULL + s), (nk_loads[s] - 1) & 1u, lim);
                if (nv_loads[s]) wait_bounded(BAR(B_V_FULL + s), (nv_loads[s] - 1) & 1u, lim);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t kIdQK = idesc_bf16_f32(128, 128, false, false);
            constexpr uint32_t kIdPV = idesc_bf16_f32(128, 128, false, true);
            uint32_t kc = 0, items = 0, pc = 0;
            bool ok = true;
            bool pend = false;
            uint32_t p_s = 0, p_ph = 0, p_first = 0, p_item = 0;
            auto issue_pv = [&]() -> bool {
                if (!wait_bounded(BAR(B_P_FULL), pc & 1u, lim)) return false;
                if (!wait_bounded(BAR(B_V_FULL + p_s), p_ph, lim)) return false;
                if (p_first && !wait_bounded(BAR(B_O_FREE), (p_item & 1u) ^ 1u, lim)) return false;
                tc_fence_after();
                const uint32_t vbase = base + kOffV + p_s * kTileBytes;
#pragma unroll
                for (uint32_t kk = 0; kk < 8; ++kk) {
                    const uint64_t da = smem_desc(base + kOffP + (kk >> 2) * kBoxBytes + (kk & 3u) * 32u, 16, 1024);
                    const uint64_t db = smem_desc(vbase + kk * 2048u, kBoxBytes, 1024);
                    tc_mma_ss(tmem + 256u, da, db, kIdPV, (p_first && kk == 0) ? 0u : 1u);
                }
                tc_commit(BAR(B_V_EMPTY + p_s));
                tc_commit(BAR(B_O_READY));
                ++pc;
                return true;
            };
            ItemInfo it;
            for (int round = 0; ok && next_item(a, round, it); ++round) {
                if (it.count <= 0) continue;
                if (!(ok = wait_bounded(BAR(B_Q_FULL), items & 1u, lim))) break;
                tc_fence_after();
                for (int t = 0; t < it.count; ++t, ++kc) {
                    const uint32_t s = kc & 1u, ph = (kc >> 1) & 1u;
                    if (!(ok = wait_bounded(BAR(B_K_FULL + s), ph, lim))) break;
                    if (!(ok = wait_bounded(BAR(B_S_FREE + s), ph ^ 1u, lim))) break;
                    tc_fence_after();
                    const uint32_t kbase = base + kOffK + s * kTileBytes;
#pragma unroll
                    for (uint32_t kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * kBoxBytes + (kk & 3u) * 32u;
                        tc_mma_ss(tmem + s * 128u, smem_desc(base + kOffQ + off, 16, 1024),
                                  smem_desc(kbase + off, 16, 1024), kIdQK, kk ? 1u : 0u);
                    }
                    tc_commit(BAR(B_S_FULL + s));
                    tc_commit(BAR(B_K_EMPTY + s));
                    if (t == it.count - 1) tc_commit(BAR(B_Q_EMPTY));
                    if (MODE == TcMode::Fwd) {
                        if (pend && !(ok = issue_pv())) break;
                        pend = true;
                        p_s = s;
                        p_ph = ph;
                        p_first = (t == 0);
                        p_item = items;
                    }
                }
                ++items;
            }
            if (MODE == TcMode::Fwd && ok && pend) issue_pv();
            tc_commit(BAR(B_MMA_DONE));
            wait_bounded(BAR(B_MMA_DONE), 0, lim);
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------------------------------ softmax / epilogue
        const uint32_t wl = (uint32_t)warp & 3u;
        const int row = (int)(wl * 32u + lane);
        const uint32_t lane_off = (wl * 32u) << 16;
        float* const part = reinterpret_cast<float*>(base_ptr + kOffPart);
        uint32_t kc = 0, oc = 0, done_items = 0;
        bool ok = true;
        ItemInfo it;
        for (int round = 0; ok && next_item(a, round, it); ++round) {
            if (it.count <= 0) continue;
            float* const pbuf = part + (done_items & 1u) * kPartFloats;
            const int qrow = it.qb * kTcRows + row;
            const size_t grow = (size_t)it.h * a.Np + qrow;
            float m_run = -INFINITY, l_run = 0.0f, lse2 = 0.0f;
            const bool qvalid = qrow < a.N;
            if (MODE == TcMode::Mass) lse2 = qvalid ? a.lse[grow] * 1.4426950408889634f : 0.0f;
            for (int t = 0; t < it.count; ++t, ++kc) {
                const uint32_t s = kc & 1u, ph = (kc >> 1) & 1u;
                if (!(ok = wait_bounded_warp(BAR(B_S_FULL + s), ph, lim))) break;
                tc_fence_after();
                uint32_t sr[128];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t (&chunk)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[c * 32]);
                    tmem_ld32(tmem + lane_off + s * 128u + c * 32u, chunk);
                }
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(BAR(B_S_FREE + s));
                const int j = tile_block(a, it, t);
                const int kvalid = min(kTcRows, a.N - j * kTcRows);
                if (MODE == TcMode::Mass) {
                    float sum = 0.0f;
#pragma unroll
                    for (int c = 0; c < 128; ++c) {
                        const float p = ex2_approx(fmaf(__uint_as_float(sr[c]), a.scale_log2, -lse2));
                        sum += (c < kvalid) ? p : 0.0f;
                    }
                    if (!qvalid) sum = 0.0f;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                    if (lane == 0) pbuf[wl * 1024u + (uint32_t)j] = sum;
                } else {
                    float x[128];
                    float tmax = -INFINITY;
#pragma unroll
                    for (int c = 0; c < 128; ++c) {
                        x[c] = (c < kvalid) ? __uint_as_float(sr[c]) * a.scale_log2 : -INFINITY;
                        tmax = fmaxf(tmax, x[c]);
                    }
                    if (t == 0) {
                        m_run = tmax;
                    } else {
                        // PV of the previous tile must be complete before P is overwritten or O is rescaled.
                        if (!(ok = wait_bounded_warp(BAR(B_O_READY), oc & 1u, lim))) break;
                        ++oc;
                        const bool need = tmax > m_run + 8.0f;
                        if (__any_sync(0xffffffffu, need)) {
                            const float alpha = need ? ex2_approx(m_run - tmax) : 1.0f;
                            tc_fence_after();
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                uint32_t ov[32];
                                tmem_ld32(tmem + lane_off + 256u + c * 32u, ov);
                                tmem_wait_ld();
#pragma unroll
                                for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
                                tmem_st32(tmem + lane_off + 256u + c * 32u, ov);
                            }
                            tmem_wait_st();
                            if (need) {
                                l_run *= alpha;
                                m_run = tmax;
                            }
                        }
                    }
                    // P = 2^(x - m_run) in bf16, stored in the 128B-swizzled K-major layout.
                    const uint32_t prow = base + kOffP + (uint32_t)row * 128u;
                    float lsum = 0.0f;
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
#pragma unroll
                        for (int ch = 0; ch < 8; ++ch) {
                            uint32_t w[4];
#pragma unroll
                            for (int e = 0; e < 4; ++e) {
                                const int c = half * 64 + ch * 8 + e * 2;
                                const float p0 = ex2_approx(x[c] - m_run);
                                const float p1 = ex2_approx(x[c + 1] - m_run);
                                lsum += p0 + p1;
                                w[e] = pack_bf16x2(p0, p1);
                            }
                            const uint32_t addr = prow + (uint32_t)half * kBoxBytes +
                                                  (uint32_t)((ch ^ (row & 7)) * 16);
                            st_shared_v4(addr, w[0], w[1], w[2], w[3]);
                        }
                    }
                    l_run += lsum;
                    fence_proxy_async_smem();
                    tc_fence_before();
                    mbar_arrive(BAR(B_P_FULL));
                }
            }
            if (!ok) break;
            if (MODE == TcMode::Mass) {
                // All four warps' partial sums of this item are in pbuf once the 128 threads have arrived. The
                // next item writes the other buffer, and the one after that only starts once every thread has
                // arrived again, i.e. finished reading this one.
                mbar_arrive(BAR(B_PART));
                if (!(ok = wait_bounded_warp(BAR(B_PART), done_items & 1u, lim))) break;
                const float inv_rows = 1.0f / (float)min(kTcRows, a.N - it.qb * kTcRows);
                float* mrow = a.mass + (size_t)it.id * a.nk;
                for (int jj = row; jj < a.nk; jj += 128)
                    mrow[jj] = (pbuf[jj] + pbuf[1024 + jj] + pbuf[2048 + jj] + pbuf[3072 + jj]) * inv_rows;
            } else {
                if (!(ok = wait_bounded_warp(BAR(B_O_READY), oc & 1u, lim))) break;
                ++oc;
                tc_fence_after();
                const float inv_l = 1.0f / l_run;
                __nv_bfloat16* orow = a.o + grow * kTcDim;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t ov[32];
                    tmem_ld32(tmem + lane_off + 256u + c * 32u, ov);
                    tmem_wait_ld();
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(ov[q4 * 8 + 0]) * inv_l, __uint_as_float(ov[q4 * 8 + 1]) * inv_l);
                        v.y = pack_bf16x2(__uint_as_float(ov[q4 * 8 + 2]) * inv_l, __uint_as_float(ov[q4 * 8 + 3]) * inv_l);
                        v.z = pack_bf16x2(__uint_as_float(ov[q4 * 8 + 4]) * inv_l, __uint_as_float(ov[q4 * 8 + 5]) * inv_l);
                        v.w = pack_bf16x2(__uint_as_float(ov[q4 * 8 + 6]) * inv_l, __uint_as_float(ov[q4 * 8 + 7]) * inv_l);
                        dst[q4] = v;
                    }
                }
                if (a.lse) a.lse[grow] = (m_run + lg2_approx(l_run)) * 0.6931471805599453f;
                tc_fence_before();
                mbar_arrive(BAR(B_O_FREE));
            }
            ++done_items;
        }
    }
    // Teardown: every role has left its loop (normally or after a bounded wait ran out).
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace losa
