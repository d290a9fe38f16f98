// Mass-threshold block selection (LoSA page, Methodology Summary, "One-time pattern construction"), and the
// fixed-count top-k rule the page's ablation compares it with (Experiments Summary, "Retained mass vs. a fixed
// sparsity ratio").
//
// Rule per row (head, query block): order the key blocks by (mass descending, index ascending); integer units
// u_j = ceil(M_j * 2^52); T = ceil(tau * sum_j u_j) in IEEE double; keep the first s >= 1 blocks whose integer prefix
// reaches T, listed in ascending index order. Input domain: every mass finite and >= 0, every row summing to at most 2
// (rows are normalised to one; the slack covers rounding). Outside it the device error word is set and the row's
// result is unspecified, without undefined arithmetic (units are computed from min(M_j, 2)).
//
// Launches, all stream-ordered:
//   1. select_pick_warp_kernel<E> (nk <= 1024)  one warp per row, keys in registers. At a threshold near one a row
//        keeps a handful of blocks, so the first s positions of the sorted order are found as successive warp-wide
//        minima (the pick path, up to kPickCap positions): each lane keeps its smallest unconsumed keys sorted in
//        registers, a pick is two 32-bit warp reductions over the lanes' first entries, and a lane rescans its keys
//        only when those are used up. A row whose cut lies further is left undecided (count -1) for
//        select_sort_warp_kernel<E>, a bitonic sort of all its keys in registers. Both give the same s and kept
//        set: the prefix runs over the same positions in the same order.
//      select_pick_smem_kernel + select_rows_kernel (nk > 1024)  the pick path with the row in shared memory; rows it
//        leaves undecided are sorted by one CTA each in shared memory.
//      The kept blocks of each row are staged in ascending order in the workspace, with the count s.
//   2. select_hist_kernel   chunks of 1024 rows: a histogram of the counts per chunk and the chunk's sum of counts;
//        the last chunk to finish scans the histograms (count descending, chunk ascending) and the chunk sums.
//   3. select_order_kernel  per chunk: indptr (exclusive scan of the counts) and the longest-first work order, a stable
//        counting sort of the rows by count descending (rows of equal count keep ascending ids).
//   4. select_scatter_kernel one warp per row copies its staged indices to kv_block_idx[indptr[row] ...].
#pragma once
#include <cstdint>
#include "ptx.cuh"

namespace losa {

constexpr int kSelectThreads = 256;
constexpr int kPickSlots = 4;                 // picks held per lane
constexpr int kPickCap = 32 * kPickSlots;     // positions the pick path tries before falling back to the sort
// Smallest unconsumed keys each lane keeps in registers on the pick path: two for rows in registers (where most rows
// keep a few blocks and a rescan costs one pass over the lane's registers), four for rows in shared memory (longer
// lists, and a rescan reads nk / 32 words of shared memory).
constexpr int kPickCacheReg = 2, kPickCacheSmem = 4;
constexpr int kOrderChunk = 1024;             // rows per chunk of the order kernels (one thread each)
constexpr uint64_t kMaxRowUnits = 9007199254740992ull;          // 2^53: a row summing to 2

__device__ __forceinline__ uint64_t warp_incl_scan_u64(uint64_t x) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if ((int)lane_id() >= o) x += y;
    }
    return x;
}

__device__ __forceinline__ uint64_t warp_sum_u64(uint64_t x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

// Block-wide exclusive scan of one uint64 per thread (NT threads); returns the exclusive prefix and the total.
template <int NT>
__device__ __forceinline__ uint64_t block_excl_scan_u64(uint64_t x, uint64_t* warp_tot, uint64_t& total) {
    constexpr int NW = NT / 32;
    const int w = threadIdx.x >> 5;
    const uint64_t inc = warp_incl_scan_u64(x);
    if (lane_id() == 31) warp_tot[w] = inc;
    __syncthreads();
    if (w == 0) {
        uint64_t t = (lane_id() < NW) ? warp_tot[lane_id()] : 0ull;
        t = warp_incl_scan_u64(t);
        if (lane_id() < NW) warp_tot[lane_id()] = t;  // inclusive per warp
    }
    __syncthreads();
    total = warp_tot[NW - 1];
    const uint64_t before = (w > 0) ? warp_tot[w - 1] : 0ull;
    __syncthreads();  // warp_tot may be reused by the caller
    return before + inc - x;
}

// Shared-memory bitonic sort, ascending, of n (power of two) keys by NT threads.
template <int NT, typename K>
__device__ __forceinline__ void bitonic_sort_smem(K* keys, int n) {
    for (int k = 2; k <= n; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int i = threadIdx.x; i < (n >> 1); i += NT) {
                const int lo = 2 * i - (i & (j - 1));
                const int hi = lo + j;
                const K a = keys[lo], b = keys[hi];
                const bool up = (lo & k) == 0;
                if ((a > b) == up) {
                    keys[lo] = b;
                    keys[hi] = a;
                }
            }
            __syncthreads();
        }
    }
}

// Bitonic sort, ascending, of 32 * E values held E per lane; afterwards lane l holds sorted positions l*E .. l*E+E-1.
// Partners at distance j < E sit in the same lane; partners at distance j >= E in lane l ^ (j / E).
template <int E, typename T>
__device__ __forceinline__ void warp_bitonic_sort(T (&key)[E], int lane) {
#pragma unroll
    for (int k = 2; k <= 32 * E; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j < E) {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int pe = e ^ j;
                    if (pe > e) {
                        const bool up = ((lane * E + e) & k) == 0;
                        const T a = key[e], b = key[pe];
                        const bool swap = (a > b) == up;
                        key[e] = swap ? b : a;
                        key[pe] = swap ? a : b;
                    }
                }
            } else {
                const int dl = j / E;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const T other = __shfl_xor_sync(0xffffffffu, key[e], dl);
                    const bool up = ((lane * E + e) & k) == 0;
                    const bool lower = (lane & dl) == 0;  // this position is the lower index of the pair
                    const T mn = key[e] < other ? key[e] : other;
                    const T mx = key[e] < other ? other : key[e];
                    key[e] = (lower == up) ? mn : mx;
                }
            }
        }
    }
}

// Sort key of block j: high word = bitwise NOT of the fp32 bits (for masses >= 0 ascending keys are descending
// masses), low word = j (ascending among equal masses). A negative, NaN or infinite mass sets bad and counts as 0;
// -0 counts as +0. Padding keys (all ones) sort last.
__device__ __forceinline__ uint64_t sel_key(float x, uint32_t j, bool& bad) {
    uint32_t bits = __float_as_uint(x);
    bits = (bits == 0x80000000u) ? 0u : bits;  // -0 is 0
    const bool ok = bits < 0x7F800000u;          // finite and not negative
    bad |= !ok;
    return ((uint64_t)(~(ok ? bits : 0u)) << 32) | j;
}

// u = ceil(min(M, 2) * 2^52) of a key's mass (0 for the padding key), in integer arithmetic on the fp32 fields:
// M = m24 * 2^(e - 150) for a normal mass, so M * 2^52 = m24 * 2^(e - 98), a shift or a rounded-up shift; a
// subnormal mass is below 2^-126 and gives 1. The result equals ceil(M * 2^52) taken in fp64, which is exact. Masses
// above 2 lie outside the input domain (the row-sum check reports them); the clamp keeps every unit at most 2^53.
__device__ __forceinline__ uint64_t sel_units(uint64_t key) {
    uint32_t bits = ~(uint32_t)(key >> 32);  // fp32 bits of a mass >= 0 (the padding key gives 0)
    bits = bits > 0x40000000u ? 0x40000000u : bits;  // min(M, 2): non-negative floats order as their bits
    const uint32_t e = bits >> 23;
    const uint32_t m = bits & 0x7FFFFFu;
    const uint64_t m24 = (uint64_t)(m | 0x800000u);
    const int sh = (int)e - 98;  // at most 30 after the clamp
    // Both shifts without a branch: the left one for sh >= 0; the rounded-up right one for sh < 0, where a shift by
    // 25 or more (0 < M * 2^52 < 1/2) gives 1 because 2^23 <= m24 < 2^24.
    const uint32_t ls = (uint32_t)(sh > 0 ? sh : 0);
    const uint32_t rs = (uint32_t)(sh < 0 ? (sh < -25 ? 25 : -sh) : 0);
    const uint64_t u = sh >= 0 ? (m24 << ls) : ((m24 + ((1ull << rs) - 1ull)) >> rs);
    return e == 0 ? (m ? 1ull : 0ull) : u;
}

// The same units through the conversion unit: the scaling by 2^52 only moves the exponent (min(M, 2) * 2^52 <= 2^53,
// and a subnormal M becomes a normal number) and the conversion rounds up, so the result is exactly the ceiling; a
// subnormal mass gives 1 whatever the compiler's handling of subnormal operands. Fewer instructions, but the 64-bit
// conversion has a low rate: the shared-memory pick path (latency-bound) uses this form, the register path (issue-
// bound) the integer one.
__device__ __forceinline__ uint64_t sel_units_cvt(uint64_t key) {
    const uint32_t bits = ~(uint32_t)(key >> 32);
    const uint64_t u = __float2ull_ru(fminf(__uint_as_float(bits), 2.0f) * 4503599627370496.0f);
    return (bits - 1u < 0x7FFFFFu) ? 1ull : u;
}

// Per-thread partial of a row total: capped just above the largest valid total, so that sums of partials cannot wrap
// and a capped partial still marks the row as out of the domain.
__device__ __forceinline__ uint64_t cap_units(uint64_t x) { return x > kMaxRowUnits ? kMaxRowUnits + 1 : x; }

__device__ __forceinline__ uint64_t sel_target(double tau, uint64_t total) {
    return (uint64_t)ceil(__dmul_rn(tau, __ull2double_rn(total)));
}

// ------------------------------------------------------------------------------------------------ pick path
// Warp-wide minimum of 64-bit keys with two 32-bit reductions: the high words, then the low words of the lanes that
// hold the smallest high word.
__device__ __forceinline__ uint64_t warp_min_key(uint64_t k) {
    const uint32_t h = (uint32_t)(k >> 32);
    const uint32_t hm = __reduce_min_sync(0xffffffffu, h);
    const uint32_t lm = __reduce_min_sync(0xffffffffu, h == hm ? (uint32_t)k : 0xffffffffu);
    return ((uint64_t)hm << 32) | lm;
}

// Puts key k into the ascending list c (keeping its D smallest entries): one bubble pass.
template <int D>
__device__ __forceinline__ void cache_insert(uint64_t (&c)[D], uint64_t k) {
#pragma unroll
    for (int i = 0; i < D; ++i) {
        const uint64_t lo = k < c[i] ? k : c[i];
        k = k < c[i] ? c[i] : k;
        c[i] = lo;
    }
}

// The pick loop of one row (one warp). c: this lane's smallest unconsumed keys, ascending (all ones where there are
// none), so c[0] is the lane's next candidate; refill(c, w) refills an emptied list with the lane's smallest keys
// above w. Keys are distinct (the block index is their low word), so exactly one lane owns each pick. Returns s (> 0)
// when the cut lies within kPickCap positions, else 0; pick t is left in lane t % 32, slot t / 32 of pk (all ones in
// unused entries).
template <int D, typename Refill>
__device__ __forceinline__ int pick_row(uint64_t (&c)[D], uint64_t target, int want, int lane,
                                        uint32_t (&pk)[kPickSlots], Refill refill) {
    uint64_t run = 0;
#pragma unroll
    for (int p = 0; p < kPickSlots; ++p) pk[p] = 0xffffffffu;
    for (int it = 0; it < kPickCap; ++it) {
        const uint64_t w = warp_min_key(c[0]);
        if (w == ~0ull) return 0;  // no keys left (the cut is always reached before; kept as a guard)
        if (lane == (it & 31)) {
#pragma unroll
            for (int p = 0; p < kPickSlots; ++p)
                if ((it >> 5) == p) pk[p] = (uint32_t)w;
        }
        run += sel_units(w);
        if (c[0] == w) {
#pragma unroll
            for (int i = 0; i + 1 < D; ++i) c[i] = c[i + 1];
            c[D - 1] = ~0ull;
            if (c[0] == ~0ull) refill(c, w);
        }
        if (want ? it + 1 >= want : run >= target) return it + 1;
    }
    return 0;
}

// Writes the s picked block indices of a row in ascending order.
__device__ __forceinline__ void pick_emit(uint32_t (&pk)[kPickSlots], int s, int lane, int32_t* __restrict__ out) {
    if (s <= 32) {  // one pick per lane (slot 0): a 32-entry sort
        uint32_t one[1] = {pk[0]};
        warp_bitonic_sort<1>(one, lane);
        if (lane < s) out[lane] = (int32_t)one[0];
        return;
    }
    warp_bitonic_sort<kPickSlots>(pk, lane);
#pragma unroll
    for (int p = 0; p < kPickSlots; ++p)
        if (lane * kPickSlots + p < s) out[lane * kPickSlots + p] = (int32_t)pk[p];
}

// Kernel 1a, register form for rows of nk <= 32 * E keys (E a power of two <= 32): one warp per row, 8 rows per CTA.
// Lane l loads blocks j = e * 32 + l (coalesced) and keeps only the high word of each key (the bitwise NOT of the
// mass bits; all ones for padding), the index being implied by (e, l): half the registers of full keys, so several
// CTAs share an SM and hide each other's latencies. A row whose cut lies beyond kPickCap positions gets count -1 and
// is sorted by kernel 1b. topk > 0 switches from the mass threshold to a fixed count. Block 0 also clears the order
// kernels' completion counter (it runs before them on the stream).
template <int E>
__global__ void __launch_bounds__(256, 2) select_pick_warp_kernel(const float* __restrict__ mass, int nk, int rows,
                                                                double tau, int topk, int32_t* __restrict__ counts,
                                                                int32_t* __restrict__ staged,
                                                                uint32_t* __restrict__ ticket) {
    if (blockIdx.x == 0 && threadIdx.x == 0) ticket[0] = ticket[1] = 0u;  // the order kernels' counter and max
    const int warp = threadIdx.x >> 5;
    const int lane = (int)lane_id();
    const int row = blockIdx.x * 8 + warp;
    if (row >= rows) return;
    const float* m = mass + (size_t)row * nk;
    uint32_t hi[E];  // high words of the keys of blocks e * 32 + lane
    bool bad = false;
    uint64_t local = 0, c[kPickCacheReg];
#pragma unroll
    for (int i = 0; i < kPickCacheReg; ++i) c[i] = ~0ull;
    float mv[E];  // every load of the row goes out before the first use
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int j = e * 32 + lane;
        mv[e] = (j < nk) ? __ldg(m + j) : 0.0f;
    }
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int j = e * 32 + lane;
        const uint64_t key = (j < nk) ? sel_key(mv[e], (uint32_t)j, bad) : ((0xFFFFFFFFull << 32) | (uint32_t)j);
        hi[e] = (uint32_t)(key >> 32);
        local += sel_units(key);
        cache_insert(c, key);
    }
    const uint64_t total = warp_sum_u64(cap_units(local));
    if (topk == 0 && total > kMaxRowUnits) bad = true;
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&g_device_error, kDevErrBadData);
    const int want = topk > 0 ? (topk < nk ? topk : nk) : 0;
    uint32_t pk[kPickSlots];
    const int s = (want > kPickCap) ? 0 : pick_row(c, sel_target(tau, total), want, lane, pk,
                                                   [&](uint64_t (&cc)[kPickCacheReg], uint64_t w) {
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const uint64_t key = ((uint64_t)hi[e] << 32) | (uint32_t)(e * 32 + lane);
            cache_insert(cc, key > w ? key : ~0ull);
        }
    });
    if (s > 0) pick_emit(pk, s, lane, staged + (size_t)row * nk);
    if (lane == 0) counts[row] = s > 0 ? s : -1;
}

// Kernel 1b, register form: the rows kernel 1a left undecided (count -1), each sorted whole by one warp in registers;
// lane l then holds sorted positions l*E .. l*E+E-1.
template <int E>
__global__ void __launch_bounds__(256) select_sort_warp_kernel(const float* __restrict__ mass, int nk, int rows,
                                                                double tau, int topk, int32_t* __restrict__ counts,
                                                                int32_t* __restrict__ staged) {
    __shared__ uint32_t bitmap_all[8][32];
    const int warp = threadIdx.x >> 5;
    const int lane = (int)lane_id();
    // A grid of at most one CTA per SM walks the rows in chunks of 32: one coalesced load of the chunk's counts, then
    // the undecided rows of the chunk one after another.
    for (int base = (blockIdx.x * 8 + warp) * 32; base < rows; base += gridDim.x * 8 * 32) {
        uint32_t todo = __ballot_sync(0xffffffffu, base + lane < rows && counts[base + lane] < 0);
        for (; todo; todo &= todo - 1u) {
            const int row = base + (__ffs(todo) - 1);
            const float* m = mass + (size_t)row * nk;
            uint64_t key[E];
            bool bad = false;  // reported by kernel 1a, which read the same row
            uint64_t local = 0;
            float mv[E];  // every load of the row goes out before the first use
    #pragma unroll
            for (int e = 0; e < E; ++e) {
                const int j = e * 32 + lane;
                mv[e] = (j < nk) ? __ldg(m + j) : 0.0f;
            }
    #pragma unroll
            for (int e = 0; e < E; ++e) {
                const int j = e * 32 + lane;
                key[e] = (j < nk) ? sel_key(mv[e], (uint32_t)j, bad) : ~0ull;
                local += sel_units(key[e]);
            }
            const uint64_t target = sel_target(tau, warp_sum_u64(cap_units(local)));
            const int want = topk > 0 ? (topk < nk ? topk : nk) : 0;
            int32_t* out = staged + (size_t)row * nk;
            warp_bitonic_sort<E>(key, lane);
            uint64_t ls = 0;
    #pragma unroll
            for (int e = 0; e < E; ++e) ls += sel_units(key[e]);
            const uint64_t incl = warp_incl_scan_u64(cap_units(ls));
            uint64_t run = incl - cap_units(ls);
            int below = 0;
    #pragma unroll
            for (int e = 0; e < E; ++e) {
                run += sel_units(key[e]);
                below += (run < target) ? 1 : 0;
            }
    #pragma unroll
            for (int o = 16; o > 0; o >>= 1) below += __shfl_xor_sync(0xffffffffu, below, o);
            int s = (below + 1 < nk) ? below + 1 : nk;
            if (want) s = want;
            // Kept set (sorted positions < s) -> bitmap by block index -> ascending compaction.
            uint32_t* bitmap = bitmap_all[warp];
            for (int w = lane; w < E; w += 32) bitmap[w] = 0u;
            __syncwarp();
    #pragma unroll
            for (int e = 0; e < E; ++e)
                if (lane * E + e < s) {
                    const uint32_t j = (uint32_t)(key[e] & 0xffffffffu);
                    atomicOr(&bitmap[j >> 5], 1u << (j & 31));
                }
            __syncwarp();
            // Lane l emits the kept blocks among [l*E, l*E + E) at its exclusive prefix of kept counts.
            uint32_t myb = 0;
            const int j0 = lane * E;
    #pragma unroll
            for (int e = 0; e < E; ++e) {
                const int j = j0 + e;
                if (j < nk && ((bitmap[j >> 5] >> (j & 31)) & 1u)) myb |= 1u << e;
            }
            const int cnt = __popc(myb);
            int pre = cnt;
    #pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, pre, o);
                if (lane >= o) pre += y;
            }
            pre -= cnt;
    #pragma unroll
            for (int e = 0; e < E; ++e)
                if ((myb >> e) & 1u) out[pre++] = j0 + e;
            __syncwarp();
            if (lane == 0) counts[row] = s;
            __syncwarp();  // the bitmap is reused by the warp's next row
        }
    }
}

// Kernel 1a for nk > 1024: the pick path with the row in shared memory. W = blockDim.x / 32 warps, one row each;
// warp w keeps its row's sanitised mass bits in nk words of dynamic shared memory (W * nk * 4 bytes). Rows whose cut
// lies beyond kPickCap positions get count -1 for kernel 1b. Block 0 clears the order kernels' completion counter.
__global__ void __launch_bounds__(256) select_pick_smem_kernel(const float* __restrict__ mass, int nk, int rows,
                                                                double tau, int topk, int32_t* __restrict__ counts,
                                                                int32_t* __restrict__ staged,
                                                                uint32_t* __restrict__ ticket) {
    extern __shared__ __align__(16) uint32_t pick_bits[];
    if (blockIdx.x == 0 && threadIdx.x == 0) ticket[0] = ticket[1] = 0u;  // the order kernels' counter and max
    const int warp = threadIdx.x >> 5;
    const int lane = (int)lane_id();
    const int row = blockIdx.x * (int)(blockDim.x >> 5) + warp;
    if (row >= rows) return;
    uint32_t* kb = pick_bits + (size_t)warp * nk;
    const float* m = mass + (size_t)row * nk;
    bool bad = false;
    uint64_t local = 0, c[kPickCacheSmem];
#pragma unroll
    for (int i = 0; i < kPickCacheSmem; ++i) c[i] = ~0ull;
    for (int j0 = lane; j0 < nk; j0 += 32 * 8) {  // eight loads in flight per lane before their first use
        float v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) v[u] = (j0 + 32 * u < nk) ? __ldg(m + j0 + 32 * u) : 0.0f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int j = j0 + 32 * u;
            if (j < nk) {
                const uint64_t k = sel_key(v[u], (uint32_t)j, bad);
                kb[j] = (uint32_t)(k >> 32);
                local += sel_units_cvt(k);
                cache_insert(c, k);
            }
        }
    }
    __syncwarp();
    const uint64_t total = warp_sum_u64(cap_units(local));
    if (topk == 0 && total > kMaxRowUnits) bad = true;
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&g_device_error, kDevErrBadData);
    const int want = topk > 0 ? (topk < nk ? topk : nk) : 0;
    uint32_t pk[kPickSlots];
    const int s = (want > kPickCap) ? 0 : pick_row(c, sel_target(tau, total), want, lane, pk,
                                                   [&](uint64_t (&cc)[kPickCacheSmem], uint64_t w) {
        for (int j = lane; j < nk; j += 32) {
            const uint64_t k = ((uint64_t)kb[j] << 32) | (uint32_t)j;
            cache_insert(cc, k > w ? k : ~0ull);
        }
    });
    if (s > 0) pick_emit(pk, s, lane, staged + (size_t)row * nk);
    if (lane == 0) counts[row] = s > 0 ? s : -1;
}

// Kernel 1b for nk > 1024: one CTA per row left undecided by kernel 1a (count -1; decided rows return at once).
// Dynamic shared memory: n2 uint64 keys + nk bytes of kept flags (n2 = next power of two >= nk).
template <int NT>
__global__ void __launch_bounds__(NT) select_rows_kernel(const float* __restrict__ mass, int nk, int n2, double tau,
                                                          int topk, int32_t* __restrict__ counts,
                                                          int32_t* __restrict__ staged) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint64_t* keys = reinterpret_cast<uint64_t*>(smem_raw);
    uint8_t* kept = smem_raw + (size_t)n2 * sizeof(uint64_t);
    __shared__ uint64_t warp_tot[NT / 32];

    const int row = blockIdx.x;
    if (counts[row] >= 0) return;  // the pick kernel has cut this row (and reported any bad data)
    const float* m = mass + (size_t)row * nk;
    for (int j0 = threadIdx.x; j0 < n2; j0 += NT * 4) {  // four loads in flight per thread before their first use
        float v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = (j0 + NT * u < nk) ? __ldg(m + j0 + NT * u) : 0.0f;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int j = j0 + NT * u;
            if (j >= n2) break;
            uint64_t key = ~0ull;
            if (j < nk) {
                bool bad = false;  // reported by the pick kernel, which read the same row
                key = sel_key(v[u], (uint32_t)j, bad);
                kept[j] = 0;
            }
            keys[j] = key;
        }
    }
    __syncthreads();

    bitonic_sort_smem<NT>(keys, n2);

    // Each thread owns E consecutive sorted positions.
    const int E = n2 / NT > 0 ? n2 / NT : 1;
    const int p0 = threadIdx.x * E;
    uint64_t local = 0;
    for (int e = 0; e < E; ++e)
        if (p0 + e < n2) local += sel_units(keys[p0 + e]);
    uint64_t total;
    const uint64_t before = block_excl_scan_u64<NT>(cap_units(local), warp_tot, total);
    const uint64_t target = sel_target(tau, total);

    // Count sorted positions whose inclusive prefix stays below the target; s = that count + 1.
    uint64_t run = before;
    uint64_t below = 0;
    for (int e = 0; e < E; ++e)
        if (p0 + e < n2) {
            run += sel_units(keys[p0 + e]);
            if (run < target) ++below;
        }
    uint64_t n_below;
    block_excl_scan_u64<NT>(below, warp_tot, n_below);
    int s = (n_below + 1 < (uint64_t)nk) ? (int)(n_below + 1) : nk;
    if (topk > 0) s = topk < nk ? topk : nk;

    for (int p = threadIdx.x; p < s; p += NT) kept[(uint32_t)(keys[p] & 0xffffffffu)] = 1;
    __syncthreads();

    // Compact kept indices in ascending block order: thread t scans block indices [t*F, (t+1)*F).
    const int F = (nk + NT - 1) / NT;
    const int j0 = threadIdx.x * F;
    uint64_t cnt = 0;
    for (int f = 0; f < F; ++f)
        if (j0 + f < nk && kept[j0 + f]) ++cnt;
    uint64_t all;
    uint64_t pos = block_excl_scan_u64<NT>(cnt, warp_tot, all);
    int32_t* out = staged + (size_t)row * nk;
    for (int f = 0; f < F; ++f)
        if (j0 + f < nk && kept[j0 + f]) out[pos++] = j0 + f;
    __syncthreads();
    if (threadIdx.x == 0) counts[row] = s;
}

// ------------------------------------------------------------------------------------- order and indptr
// Rows are cut into nch chunks of kOrderChunk. table is [nk][nch] (bin-major); bin b = nk - count, so ascending bins
// are descending counts.

// Kernel 2 (grid nch, kOrderChunk threads, dynamic shared memory nk int32): histogram of the chunk's counts into its
// column of table, and the chunk's sum of counts. The last chunk to finish turns table into starting positions (an
// exclusive scan in bin-major order) and chunk_off into exclusive prefixes of the chunk sums, writes indptr[rows] and
// clears the completion counter.
__global__ void __launch_bounds__(kOrderChunk) select_hist_kernel(const int32_t* __restrict__ counts, int rows, int nk,
                                                                   int nch, int32_t* __restrict__ table,
                                                                   int64_t* __restrict__ chunk_off,
                                                                   uint32_t* __restrict__ ticket,
                                                                   int32_t* __restrict__ indptr) {
    extern __shared__ __align__(16) int32_t hist[];
    __shared__ uint64_t warp_tot[kOrderChunk / 32];
    __shared__ int is_last;
    for (int b = threadIdx.x; b < nk; b += kOrderChunk) hist[b] = 0;
    __syncthreads();
    const int r = blockIdx.x * kOrderChunk + (int)threadIdx.x;
    int c = 0;
    if (r < rows) {
        c = counts[r];
        if (c < 1 || c > nk) {  // cannot come from kernel 1; clamped so that every index stays in range
            atomicOr(&g_device_error, kDevErrBadData);
            c = c < 1 ? 1 : nk;
        }
        atomicAdd(&hist[nk - c], 1);
    }
    const int cmax = __reduce_max_sync(0xffffffffu, c);
    if ((threadIdx.x & 31u) == 0 && cmax > 0) atomicMax(&ticket[1], (uint32_t)cmax);  // the longest list anywhere
    uint64_t tot;
    block_excl_scan_u64<kOrderChunk>((uint64_t)c, warp_tot, tot);  // also orders the histogram updates
    for (int b = threadIdx.x; b < nk; b += kOrderChunk) table[(size_t)b * nch + blockIdx.x] = hist[b];
    if (threadIdx.x == 0) chunk_off[blockIdx.x] = (int64_t)tot;
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) is_last = (atomicAdd(ticket, 1u) == (uint32_t)nch - 1u);
    __syncthreads();
    if (!is_last) return;
    __threadfence();
    // The last chunk: exclusive scan of table (n = nk * nch entries) in linear order, kScanSeg entries at a time.
    // Each segment is loaded with coalesced reads into shared memory (the histogram space, free again), where every
    // thread scans kScanPer contiguous entries; the running total carries from segment to segment. The bins of counts
    // above the longest list are empty, so the scan starts at the bin of that count: every entry before it is zero
    // and none is read by the order kernel.
    constexpr int kScanPer = 8, kScanSeg = kOrderChunk * kScanPer;
    __shared__ int32_t seg[kScanSeg];  // 32 KB
    const size_t n = (size_t)nk * nch;
    const uint32_t lmax = __ldcg(&ticket[1]);
    const size_t first = (size_t)(nk - (int)(lmax < 1u ? 1u : (lmax > (uint32_t)nk ? (uint32_t)nk : lmax))) * nch;
    uint64_t carry = 0;
    for (size_t s0 = first; s0 < n; s0 += kScanSeg) {
        const int cnt = (int)min((size_t)kScanSeg, n - s0);
#pragma unroll
        for (int u = 0; u < kScanPer; ++u) {
            const int i = u * kOrderChunk + (int)threadIdx.x;
            seg[i] = i < cnt ? __ldcg(table + s0 + i) : 0;
        }
        __syncthreads();
        int32_t v[kScanPer];
        uint64_t loc = 0;
#pragma unroll
        for (int u = 0; u < kScanPer; ++u) {
            v[u] = seg[threadIdx.x * kScanPer + u];
            loc += (uint64_t)v[u];
        }
        uint64_t all;
        uint64_t pre = carry + block_excl_scan_u64<kOrderChunk>(loc, warp_tot, all);  // also orders the reads above
#pragma unroll
        for (int u = 0; u < kScanPer; ++u) {
            seg[threadIdx.x * kScanPer + u] = (int32_t)pre;
            pre += (uint64_t)v[u];
        }
        __syncthreads();
#pragma unroll
        for (int u = 0; u < kScanPer; ++u) {
            const int i = u * kOrderChunk + (int)threadIdx.x;
            if (i < cnt) table[s0 + i] = seg[i];
        }
        carry += all;
        __syncthreads();
    }
    // chunk offsets: exclusive scan of the chunk sums (nch <= kOrderChunk)
    const uint64_t cs = threadIdx.x < (unsigned)nch ? (uint64_t)__ldcg(chunk_off + threadIdx.x) : 0ull;
    uint64_t total;
    const uint64_t cpre = block_excl_scan_u64<kOrderChunk>(cs, warp_tot, total);
    if (threadIdx.x < (unsigned)nch) chunk_off[threadIdx.x] = (int64_t)cpre;
    if (threadIdx.x == 0) {
        indptr[rows] = (int32_t)total;
        ticket[0] = ticket[1] = 0u;
    }
}

// Kernel 3 (grid nch, kOrderChunk threads, dynamic shared memory nk int32): indptr of the chunk's rows, and each row's
// place in the longest-first order: the start of its count's bin for this chunk (from table) plus the rows of the
// same count before it in the chunk. The warps of the chunk take turns in row order, so equal counts keep ascending
// ids.
__global__ void __launch_bounds__(kOrderChunk) select_order_kernel(const int32_t* __restrict__ counts, int rows, int nk,
                                                                    int nch, const int32_t* __restrict__ table,
                                                                    const int64_t* __restrict__ chunk_off,
                                                                    int32_t* __restrict__ indptr,
                                                                    int32_t* __restrict__ order) {
    extern __shared__ __align__(16) int32_t run[];
    __shared__ uint64_t warp_tot[kOrderChunk / 32];
    for (int b = threadIdx.x; b < nk; b += kOrderChunk) run[b] = table[(size_t)b * nch + blockIdx.x];
    const int r = blockIdx.x * kOrderChunk + (int)threadIdx.x;
    int c = 0;
    if (r < rows) {
        c = counts[r];
        c = c < 1 ? 1 : (c > nk ? nk : c);  // out-of-range counts were reported by kernel 2
    }
    uint64_t tot;
    const uint64_t pre = block_excl_scan_u64<kOrderChunk>((uint64_t)c, warp_tot, tot);  // also publishes run[]
    if (r < rows) indptr[r] = (int32_t)((uint64_t)chunk_off[blockIdx.x] + pre);
    const int warp = threadIdx.x >> 5;
    const int lane = (int)lane_id();
    const int b = (r < rows) ? nk - c : -1;
    for (int w = 0; w < kOrderChunk / 32; ++w) {
        if (warp == w) {
            const uint32_t same = __match_any_sync(0xffffffffu, b);
            const uint32_t lower = (1u << lane) - 1u;
            int start = 0;
            if (b >= 0) {
                start = run[b];
                order[start + __popc(same & lower)] = r;
            }
            __syncwarp();
            if (b >= 0 && lane == __ffs(same) - 1) run[b] = start + __popc(same);
        }
        __syncthreads();
    }
}

// Kernel 4: one warp per row copies the staged list to its CSR slot.
__global__ void select_scatter_kernel(const int32_t* __restrict__ staged, const int32_t* __restrict__ counts,
                                      const int32_t* __restrict__ indptr, int rows, int nk,
                                      int32_t* __restrict__ kv_block_idx) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (warp >= rows) return;
    int c = counts[warp];
    c = c < 1 ? 1 : (c > nk ? nk : c);
    const int32_t* src = staged + (size_t)warp * nk;
    int32_t* dst = kv_block_idx + indptr[warp];
    for (int t = lane_id(); t < c; t += 32) dst[t] = src[t];
}

}  // namespace losa
