// Mass-threshold block selection (LoSA page, Methodology Summary, "One-time pattern construction"), and the
// fixed-count top-k rule the page's ablation compares it with (Experiments Summary, "Retained mass vs. a fixed
// sparsity ratio").
//
// Three launches, all stream-ordered:
//   1. select_rows_kernel    one CTA per (head, query block) row: bitonic sort of the row's masses in shared memory
//                            as 64-bit keys (mass descending, block index ascending), integer inclusive scan
//                            (warp shuffles), first crossing of T, then the kept blocks compacted in ascending
//                            index order into a per-row staging slot of the workspace and the count s.
//   2. select_finalize_kernel one CTA: exclusive scan of the counts -> indptr, and the longest-first work order
//                            (bitonic sort of (nk - count, id) keys in shared memory).
//   3. select_scatter_kernel  one warp per row copies its staged indices to kv_block_idx[indptr[row] ...].
#pragma once
#include <cstdint>
#include "ptx.cuh"

namespace losa {

constexpr int kSelectThreads = 256;

__device__ __forceinline__ uint64_t warp_incl_scan_u64(uint64_t x) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if ((int)lane_id() >= o) x += y;
    }
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

// Shared-memory bitonic sort, ascending, of n (power of two) 64-bit keys by NT threads.
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

// Kernel 1. Dynamic shared memory: n2 uint64 keys + nk bytes of kept flags (n2 = next power of two >= nk).
// topk > 0 switches from the mass threshold to a fixed count: keep the topk largest blocks (ties by index).
template <int NT>
__global__ void __launch_bounds__(NT) select_rows_kernel(const float* __restrict__ mass, int nk, int n2, double tau,
                                                          int topk, int32_t* __restrict__ counts,
                                                          int32_t* __restrict__ staged) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint64_t* keys = reinterpret_cast<uint64_t*>(smem_raw);
    uint8_t* kept = smem_raw + (size_t)n2 * sizeof(uint64_t);
    __shared__ uint64_t warp_tot[NT / 32];
    __shared__ int bad_flag;

    const int row = blockIdx.x;
    const float* m = mass + (size_t)row * nk;
    if (threadIdx.x == 0) bad_flag = 0;
    __syncthreads();

    // Keys: high word = bitwise NOT of the fp32 bits (for masses >= 0 this orders by decreasing mass),
    // low word = block index (ascending among equal masses). Padding keys (all ones) sort last.
    for (int j = threadIdx.x; j < n2; j += NT) {
        uint64_t key = ~0ull;
        if (j < nk) {
            float x = m[j];
            if (!(x >= 0.0f) || isinf(x)) {  // negative, NaN or infinite: report, treat as zero
                bad_flag = 1;
                x = 0.0f;
            }
            const uint32_t bits = (x == 0.0f) ? 0u : __float_as_uint(x);
            key = ((uint64_t)(~bits) << 32) | (uint32_t)j;
            kept[j] = 0;
        }
        keys[j] = key;
    }
    __syncthreads();
    if (threadIdx.x == 0 && bad_flag) atomicOr(&g_device_error, kDevErrBadData);

    bitonic_sort_smem<NT>(keys, n2);

    // Each thread owns E consecutive sorted positions. u = ceil(M * 2^52) (exact in fp64).
    const int E = n2 / NT > 0 ? n2 / NT : 1;
    const int p0 = threadIdx.x * E;
    uint64_t local = 0;
    for (int e = 0; e < E; ++e) {
        const int p = p0 + e;
        if (p < n2) {
            const float x = __uint_as_float(~(uint32_t)(keys[p] >> 32));
            local += (uint64_t)ceil((double)x * 4503599627370496.0);
        }
    }
    uint64_t total;
    const uint64_t before = block_excl_scan_u64<NT>(local, warp_tot, total);
    const uint64_t target = (uint64_t)ceil(__dmul_rn(tau, __ull2double_rn(total)));

    // Count sorted positions whose inclusive prefix stays below the target; s = that count + 1.
    uint64_t run = before;
    uint64_t below = 0;
    for (int e = 0; e < E; ++e) {
        const int p = p0 + e;
        if (p < n2) {
            const float x = __uint_as_float(~(uint32_t)(keys[p] >> 32));
            run += (uint64_t)ceil((double)x * 4503599627370496.0);
            if (run < target) ++below;
        }
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
    for (int f = 0; f < F; ++f) {
        const int j = j0 + f;
        if (j < nk && kept[j]) ++cnt;
    }
    uint64_t all;
    uint64_t pos = block_excl_scan_u64<NT>(cnt, warp_tot, all);
    int32_t* out = staged + (size_t)row * nk;
    for (int f = 0; f < F; ++f) {
        const int j = j0 + f;
        if (j < nk && kept[j]) out[pos++] = j;
    }
    if (threadIdx.x == 0) counts[row] = s;
}

// Kernel 1, warp-per-row form for rows of nk <= 32 * E keys (E a power of two <= 32): the same bitonic network held
// in registers. Lane l owns sorted positions [l*E, l*E + E): compare-exchange partners at distance j < E sit in the
// same lane, partners at distance j >= E in lane l ^ (j / E) (exchanged by shuffle). No shared memory or block
// barrier is involved in the sort; the integer prefix is an in-lane scan plus a warp scan of lane totals; the kept
// set is turned into ascending block order through a per-warp bitmap of E words.
template <int E>
__global__ void __launch_bounds__(256) select_rows_warp_kernel(const float* __restrict__ mass, int nk, int rows,
                                                                double tau, int topk, int32_t* __restrict__ counts,
                                                                int32_t* __restrict__ staged) {
    __shared__ uint32_t bitmap_all[8][32];
    const int warp = threadIdx.x >> 5;
    const int lane = (int)lane_id();
    const int row = blockIdx.x * 8 + warp;
    if (row >= rows) return;
    uint32_t* bitmap = bitmap_all[warp];
    const float* m = mass + (size_t)row * nk;
    uint64_t key[E];
    bool bad = false;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        const int j = lane * E + e;
        uint64_t kk = ~0ull;
        if (j < nk) {
            float xv = m[j];
            if (!(xv >= 0.0f) || isinf(xv)) {
                bad = true;
                xv = 0.0f;
            }
            const uint32_t bits = (xv == 0.0f) ? 0u : __float_as_uint(xv);
            kk = ((uint64_t)(~bits) << 32) | (uint32_t)j;
        }
        key[e] = kk;
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) atomicOr(&g_device_error, kDevErrBadData);
    // Bitonic sort, ascending, of the 32 * E keys.
#pragma unroll
    for (int k = 2; k <= 32 * E; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j < E) {
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const int pe = e ^ j;
                    if (pe > e) {
                        const int i = lane * E + e;
                        const bool up = (i & k) == 0;
                        const uint64_t a = key[e], b = key[pe];
                        const bool swap = (a > b) == up;
                        key[e] = swap ? b : a;
                        key[pe] = swap ? a : b;
                    }
                }
            } else {
                const int dl = j / E;
#pragma unroll
                for (int e = 0; e < E; ++e) {
                    const uint64_t other = __shfl_xor_sync(0xffffffffu, key[e], dl);
                    const int i = lane * E + e;
                    const bool up = (i & k) == 0;
                    const bool lower = (lane & dl) == 0;   // this position is the lower index of the pair
                    const uint64_t mn = key[e] < other ? key[e] : other;
                    const uint64_t mx = key[e] < other ? other : key[e];
                    key[e] = (lower == up) ? mn : mx;
                }
            }
        }
    }
    // Integer prefix over sorted positions; u = ceil(M * 2^52) exactly in fp64.
    uint64_t local = 0;
#pragma unroll
    for (int e = 0; e < E; ++e)
        local += (uint64_t)ceil((double)__uint_as_float(~(uint32_t)(key[e] >> 32)) * 4503599627370496.0);
    const uint64_t incl = warp_incl_scan_u64(local);
    const uint64_t total = __shfl_sync(0xffffffffu, incl, 31);
    const uint64_t target = (uint64_t)ceil(__dmul_rn(tau, __ull2double_rn(total)));
    uint64_t run = incl - local;
    int below = 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
        run += (uint64_t)ceil((double)__uint_as_float(~(uint32_t)(key[e] >> 32)) * 4503599627370496.0);
        below += (run < target) ? 1 : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) below += __shfl_xor_sync(0xffffffffu, below, o);
    int s = (below + 1 < nk) ? below + 1 : nk;
    if (topk > 0) s = topk < nk ? topk : nk;
    // Kept set (sorted positions < s) -> bitmap by block index -> ascending compaction.
    for (int w = lane; w < E; w += 32) bitmap[w] = 0u;
    __syncwarp();
#pragma unroll
    for (int e = 0; e < E; ++e)
        if (lane * E + e < s) {
            const uint32_t j = (uint32_t)(key[e] & 0xffffffffu);
            atomicOr(&bitmap[j >> 5], 1u << (j & 31));
        }
    __syncwarp();
    // Lane l emits block indices [l*E, l*E + E) that are kept, at its exclusive prefix of kept counts.
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
    int32_t* out = staged + (size_t)row * nk;
#pragma unroll
    for (int e = 0; e < E; ++e)
        if ((myb >> e) & 1u) out[pre++] = j0 + e;
    if (lane == 0) counts[row] = s;
}

// Kernel 2 (one CTA, NT threads). Dynamic shared memory: n2 uint32 keys (n2 = power of two >= rows).
template <int NT>
__global__ void __launch_bounds__(NT) select_finalize_kernel(const int32_t* __restrict__ counts, int rows, int nk,
                                                              int n2, int32_t* __restrict__ indptr,
                                                              int32_t* __restrict__ order) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw);
    __shared__ uint64_t warp_tot[NT / 32];

    // indptr: exclusive scan of counts, in chunks of NT * E rows.
    const int E = 8;
    uint64_t carry = 0;
    for (int base = 0; base < rows; base += NT * E) {
        const int r0 = base + threadIdx.x * E;
        uint64_t loc = 0;
        for (int e = 0; e < E; ++e)
            if (r0 + e < rows) loc += (uint64_t)counts[r0 + e];
        uint64_t tot;
        uint64_t pre = carry + block_excl_scan_u64<NT>(loc, warp_tot, tot);
        for (int e = 0; e < E; ++e)
            if (r0 + e < rows) {
                indptr[r0 + e] = (int32_t)pre;
                pre += (uint64_t)counts[r0 + e];
            }
        carry += tot;
    }
    if (threadIdx.x == 0) indptr[rows] = (int32_t)carry;

    // Longest-first order: ascending sort of (nk - count) << 17 | id; ids < 2^17, counts <= nk < 2^15.
    for (int i = threadIdx.x; i < n2; i += NT)
        keys[i] = (i < rows) ? (((uint32_t)(nk - counts[i]) << 17) | (uint32_t)i) : 0xffffffffu;
    __syncthreads();
    bitonic_sort_smem<NT>(keys, n2);
    for (int i = threadIdx.x; i < rows; i += NT) order[i] = (int32_t)(keys[i] & 0x1ffffu);
}

// Kernel 3: one warp per row copies the staged list to its CSR slot.
__global__ void select_scatter_kernel(const int32_t* __restrict__ staged, const int32_t* __restrict__ counts,
                                      const int32_t* __restrict__ indptr, int rows, int nk,
                                      int32_t* __restrict__ kv_block_idx) {
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (warp >= rows) return;
    const int c = counts[warp];
    const int32_t* src = staged + (size_t)warp * nk;
    int32_t* dst = kv_block_idx + indptr[warp];
    for (int t = lane_id(); t < c; t += 32) dst[t] = src[t];
}

}  // namespace losa
