// Exact fp32 attention kernels (CUDA cores) for the small fp32 configuration: dense forward, block masses and
// block-sparse forward. One CTA per (head, query block), one thread per query row; key/value blocks are staged in
// shared memory. These keep full fp32 precision (expf, fp32 dot products): the tensor-core tf32 format would
// truncate the logits to 10 mantissa bits, too coarse for the 1e-4 relative mass tolerance.
#pragma once
#include <cstdint>
#include "ptx.cuh"

namespace losa {

struct F32Args {
    const float* q;
    const float* k;
    const float* v;
    int H, N, Np, R, C, nq, nk;
    float scale;
    const int32_t* indptr;   // null: dense (all nk blocks in order)
    const int32_t* kv_idx;
    const int32_t* order;    // null: blockIdx.x is the item id
    float* o;
    float* lse;              // may be null
};

// Online-softmax forward over the listed key blocks. Dynamic shared memory: 2 * C * D floats.
template <int D>
__global__ void __launch_bounds__(128) attn_f32_fwd_kernel(const F32Args a) {
    extern __shared__ __align__(16) float sm_f32[];
    float* ks = sm_f32;
    float* vs = sm_f32 + (size_t)a.C * D;
    const int item = a.order ? a.order[blockIdx.x] : (int)blockIdx.x;
    if (item < 0 || item >= a.H * a.nq) {  // not a permutation of the items: report it and skip the entry
        if (threadIdx.x == 0) atomicOr(&g_device_error, kDevErrBadData);
        return;
    }
    const int h = item / a.nq, i = item % a.nq;
    const int r = threadIdx.x;
    const int qi = i * a.R + r;
    const bool active = r < a.R;
    const size_t head = (size_t)h * a.Np * D;

    float qreg[D];
    float acc[D];
#pragma unroll
    for (int c = 0; c < D; ++c) {
        qreg[c] = active ? a.q[head + (size_t)qi * D + c] * a.scale : 0.0f;
        acc[c] = 0.0f;
    }
    float m = -INFINITY, l = 0.0f;

    const int begin = a.indptr ? a.indptr[item] : 0;
    const int count = a.indptr ? a.indptr[item + 1] - begin : a.nk;
    if (a.indptr && count <= 0 && threadIdx.x == 0) atomicOr(&g_device_error, kDevErrBadData);
    for (int t = 0; t < count; ++t) {
        const int j = a.indptr ? a.kv_idx[begin + t] : t;
        if (j < 0 || j >= a.nk) {
            if (threadIdx.x == 0) atomicOr(&g_device_error, kDevErrBadData);
            continue;  // uniform across the CTA
        }
        __syncthreads();
        for (int e = threadIdx.x; e < a.C * D; e += blockDim.x) {
            ks[e] = a.k[head + (size_t)j * a.C * D + e];
            vs[e] = a.v[head + (size_t)j * a.C * D + e];
        }
        __syncthreads();
        const int kend = min(a.C, a.N - j * a.C);  // keys t >= N do not exist
        if (!active) continue;
        for (int c = 0; c < kend; ++c) {
            float s = 0.0f;
#pragma unroll
            for (int e = 0; e < D; ++e) s = fmaf(qreg[e], ks[c * D + e], s);
            if (s > m) {
                const float alpha = expf(m - s);
                l *= alpha;
#pragma unroll
                for (int e = 0; e < D; ++e) acc[e] *= alpha;
                m = s;
            }
            const float p = expf(s - m);
            l += p;
#pragma unroll
            for (int e = 0; e < D; ++e) acc[e] = fmaf(p, vs[c * D + e], acc[e]);
        }
    }
    if (!active) return;
    const float inv = 1.0f / l;
    float* orow = a.o + head + (size_t)qi * D;
#pragma unroll
    for (int e = 0; e < D; ++e) orow[e] = acc[e] * inv;
    if (a.lse) a.lse[(size_t)h * a.Np + qi] = m + logf(l);
}

// Block masses from a known log-sum-exp: mass[item][j] = (1 / R_i) sum_{real q in block i} sum_{real k in block j}
// exp(s_qk - lse_q). Dynamic shared memory: C * D floats + blockDim floats for the row reduction.
template <int D>
__global__ void __launch_bounds__(128) mass_f32_kernel(const F32Args a, float* __restrict__ mass) {
    extern __shared__ __align__(16) float sm_f32[];
    float* ks = sm_f32;
    float* red = sm_f32 + (size_t)a.C * D;
    const int item = blockIdx.x;
    const int h = item / a.nq, i = item % a.nq;
    const int r = threadIdx.x;
    const int qi = i * a.R + r;
    const bool valid = r < a.R && qi < a.N;
    const int rows = min(a.R, a.N - i * a.R);
    const size_t head = (size_t)h * a.Np * D;

    float qreg[D];
#pragma unroll
    for (int c = 0; c < D; ++c) qreg[c] = valid ? a.q[head + (size_t)qi * D + c] * a.scale : 0.0f;
    const float lse = valid ? a.lse[(size_t)h * a.Np + qi] : 0.0f;

    for (int j = 0; j < a.nk; ++j) {
        __syncthreads();
        for (int e = threadIdx.x; e < a.C * D; e += blockDim.x) ks[e] = a.k[head + (size_t)j * a.C * D + e];
        __syncthreads();
        float sum = 0.0f;
        if (valid) {
            const int kend = min(a.C, a.N - j * a.C);
            for (int c = 0; c < kend; ++c) {
                float s = 0.0f;
#pragma unroll
                for (int e = 0; e < D; ++e) s = fmaf(qreg[e], ks[c * D + e], s);
                sum += expf(s - lse);
            }
        }
        red[threadIdx.x] = sum;
        __syncthreads();
        for (int w = blockDim.x >> 1; w > 0; w >>= 1) {
            if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
            __syncthreads();
        }
        if (threadIdx.x == 0) mass[(size_t)item * a.nk + j] = red[0] / (float)rows;
    }
}

}  // namespace losa
