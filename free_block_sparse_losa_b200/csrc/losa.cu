// C ABI of the LoSA hot path (declared in include/losa.h): host-side argument checks, TMA descriptor encoding and
// kernel launches. All device work is in the kernels included below; nothing here computes on the host.
#include "losa.h"

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

namespace losa {
// Per-device error word written by kernels (bitwise OR of the codes below), read and cleared by
// losa_get_device_error.
__device__ unsigned int g_device_error = 0;
constexpr unsigned int kDevErrTimeout = 1u;
constexpr unsigned int kDevErrBadData = 2u;
}  // namespace losa

#include "attn_f32.cuh"
#include "attn_tc.cuh"
#include "attn_dense.cuh"
#include "attn_sparse.cuh"
#include "ptx.cuh"
#include "select.cuh"

using namespace losa;

namespace {

unsigned long long g_wait_limit_ns = 2000000000ull;

constexpr long long kMaxSelectItems = 1ll << 20;  // (head, query block) rows per selection call
constexpr int kMaxSelectBlocks = 8192;            // per-row sort in shared memory

bool aligned16(const void* p) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Generic shape consistency (independent of which kernels exist).
losa_status check_shape(const losa_shape* s) {
    if (!s) return LOSA_ERR_INVALID_ARG;
    if (s->heads <= 0 || s->n_tokens <= 0 || s->head_dim <= 0 || s->block_q <= 0 || s->block_k <= 0)
        return LOSA_ERR_INVALID_ARG;
    if (s->n_padded < s->n_tokens || s->n_padded % s->block_q != 0 || s->n_padded % s->block_k != 0)
        return LOSA_ERR_INVALID_ARG;
    // Every query block must hold at least one real row. Key blocks smaller than the query blocks may lie entirely in
    // the padding (they then carry zero mass and are never selected).
    if (s->n_padded - s->n_tokens >= s->block_q) return LOSA_ERR_INVALID_ARG;
    if (s->block_k >= s->block_q && s->n_padded - s->n_tokens >= s->block_k) return LOSA_ERR_INVALID_ARG;
    if (s->dtype != LOSA_DTYPE_BF16 && s->dtype != LOSA_DTYPE_F32) return LOSA_ERR_INVALID_ARG;
    if ((long long)s->heads * s->n_padded * s->head_dim > (1ll << 40)) return LOSA_ERR_INVALID_ARG;
    return LOSA_OK;
}

// Tensor-core path: bf16, head_dim 128, query blocks of 128 rows, key blocks of 128 or 32 keys (the LoSA page's
// experimental setup uses R = 128, C = 32), at most 1024 tiles of 128 keys per head.
bool tc_shape(const losa_shape* s) {
    return s->dtype == LOSA_DTYPE_BF16 && s->head_dim == kTcDim && s->block_q == kTcRows &&
           (s->block_k == kTcRows || s->block_k == 32) && s->n_padded % kTcRows == 0 &&
           s->n_padded / kTcRows <= kMaxMassBlocks;
}

bool f32_shape(const losa_shape* s) {
    return s->dtype == LOSA_DTYPE_F32 && (s->head_dim == 64 || s->head_dim == 128) && s->block_q == s->block_k &&
           (s->block_q == 32 || s->block_q == 64 || s->block_q == 128);
}

losa_status launch_status() {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? LOSA_OK : LOSA_ERR_CUDA;
}

int sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

// cuTensorMapEncodeTiled, looked up once through the runtime (no link-time dependency on the driver library).
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Tensor map over a [rows][128] bf16 matrix, boxes of box_rows rows x 64 columns, 128-byte swizzle.
bool make_tile_map(CUtensorMap* map, const void* ptr, uint64_t rows, uint32_t box_rows = kTcRows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t gdim[2] = {(cuuint64_t)kTcDim, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)kTcDim * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estride[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gdim, gstride, box, estride,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool M, int SUB, bool ONE_PASS = false>
losa_status launch_dense_kernel(int grid, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                const TcArgs& a, cudaStream_t stream) {
    if (cudaFuncSetAttribute(attn_dense_kernel<M, SUB, ONE_PASS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kDnSmem) != cudaSuccess)
        return LOSA_ERR_CUDA;
    attn_dense_kernel<M, SUB, ONE_PASS><<<grid, kTcThreads, kDnSmem, stream>>>(tq, tk, tv, a);
    return launch_status();
}

template <int SUB>
losa_status launch_sparse_kernel(int grid, const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                                 const CUtensorMap& tk32, const CUtensorMap& tv32, const CUtensorMap& to,
                                 const TcArgs& a, cudaStream_t stream) {
    if (cudaFuncSetAttribute(attn_sparse_kernel<SUB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSpSmem) !=
        cudaSuccess)
        return LOSA_ERR_CUDA;
    attn_sparse_kernel<SUB><<<grid, kSpThreads, kSpSmem, stream>>>(tq, tk, tv, tk32, tv32, to, a);
    return launch_status();
}

// Tensor-core path: fills the argument block and launches one persistent CTA per SM, the dense-step kernel
// without a list, the sparse-step kernel with one.
losa_status launch_tc(const losa_shape* s, bool with_mass, const void* q, const void* k, const void* v, float scale,
                      const int32_t* indptr, const int32_t* kv_idx, const int32_t* order, void* o, float* lse,
                      float* mass, cudaStream_t stream, float* mass_part = nullptr) {
    const uint64_t rows = (uint64_t)s->heads * s->n_padded;
    const bool c32 = s->block_k == 32;
    CUtensorMap tq, tk, tv, tk32, tv32;
    if (!make_tile_map(&tq, q, rows) || !make_tile_map(&tk, k, rows) || !make_tile_map(&tv, v, rows))
        return LOSA_ERR_CUDA;
    if (c32 && (!make_tile_map(&tk32, k, rows, 32) || !make_tile_map(&tv32, v, rows, 32))) return LOSA_ERR_CUDA;
    if (!c32) {
        tk32 = tk;
        tv32 = tv;
    }
    TcArgs a;
    a.H = s->heads;
    a.N = s->n_tokens;
    a.Np = s->n_padded;
    a.nq = s->n_padded / kTcRows;
    a.nk = s->n_padded / kTcRows;
    a.nkb = s->n_padded / s->block_k;
    a.n_items = s->heads * a.nq;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.indptr = indptr;
    a.kv_idx = kv_idx;
    a.order = order;
    a.o = static_cast<__nv_bfloat16*>(o);
    a.lse = lse;
    a.mass = mass;
    a.mass_part = mass_part;
    a.wait_limit_ns = g_wait_limit_ns;
    const int sms = sm_count();
    if (sms <= 0) return LOSA_ERR_CUDA;
    if (!indptr) {
        // dense step: one item per CTA at a time, 256-key tiles
        const int dgrid = a.n_items < sms ? a.n_items : sms;
        if (with_mass && mass_part)  // one pass: block sums from the forward, reduced per item (dgrid scratch slots)
            return c32 ? launch_dense_kernel<true, 4, true>(dgrid, tq, tk, tv, a, stream)
                       : launch_dense_kernel<true, 1, true>(dgrid, tq, tk, tv, a, stream);
        if (with_mass)
            return c32 ? launch_dense_kernel<true, 4>(dgrid, tq, tk, tv, a, stream)
                       : launch_dense_kernel<true, 1>(dgrid, tq, tk, tv, a, stream);
        return c32 ? launch_dense_kernel<false, 4>(dgrid, tq, tk, tv, a, stream)
                   : launch_dense_kernel<false, 1>(dgrid, tq, tk, tv, a, stream);
    }
    // retained lists: one persistent CTA per SM, one stream of items each; masses come from dense steps only
    if (with_mass) return LOSA_ERR_UNSUPPORTED;
    const int grid = a.n_items < sms ? (a.n_items > 0 ? a.n_items : 1) : sms;
    CUtensorMap to;  // O rows leave through TMA stores of 64-column boxes
    if (!make_tile_map(&to, o, rows)) return LOSA_ERR_CUDA;
    return c32 ? launch_sparse_kernel<4>(grid, tq, tk, tv, tk32, tv32, to, a, stream)
               : launch_sparse_kernel<1>(grid, tq, tk, tv, tk32, tv32, to, a, stream);
}

template <int D>
losa_status launch_f32(const losa_shape* s, const void* q, const void* k, const void* v, float scale,
                       const int32_t* indptr, const int32_t* kv_idx, const int32_t* order, void* o, float* lse,
                       float* mass, cudaStream_t stream) {
    F32Args a;
    a.q = static_cast<const float*>(q);
    a.k = static_cast<const float*>(k);
    a.v = static_cast<const float*>(v);
    a.H = s->heads;
    a.N = s->n_tokens;
    a.Np = s->n_padded;
    a.R = s->block_q;
    a.C = s->block_k;
    a.nq = s->n_padded / s->block_q;
    a.nk = s->n_padded / s->block_k;
    a.scale = scale;
    a.indptr = indptr;
    a.kv_idx = kv_idx;
    a.order = order;
    a.o = static_cast<float*>(o);
    a.lse = lse;
    const int items = a.H * a.nq;
    const size_t smem_fwd = (size_t)2 * a.C * D * sizeof(float);
    if (cudaFuncSetAttribute(attn_f32_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_fwd) !=
        cudaSuccess)
        return LOSA_ERR_CUDA;
    attn_f32_fwd_kernel<D><<<items, a.R, smem_fwd, stream>>>(a);
    losa_status st = launch_status();
    if (st != LOSA_OK || !mass) return st;
    const size_t smem_mass = (size_t)a.C * D * sizeof(float) + (size_t)a.R * sizeof(float);
    if (cudaFuncSetAttribute(mass_f32_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_mass) !=
        cudaSuccess)
        return LOSA_ERR_CUDA;
    a.indptr = nullptr;
    a.order = nullptr;
    mass_f32_kernel<D><<<items, a.R, smem_mass, stream>>>(a, mass);
    return launch_status();
}

int next_pow2(int n) {
    int p = 1;
    while (p < n) p <<= 1;
    return p;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace of the selection calls: per-row staged lists and counts, then the order kernels' per-chunk histograms,
// chunk offsets and completion counter. Every region starts on a 256-byte boundary.
struct SelectLayout {
    size_t staged, counts, table, chunk_off, ticket, total;
    int nch;
};

SelectLayout select_layout(long long rows, int nk) {
    SelectLayout L;
    L.nch = (int)((rows + kOrderChunk - 1) / kOrderChunk);
    size_t off = 0;
    L.staged = off;
    off += align256((size_t)rows * nk * sizeof(int32_t));
    L.counts = off;
    off += align256((size_t)rows * sizeof(int32_t));
    L.table = off;
    off += align256((size_t)nk * L.nch * sizeof(int32_t));
    L.chunk_off = off;
    off += align256((size_t)L.nch * sizeof(int64_t));
    L.ticket = off;
    off += 256;
    L.total = off;
    return L;
}

size_t select_ws_bytes(const losa_shape* s) {
    const long long rows = (long long)s->heads * (s->n_padded / s->block_q);
    return select_layout(rows, s->n_padded / s->block_k).total;
}

// Kernel 1: the pick path, one warp per row (in registers for nk <= 1024, in shared memory above), then a full sort
// of the rows it leaves undecided (one warp per row in registers, or one CTA per row in shared memory).
losa_status launch_select_rows(const float* mass, int nk, int rows, double tau, int topk, int32_t* counts,
                               int32_t* staged, uint32_t* ticket, cudaStream_t stream) {
    const unsigned wgrid = (unsigned)((rows + 7) / 8);
    const int sms = sm_count();
    const unsigned sgrid = (sms > 0 && (unsigned)sms < wgrid) ? (unsigned)sms : wgrid;  // the sort kernel walks rows
#define LOSA_ROWS_WARP(E)                                                                                        \
    do {                                                                                                         \
        select_pick_warp_kernel<E><<<wgrid, 256, 0, stream>>>(mass, nk, rows, tau, topk, counts, staged, ticket); \
        const losa_status st1 = launch_status();                                                                 \
        if (st1 != LOSA_OK) return st1;                                                                          \
        select_sort_warp_kernel<E><<<sgrid, 256, 0, stream>>>(mass, nk, rows, tau, topk, counts, staged);       \
    } while (0)
    if (nk <= 32) LOSA_ROWS_WARP(1);
    else if (nk <= 64) LOSA_ROWS_WARP(2);
    else if (nk <= 128) LOSA_ROWS_WARP(4);
    else if (nk <= 256) LOSA_ROWS_WARP(8);
    else if (nk <= 512) LOSA_ROWS_WARP(16);
    else if (nk <= 1024) LOSA_ROWS_WARP(32);
#undef LOSA_ROWS_WARP
    else {
        int wpc = (int)(65536 / ((size_t)nk * sizeof(uint32_t)));  // rows (warps) per CTA: at most 64 KB of rows
        wpc = wpc < 1 ? 1 : (wpc > 8 ? 8 : wpc);
        const size_t smem = (size_t)wpc * nk * sizeof(uint32_t);
        if (cudaFuncSetAttribute(select_pick_smem_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
            cudaSuccess)
            return LOSA_ERR_CUDA;
        select_pick_smem_kernel<<<(unsigned)((rows + wpc - 1) / wpc), (unsigned)(32 * wpc), smem, stream>>>(
            mass, nk, rows, tau, topk, counts, staged, ticket);
        losa_status st = launch_status();
        if (st != LOSA_OK) return st;
        const int n2 = next_pow2(nk);
        const size_t smem1 = (size_t)n2 * sizeof(uint64_t) + (size_t)nk;
        if (cudaFuncSetAttribute(select_rows_kernel<kSelectThreads>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem1) != cudaSuccess)
            return LOSA_ERR_CUDA;
        select_rows_kernel<kSelectThreads><<<(unsigned)rows, kSelectThreads, smem1, stream>>>(mass, nk, n2, tau, topk,
                                                                                             counts, staged);
    }
    return launch_status();
}

// The selection shared by losa_select, losa_select_topk and losa_select_noalloc: argument checks, then the
// stream-ordered launches (the rows' cut in two kernels, histograms, order and indptr, scatter). topk > 0 selects a fixed count instead of
// the mass threshold tau. ws is the workspace (at least select_ws_bytes); ws_bytes is its size.
losa_status run_select(const losa_shape* shape, const float* mass, double tau, int topk, int32_t* indptr,
                       int32_t* kv_block_idx, int64_t idx_capacity, int32_t* order, void* ws, size_t ws_bytes,
                       cudaStream_t stream) {
    losa_status st = check_shape(shape);
    if (st != LOSA_OK) return st;
    if (topk == 0 && !(tau > 0.0 && tau <= 1.0)) return LOSA_ERR_INVALID_ARG;
    if (topk < 0) return LOSA_ERR_INVALID_ARG;
    if (!aligned16(mass) || !indptr || !kv_block_idx || !order || !aligned16(ws)) return LOSA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(indptr) | reinterpret_cast<uintptr_t>(kv_block_idx) |
         reinterpret_cast<uintptr_t>(order)) & 3u)
        return LOSA_ERR_INVALID_ARG;
    const int nq = shape->n_padded / shape->block_q, nk = shape->n_padded / shape->block_k;
    const long long rows = (long long)shape->heads * nq;
    // indptr is int32: every row's list, even at its longest, must fit
    if (rows > kMaxSelectItems || nk > kMaxSelectBlocks || rows * nk > 2147483647ll) return LOSA_ERR_UNSUPPORTED;
    if (idx_capacity < rows * nk) return LOSA_ERR_CAPACITY;
    const SelectLayout lay = select_layout(rows, nk);
    if (ws_bytes < lay.total) return LOSA_ERR_CAPACITY;

    uint8_t* w = static_cast<uint8_t*>(ws);
    int32_t* staged = reinterpret_cast<int32_t*>(w + lay.staged);
    int32_t* counts = reinterpret_cast<int32_t*>(w + lay.counts);
    int32_t* table = reinterpret_cast<int32_t*>(w + lay.table);
    int64_t* chunk_off = reinterpret_cast<int64_t*>(w + lay.chunk_off);
    uint32_t* ticket = reinterpret_cast<uint32_t*>(w + lay.ticket);

    if ((st = launch_select_rows(mass, nk, (int)rows, topk ? 1.0 : tau, topk, counts, staged, ticket, stream)) !=
        LOSA_OK)
        return st;
    const size_t hsmem = (size_t)nk * sizeof(int32_t);  // <= 32 KB, beside the kernel's 32 KB scan segment
    if (cudaFuncSetAttribute(select_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)hsmem) !=
        cudaSuccess)
        return LOSA_ERR_CUDA;
    select_hist_kernel<<<(unsigned)lay.nch, kOrderChunk, hsmem, stream>>>(counts, (int)rows, nk, lay.nch, table,
                                                                          chunk_off, ticket, indptr);
    if ((st = launch_status()) != LOSA_OK) return st;
    select_order_kernel<<<(unsigned)lay.nch, kOrderChunk, hsmem, stream>>>(counts, (int)rows, nk, lay.nch, table,
                                                                           chunk_off, indptr, order);
    if ((st = launch_status()) != LOSA_OK) return st;
    const unsigned blocks = (unsigned)((rows * 32 + 255) / 256);
    select_scatter_kernel<<<blocks, 256, 0, stream>>>(staged, counts, indptr, (int)rows, nk, kv_block_idx);
    return launch_status();
}

}  // namespace

extern "C" {

int losa_version(void) { return 100; }

const char* losa_status_string(losa_status st) {
    switch (st) {
        case LOSA_OK: return "LOSA_OK";
        case LOSA_ERR_INVALID_ARG: return "LOSA_ERR_INVALID_ARG";
        case LOSA_ERR_UNSUPPORTED: return "LOSA_ERR_UNSUPPORTED";
        case LOSA_ERR_CAPACITY: return "LOSA_ERR_CAPACITY";
        case LOSA_ERR_CUDA: return "LOSA_ERR_CUDA";
        case LOSA_ERR_DEVICE_FAULT: return "LOSA_ERR_DEVICE_FAULT";
        case LOSA_ERR_TIMEOUT: return "LOSA_ERR_TIMEOUT";
    }
    return "LOSA_ERR_UNKNOWN";
}

void losa_set_wait_limit_ns(uint64_t limit_ns) { g_wait_limit_ns = limit_ns < 1000 ? 1000 : limit_ns; }

losa_status losa_dense_profile(const losa_shape* shape, const void* q, const void* k, const void* v, float scale,
                               void* o, float* lse, float* mass, cudaStream_t stream) {
    losa_status st = check_shape(shape);
    if (st != LOSA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o)) return LOSA_ERR_INVALID_ARG;
    if (mass && !aligned16(lse)) return LOSA_ERR_INVALID_ARG;
    if (lse && !aligned16(lse)) return LOSA_ERR_INVALID_ARG;
    if (mass && !aligned16(mass)) return LOSA_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return LOSA_ERR_INVALID_ARG;
    if (tc_shape(shape)) {
        return launch_tc(shape, mass != nullptr, q, k, v, scale, nullptr, nullptr, nullptr, o, lse, mass, stream);
    }
    if (f32_shape(shape)) {
        if (shape->head_dim == 64)
            return launch_f32<64>(shape, q, k, v, scale, nullptr, nullptr, nullptr, o, lse, mass, stream);
        return launch_f32<128>(shape, q, k, v, scale, nullptr, nullptr, nullptr, o, lse, mass, stream);
    }
    return LOSA_ERR_UNSUPPORTED;
}

size_t losa_dense_profile_workspace_bytes(const losa_shape* shape) {
    if (check_shape(shape) != LOSA_OK || !tc_shape(shape)) return 0;
    const int sms = sm_count();
    if (sms <= 0) return 0;
    return (size_t)sms * (size_t)(shape->n_padded / shape->block_k) * kTcRows * sizeof(float);
}

losa_status losa_dense_profile_ws(const losa_shape* shape, const void* q, const void* k, const void* v, float scale,
                                  void* o, float* lse, float* mass, void* workspace, size_t ws_bytes,
                                  cudaStream_t stream) {
    if (!mass || !tc_shape(shape)) return losa_dense_profile(shape, q, k, v, scale, o, lse, mass, stream);
    losa_status st = check_shape(shape);
    if (st != LOSA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(lse) || !aligned16(mass) ||
        !aligned16(workspace))
        return LOSA_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return LOSA_ERR_INVALID_ARG;
    const size_t need = losa_dense_profile_workspace_bytes(shape);
    if (need == 0) return LOSA_ERR_CUDA;
    if (ws_bytes < need) return LOSA_ERR_CAPACITY;
    return launch_tc(shape, true, q, k, v, scale, nullptr, nullptr, nullptr, o, lse, mass, stream,
                     static_cast<float*>(workspace));
}

size_t losa_select_workspace_bytes(const losa_shape* shape) {
    if (check_shape(shape) != LOSA_OK) return 0;
    return select_ws_bytes(shape);
}

losa_status losa_select(const losa_shape* shape, const float* mass, double tau, int32_t* indptr,
                        int32_t* kv_block_idx, int64_t idx_capacity, int32_t* order, void* workspace,
                        size_t ws_bytes, cudaStream_t stream) {
    return run_select(shape, mass, tau, 0, indptr, kv_block_idx, idx_capacity, order, workspace, ws_bytes, stream);
}

losa_status losa_select_topk(const losa_shape* shape, const float* mass, int32_t k_blocks, int32_t* indptr,
                             int32_t* kv_block_idx, int64_t idx_capacity, int32_t* order, void* workspace,
                             size_t ws_bytes, cudaStream_t stream) {
    if (k_blocks < 1) return LOSA_ERR_INVALID_ARG;
    return run_select(shape, mass, 1.0, k_blocks, indptr, kv_block_idx, idx_capacity, order, workspace, ws_bytes,
                      stream);
}

losa_status losa_sparse_attn(const losa_shape* shape, const void* q, const void* k, const void* v, float scale,
                             const int32_t* indptr, const int32_t* kv_block_idx, const int32_t* order, void* o,
                             float* lse, cudaStream_t stream) {
    losa_status st = check_shape(shape);
    if (st != LOSA_OK) return st;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !indptr || !kv_block_idx)
        return LOSA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(indptr) | reinterpret_cast<uintptr_t>(kv_block_idx) |
         reinterpret_cast<uintptr_t>(order)) & 3u)  // int32 arrays (order may be NULL)
        return LOSA_ERR_INVALID_ARG;
    if (lse && !aligned16(lse)) return LOSA_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return LOSA_ERR_INVALID_ARG;
    if (tc_shape(shape))
        return launch_tc(shape, false, q, k, v, scale, indptr, kv_block_idx, order, o, lse, nullptr, stream);
    if (f32_shape(shape)) {
        if (shape->head_dim == 64)
            return launch_f32<64>(shape, q, k, v, scale, indptr, kv_block_idx, order, o, lse, nullptr, stream);
        return launch_f32<128>(shape, q, k, v, scale, indptr, kv_block_idx, order, o, lse, nullptr, stream);
    }
    return LOSA_ERR_UNSUPPORTED;
}

losa_status losa_get_device_error(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return LOSA_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, g_device_error, sizeof(word)) != cudaSuccess) return LOSA_ERR_CUDA;
    const unsigned int zero = 0;
    if (word && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return LOSA_ERR_CUDA;
    if (word & kDevErrTimeout) return LOSA_ERR_TIMEOUT;
    if (word & kDevErrBadData) return LOSA_ERR_DEVICE_FAULT;
    return LOSA_OK;
}

}  // extern "C"

// Bounded-wait self-test: one thread waits on a barrier whose single expected arrival never happens.
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t addr = smem_addr(&bar);
    if (threadIdx.x == 0) {
        mbar_init(addr, 1);
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) wait_bounded(addr, 0, limit_ns);
    __syncthreads();
}

extern "C" losa_status losa_selftest_wait_timeout(uint32_t limit_ns, cudaStream_t stream) {
    selftest_wait_kernel<<<1, 32, 0, stream>>>((unsigned long long)limit_ns);
    return launch_status();
}

// ------------------------------------------------------------------------------------------------------------------
// Selection without a caller-provided workspace.
//
// Some callers cannot allocate device memory at call time: a serving process that reserved nearly all of the GPU's
// memory for its own pool at start-up (a cudaMalloc then fails or would bypass its accounting), a plugin whose host
// framework owns every buffer and offers no workspace, or a latency-critical path where cudaMalloc / cudaFree may
// synchronise the device. losa_select_noalloc serves them: it runs the same selection kernels as losa_select, but
// their scratch (the per-row staging lists and counts, the order kernels' histograms, chunk offsets and completion
// counter) lives in the fixed device array below, which every GPU that loads this library holds until the process
// exits.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB per device
static __device__ __align__(256) unsigned char g_select_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mutex;
void* g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};  // id of the context the address belongs to

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the calling thread's current context (0 if it cannot be read). A device reset ends the primary context;
// the next one gets a new id, and the library's device code (with the array) is loaded again at a new address.
unsigned long long current_context_id() {
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<CtxGetCurrentFn>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<CtxGetIdFn>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device address of g_select_scratch on the current device. In host code the array's name only stands in for the
// symbol; the address a kernel can use comes from cudaGetSymbolAddress, looked up with that device current, once per
// device and context (the lookup may load this library's device code onto the device).
void* scratch_on_current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(g_scratch_mutex);
    const unsigned long long ctx = current_context_id();
    if (g_scratch_ptr[dev] && ctx != 0 && g_scratch_ctx[dev] == ctx) return g_scratch_ptr[dev];
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_select_scratch) != cudaSuccess) return nullptr;
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = current_context_id();  // the lookup has made the device's context current
    return p;
}

}  // namespace

extern "C" losa_status losa_select_noalloc(const losa_shape* shape, const float* mass, double tau, int32_t* indptr,
                                           int32_t* kv_block_idx, int64_t idx_capacity, int32_t* order,
                                           cudaStream_t stream) {
    losa_status st = check_shape(shape);
    if (st != LOSA_OK) return st;
    // The fixed scratch must hold every region of the selection's workspace for this shape.
    if (select_ws_bytes(shape) > kNoAllocScratchBytes) return LOSA_ERR_CAPACITY;
    void* scratch = scratch_on_current_device();
    if (!scratch) return LOSA_ERR_CUDA;
    // Regions are written before they are read; the one counter that must start at zero is cleared by the call's
    // first kernel. Stale contents from an earlier call need no other clearing.
    return run_select(shape, mass, tau, 0, indptr, kv_block_idx, idx_capacity, order, scratch, kNoAllocScratchBytes,
                      stream);
}
