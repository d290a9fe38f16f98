/*
 * losa.h — C ABI of the LoSA hot path on NVIDIA B200 (sm_100a).
 *
 * The method is the one of the page "LoSA: Near-Lossless Sparse Attention for Training-Free Video Diffusion
 * Acceleration": at one dense denoising step, measure the exact attention mass of every (head, query block,
 * key block); for each head and query block keep the smallest set of key blocks whose mass reaches a
 * threshold tau; at every later step run block-sparse attention over those frozen blocks only.
 *
 * Conventions shared by every entry point:
 *   - Every pointer argument is DEVICE memory owned by the caller (allocated on the current device). The
 *     library allocates nothing and keeps no state between calls other than one per-device error word (and the
 *     fixed scratch array of losa_select_noalloc).
 *   - Every call is asynchronous and stream-ordered on `stream`, except losa_get_device_error (which
 *     synchronises the stream). Host-side argument checks run first and return before anything is launched.
 *   - Token tensors q, k, v, o are [H][Np][d] row-major, d contiguous: head h, token t starts at element
 *     (h * Np + t) * d. Tokens are the video latent's (t, y, x) grid flattened row-major, padded from N to Np
 *     (a multiple of the block sizes, N <= Np < N + block_q). Keys t >= N take no part in any softmax; output
 *     rows t >= N are written but carry no meaning. Base pointers must be 16-byte aligned.
 *   - An "item" is one (head, query block) pair with id h * nq + i, nq = Np / block_q, nk = Np / block_k.
 *   - A batch (several samples, or the conditional and unconditional branches of classifier-free guidance) is passed
 *     as heads = B * H with tensors [B][H][Np][d]: every (sample or branch, head) gets its own pattern, as the LoSA
 *     page's Methodology Summary keeps separate patterns for the two guidance branches.
 *   - Status codes below; LOSA_ERR_CUDA covers launch failures reported by the CUDA runtime.
 *
 * Supported shapes: dtype BF16 with head_dim 128, block_q = 128 and block_k = 128 or 32 (tensor-core path; 32 is the
 * LoSA page's key-block size), or dtype F32 with head_dim 64 or 128 and block_q = block_k in {32, 64, 128} (exact fp32
 * path for small checks). Size limits: the tensor-core path takes Np <= 131072 (1024 blocks of 128 tokens per head);
 * the selection calls take nk <= 8192 key blocks per row, H * nq <= 1048576 items per call and H * nq * nk < 2^31
 * (the CSR offsets are int32). Any other valid shape returns LOSA_ERR_UNSUPPORTED before anything is launched.
 */
#ifndef LOSA_H
#define LOSA_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LOSA_OK = 0,
    LOSA_ERR_INVALID_ARG = -1,   /* null / misaligned pointer, inconsistent shape, tau outside (0, 1]      */
    LOSA_ERR_UNSUPPORTED = -2,   /* a valid shape the library has no kernel for                         */
    LOSA_ERR_CAPACITY = -3,      /* an output or workspace buffer is smaller than the worst case          */
    LOSA_ERR_CUDA = -4,          /* the CUDA runtime reported an error at launch or synchronisation      */
    LOSA_ERR_DEVICE_FAULT = -5,  /* a kernel detected invalid data (bad block index, non-finite mass)   */
    LOSA_ERR_TIMEOUT = -6        /* a kernel's bounded wait ran out; the kernel exited cleanly           */
} losa_status;

enum { LOSA_DTYPE_F32 = 0, LOSA_DTYPE_BF16 = 1 };

typedef struct {
    int32_t heads;     /* H                                                        */
    int32_t n_tokens;  /* N, real tokens                                            */
    int32_t n_padded;  /* Np, multiple of block_q and block_k, N <= Np < N + block_q */
    int32_t head_dim;  /* d                                                        */
    int32_t block_q;   /* R, query block size                                       */
    int32_t block_k;   /* C, key/value block size                                   */
    int32_t dtype;     /* LOSA_DTYPE_BF16 or LOSA_DTYPE_F32, for q, k, v and o      */
} losa_shape;

/*
 * Dense profiling step (LoSA page, Motivation Summary: A = softmax(Q K^T / sqrt(d)) and the block attention
 * mass M(i, j) = sum over q in query block i and k in key block j of A(q, k); Methodology Summary: the masses are
 * exact because construction coincides with a dense step).
 *   q, k, v  : [H][Np][d] input tokens (dtype of the shape).
 *   scale    : logit scale, normally 1 / sqrt(d).
 *   o        : [H][Np][d] output, dense softmax attention (same dtype).
 *   lse      : [H][Np] fp32, natural log of each row's softmax denominator, ln sum_k exp(scale q.k).
 *              May be NULL only when mass is NULL.
 *   mass     : [H][nq][nk] fp32 or NULL. Row (h, i) is M(i, .) divided by R_i, the real rows of query block i,
 *              so every row sums to one. NULL runs the forward pass only (an ordinary dense step).
 * With mass != NULL a second pass recomputes Q K^T tile by tile and sums exp(s - lse) into block sums without
 * materialising the probability matrix.
 */
losa_status losa_dense_profile(const losa_shape* shape, const void* q, const void* k, const void* v, float scale,
                               void* o, float* lse, float* mass, cudaStream_t stream);

/*
 * The dense profiling step with the masses taken in the same pass as the forward, at the cost of a scratch buffer:
 * the same arguments and results as losa_dense_profile (same definitions; the masses agree with it and with the exact
 * values within the same 1e-4 relative bound, not bit for bit: the sums run in another order).
 *   workspace : device scratch of at least losa_dense_profile_workspace_bytes(shape) bytes (16-byte aligned),
 *               contents on entry irrelevant; ws_bytes is its size, else LOSA_ERR_CAPACITY before any launch
 *               (LOSA_ERR_CUDA if the current device cannot be queried for its SM count). The scratch is used
 *               only during the call; concurrent calls need separate workspaces.
 * The forward pass already forms every weight 2^(s c - m c) against the row's running max m; it keeps, per row and
 * key block, the exact sum of those weights (brought to one anchor max per row) in the scratch, and each item's
 * masses are reduced from them once the row's final log-sum-exp is known: one pass over the keys instead of two.
 * With mass == NULL, or on the fp32 path, the call is losa_dense_profile and the workspace is not touched.
 */
losa_status losa_dense_profile_ws(const losa_shape* shape, const void* q, const void* k, const void* v, float scale,
                                  void* o, float* lse, float* mass, void* workspace, size_t ws_bytes,
                                  cudaStream_t stream);

/* Scratch bytes losa_dense_profile_ws needs on the current device (SM count x nk x 128 fp32); 0 for an invalid
 * shape or the fp32 path. */
size_t losa_dense_profile_workspace_bytes(const losa_shape* shape);

/*
 * Mass-threshold selection (LoSA page, Methodology Summary, "One-time pattern construction": sort the key
 * blocks of one (head, query block) by decreasing mass and keep the shortest prefix whose mass reaches
 * theta times the block's total).
 *   mass          : [H][nq][nk] fp32 rows normalised to one, as losa_dense_profile writes them: every entry finite
 *                   and >= 0, every row summing to at most 2 (the slack covers rounding).
 *   tau           : retained-mass threshold in (0, 1].
 *   indptr        : [H*nq + 1] int32 output; row r's kept blocks are kv_block_idx[indptr[r] .. indptr[r+1]).
 *                   indptr[H*nq] = nnz stays on the device; reading it back is the caller's choice.
 *   kv_block_idx  : [idx_capacity] int32 output, kept key-block indices of each row in ascending order.
 *   idx_capacity  : must be >= H*nq*nk (the worst case), else LOSA_ERR_CAPACITY.
 *   order         : [H*nq] int32 output, item ids by list length descending, ties by ascending id (the
 *                   longest-first work order losa_sparse_attn consumes).
 *   workspace     : device scratch of at least losa_select_workspace_bytes(shape) bytes (16-byte aligned);
 *                   its contents on entry do not matter.
 * Rule per row: order blocks by (mass descending, index ascending); u_j = ceil(M_j * 2^52) as 64-bit integers;
 * T = ceil(tau * sum_j u_j) in IEEE double; keep the first s >= 1 blocks whose integer prefix reaches T. The
 * integer prefix makes the result independent of summation order, and tau = 1 keeps exactly the non-zero blocks.
 * A negative or non-finite mass sets the device error word (LOSA_ERR_DEVICE_FAULT) and is treated as zero. A row
 * summing to more than 2 sets it too, and that row's list is unspecified (units are formed from min(M_j, 2), so
 * nothing overflows and no arithmetic is undefined). Five stream-ordered launches: the per-row cut (a pick pass for
 * rows that keep up to 128 blocks, then a full sort of the rows it leaves undecided), per-chunk histograms of the list
 * lengths, indptr with the work order, and the copy of the lists into place.
 */
losa_status losa_select(const losa_shape* shape, const float* mass, double tau, int32_t* indptr,
                        int32_t* kv_block_idx, int64_t idx_capacity, int32_t* order, void* workspace,
                        size_t ws_bytes, cudaStream_t stream);

/*
 * Fixed-count selection, the ablation baseline of the LoSA page (Experiments Summary, "Retained mass vs. a fixed
 * sparsity ratio": keep the same number of blocks in every row, matched to the mass rule's mean coverage).
 * Same arguments, outputs and ordering as losa_select, with k_blocks (>= 1; rows keep min(k_blocks, nk)) in place of
 * tau: each row keeps its k_blocks largest-mass blocks (ties to the lower index), listed in ascending order.
 */
losa_status losa_select_topk(const losa_shape* shape, const float* mass, int32_t k_blocks, int32_t* indptr,
                             int32_t* kv_block_idx, int64_t idx_capacity, int32_t* order, void* workspace,
                             size_t ws_bytes, cudaStream_t stream);

/* Bytes of device workspace losa_select needs for this shape (0 if the shape is invalid). */
size_t losa_select_workspace_bytes(const losa_shape* shape);

/*
 * losa_select without a workspace argument, for callers that cannot allocate device memory when they call: for
 * example a server that reserved almost all device memory for its own pool at start-up, a plugin whose host
 * framework owns every buffer, or a latency-critical path where cudaMalloc / cudaFree may synchronise the device.
 * The pages have no counterpart of this entry point; it exists for such callers only.
 *   Arguments and results are those of losa_select (same kernels, same output, bit for bit); there is no workspace.
 *   Scratch: a fixed 16 MiB device array inside the library, present on every GPU that loads it until the process
 *   exits. Shapes whose scratch need (losa_select_workspace_bytes) exceeds 16 MiB return LOSA_ERR_CAPACITY: that
 *   admits H * nq * nk up to about 4.1 million (a 12-head layer of 256 x 256 blocks needs 3.2 MB).
 *   The library allocates nothing in this call. Its first call on a device (and the first after a device reset, which
 *   loads the library's device code again) looks up the array's device address, which may load the library's device
 *   code onto that device, so make that first call before any stream capture. The call's first kernel clears the two
 *   words in the array that must start at zero (a completion counter and the longest list length).
 *   Every call on a device shares the one array and overwrites what the previous call left there: calls whose GPU
 *   work can overlap (different streams without ordering between them) race on it and must be serialised.
 */
losa_status losa_select_noalloc(const losa_shape* shape, const float* mass, double tau, int32_t* indptr,
                                int32_t* kv_block_idx, int64_t idx_capacity, int32_t* order, cudaStream_t stream);

/*
 * Block-sparse attention over a frozen pattern (LoSA page, Methodology Summary, "Sparse attention with a frozen
 * pattern": each query attends only to the keys of its retained blocks, and the softmax denominator runs over
 * those keys only).
 *   q, k, v       : [H][Np][d] tokens of the current step (they may differ from the profiled step's).
 *   indptr, kv_block_idx : the CSR lists written by losa_select (any order within a row is accepted; every
 *                   index must lie in [0, nk), every row must be non-empty). indptr must be non-decreasing, and
 *                   its last entry must not exceed the length of kv_block_idx: the library cannot check the
 *                   latter (it is not told that length), and a violation is undefined behaviour.
 *   order         : [H*nq] permutation of item ids giving the work order (longest list first for balance),
 *                   or NULL for ascending item order. An entry outside [0, H*nq) is reported and its slot skipped
 *                   before the entry is used (losa_select always writes a valid permutation).
 *   o             : [H][Np][d] output; lse: [H][Np] fp32 output or NULL.
 *   indptr, kv_block_idx and order are int32 arrays and must be 4-byte aligned (else LOSA_ERR_INVALID_ARG).
 * An out-of-range block index, an empty row, a decreasing indptr or a bad work-order entry sets the device error
 * word (LOSA_ERR_DEVICE_FAULT); the affected rows are left unspecified, every other row is computed.
 * O is the restricted softmax times V with the weights rounded to bf16 for the tensor core and divided by their own
 * sum (so O is a convex combination of the listed V rows); lse uses the exact fp32 sum.
 */
losa_status losa_sparse_attn(const losa_shape* shape, const void* q, const void* k, const void* v, float scale,
                             const int32_t* indptr, const int32_t* kv_block_idx, const int32_t* order, void* o,
                             float* lse, cudaStream_t stream);

/*
 * Synchronises `stream`, then returns and clears the current device's error word: LOSA_OK,
 * LOSA_ERR_DEVICE_FAULT, LOSA_ERR_TIMEOUT, or LOSA_ERR_CUDA if the synchronisation itself failed.
 */
losa_status losa_get_device_error(cudaStream_t stream);

/*
 * Self-test of the bounded-wait path: launches one block that waits on a shared-memory barrier nothing ever
 * completes, for at most `limit_ns` nanoseconds, then records LOSA_ERR_TIMEOUT in the device error word and
 * exits. No GPU fault is involved; read the result with losa_get_device_error.
 */
losa_status losa_selftest_wait_timeout(uint32_t limit_ns, cudaStream_t stream);

/*
 * Upper bound, in nanoseconds, of every wait inside the library's kernels on this process (default 2e9).
 * Exposed for tests; values below 1000 are raised to 1000.
 */
void losa_set_wait_limit_ns(uint64_t limit_ns);

/* Human-readable name of a status code (static string). */
const char* losa_status_string(losa_status status);

/* Library version as major * 10000 + minor * 100 + patch. */
int losa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LOSA_H */
