// Oracle for the LoSA hot path — TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, obviously-correct CPU implementation in fp64 of what the CUDA library computes. Only the
// tests, the smoke check and the benchmark's two CPU legs (its cpu_baseline and its reference arm) may load it.
// It shares no code, header, table or constant with the CUDA path, and the product path never calls it.
//
// Source of every definition: the page "LoSA: Near-Lossless Sparse Attention for Training-Free Video
// Diffusion Acceleration" (m.montaan.com/papers/2608.12032):
//   * Motivation Summary: the dense attention probabilities A = softmax(Q K^T / sqrt(d)) of one head, the
//     partition of queries into blocks of R tokens and keys into blocks of C tokens, the block attention
//     mass M(i, j) = sum over q in block i, k in block j of A(q, k), Recall and Coverage of a pattern.
//   * Methodology Summary, "One-time pattern construction": sort the key blocks of a (head, query block) by
//     decreasing mass; keep the shortest prefix whose mass reaches theta * R (theta = 0.99 by default).
//   * Methodology Summary, "Sparse attention with a frozen pattern": each query attends only to the keys of
//     its retained blocks, with the softmax denominator taken over the retained keys only.
//
// Readings where the page leaves a step open (each is repeated beside the code it governs):
//   R1  Token sequences are padded to Np, a multiple of the block size; keys k >= N do not exist (they take no
//       part in any softmax) and queries q >= N produce no output (written as NaN here).
//   R2  A query block's mass row is divided by R_i, its number of real query rows, so every row of M sums to
//       one; "mass >= theta * R" becomes "normalised mass >= theta", also for the ragged last block.
//   R3  Ties in mass are broken by ascending key-block index.
//   R4  The prefix sum is taken in integers: u_j = ceil(M_j * 2^52) and T = ceil(theta * sum_j u_j); the kept
//       count s is the first m >= 1 whose integer prefix reaches T. This makes the crossing independent of
//       summation order, and theta = 1 keeps exactly the blocks of non-zero mass.
//   R5  Each retained list is emitted in ascending block order.
//   R6  The work order is the item ids h * nq + i sorted by list length, longest first, ties by ascending id.
//
// Layouts: q, k, v are [H][Np][d] row-major (values already rounded to the storage dtype and widened to
// fp32). An "item" is h * nq + i for head h and query block i.

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <numeric>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

const double kNaN = std::numeric_limits<double>::quiet_NaN();

// Logits s_k = scale * <q, k_k> for the listed keys of head h (fp64, plain dot products).
void logits(const float* qrow, const float* kh, int d, double scale, const std::vector<int>& keys,
            std::vector<double>& s) {
    s.resize(keys.size());
    for (size_t t = 0; t < keys.size(); ++t) {
        const float* kr = kh + (size_t)keys[t] * d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += (double)qrow[c] * (double)kr[c];
        s[t] = scale * acc;
    }
}

// ln sum_k exp(s_k), shifted by the maximum for range safety.
double log_sum_exp(const std::vector<double>& s) {
    double m = -std::numeric_limits<double>::infinity();
    for (double x : s) m = std::max(m, x);
    double sum = 0.0;
    for (double x : s) sum += std::exp(x - m);
    return m + std::log(sum);
}

// Softmax-weighted sum of the listed value rows: o = sum_k exp(s_k - lse) v_k.
void weighted_values(const std::vector<double>& s, double lse, const float* vh, int d,
                     const std::vector<int>& keys, double* o) {
    for (int c = 0; c < d; ++c) o[c] = 0.0;
    for (size_t t = 0; t < keys.size(); ++t) {
        const double p = std::exp(s[t] - lse);
        const float* vr = vh + (size_t)keys[t] * d;
        for (int c = 0; c < d; ++c) o[c] += p * (double)vr[c];
    }
}

bool bad_shape(int H, int N, int Np, int d, int R) {
    return H <= 0 || N <= 0 || Np < N || d <= 0 || R <= 0 || Np % R != 0;
}

// Per-row selection shared by the fp32- and fp64-input entry points (reading R3, R4, R5).
template <typename T>
int select_row(const T* m, int nk, double tau, int32_t* out) {
    std::vector<int> ord(nk);
    std::iota(ord.begin(), ord.end(), 0);
    for (int j = 0; j < nk; ++j)
        if (!(m[j] >= (T)0) || std::isinf((double)m[j])) return -1;
    // Input domain: a row of block masses normalised to one (R2), with slack for rounding. A row summing to more than
    // 2 is refused, which also keeps every unit below 2^53 and the row total far from 2^64.
    double row_sum = 0.0;
    for (int j = 0; j < nk; ++j) row_sum += (double)m[j];
    if (row_sum > 2.0) return -1;
    // Decreasing mass, ties by ascending index (R3). Comparison on the stored value itself.
    std::sort(ord.begin(), ord.end(), [&](int a, int b) { return m[a] > m[b] || (m[a] == m[b] && a < b); });
    // Integer units u_j = ceil(M_j * 2^52): scaling by a power of two is exact in fp64, so is ceil.
    std::vector<uint64_t> u(nk);
    uint64_t total = 0;
    for (int j = 0; j < nk; ++j) {
        u[j] = (uint64_t)std::ceil(std::ldexp((double)m[j], 52));
        total += u[j];
    }
    const uint64_t target = (uint64_t)std::ceil(tau * (double)total);
    // Shortest prefix m >= 1 with sum_{r <= m} u_{pi(r)} >= target.
    uint64_t prefix = 0;
    int s = nk;
    for (int r = 0; r < nk; ++r) {
        prefix += u[ord[r]];
        if (prefix >= target) { s = r + 1; break; }
    }
    std::vector<int> kept(ord.begin(), ord.begin() + s);
    std::sort(kept.begin(), kept.end());  // R5
    for (int t = 0; t < s; ++t) out[t] = kept[t];
    return s;
}

}  // namespace

extern "C" {

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

// Dense attention of the listed items (Motivation Summary: A = softmax(Q K^T / sqrt(d)); here the scale is
// an argument). Output o[item][r][c] and lse[item][r] (natural log of the softmax denominator) for the R rows of
// each query block; rows q >= N are NaN (R1). Returns 0, or -1 on bad arguments.
int oracle_dense(int H, int N, int Np, int d, int R, double scale, const float* q, const float* k,
                 const float* v, int n_items, const int32_t* items, double* o, double* lse) {
    if (bad_shape(H, N, Np, d, R) || n_items < 0) return -1;
    const int nq = Np / R;
    std::vector<int> keys(N);
    std::iota(keys.begin(), keys.end(), 0);  // R1: only the N real keys exist
#pragma omp parallel for schedule(dynamic, 1)
    for (int it = 0; it < n_items * R; ++it) {
        const int item = items[it / R], r = it % R;
        const int h = item / nq, i = item % nq, qi = i * R + r;
        double* orow = o + (size_t)it * d;
        if (item < 0 || h >= H || qi >= N) {
            for (int c = 0; c < d; ++c) orow[c] = kNaN;
            lse[it] = kNaN;
            continue;
        }
        std::vector<double> s;
        const size_t head = (size_t)h * Np * d;
        logits(q + head + (size_t)qi * d, k + head, d, scale, keys, s);
        lse[it] = log_sum_exp(s);
        weighted_values(s, lse[it], v + head, d, keys, orow);
    }
    return 0;
}

// Block attention mass of the listed items (Motivation Summary, M(i, j)), divided by the number of real rows
// of query block i (R2): mass[item][j] for j < nk = Np / C. Returns 0, or -1 on bad arguments.
int oracle_mass(int H, int N, int Np, int d, int R, int C, double scale, const float* q, const float* k,
                int n_items, const int32_t* items, double* mass) {
    if (bad_shape(H, N, Np, d, R) || C <= 0 || Np % C != 0 || n_items < 0) return -1;
    const int nq = Np / R, nk = Np / C;
    std::vector<int> keys(N);
    std::iota(keys.begin(), keys.end(), 0);
#pragma omp parallel for schedule(dynamic, 1)
    for (int it = 0; it < n_items; ++it) {
        const int item = items[it], h = item / nq, i = item % nq;
        double* row = mass + (size_t)it * nk;
        for (int j = 0; j < nk; ++j) row[j] = 0.0;
        if (item < 0 || h >= H) continue;
        const size_t head = (size_t)h * Np * d;
        const int rows = std::min(R, N - i * R);  // R_i, the real rows of block i (>= 1 since Np < N + R)
        std::vector<double> s;
        for (int r = 0; r < rows; ++r) {
            const int qi = i * R + r;
            logits(q + head + (size_t)qi * d, k + head, d, scale, keys, s);
            const double l = log_sum_exp(s);
            for (int kk = 0; kk < N; ++kk) row[kk / C] += std::exp(s[kk] - l);  // A(q, k) summed into its block
        }
        for (int j = 0; j < nk; ++j) row[j] /= (double)rows;
    }
    return 0;
}

// Mass-threshold selection (Methodology Summary, one-time pattern construction) on fp32 masses, the form the
// CUDA path stores. counts[row] = s; idx[row * nk + t] for t < s holds the kept blocks, ascending.
// Returns 0, -1 if tau is outside (0, 1] or a mass is negative / not finite.
int oracle_select_f32(int nk, int n_rows, const float* mass, double tau, int32_t* counts, int32_t* idx) {
    if (!(tau > 0.0 && tau <= 1.0) || nk <= 0 || n_rows < 0) return -1;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 16) reduction(| : bad)
    for (int r = 0; r < n_rows; ++r) {
        const int s = select_row(mass + (size_t)r * nk, nk, tau, idx + (size_t)r * nk);
        counts[r] = s;
        if (s < 0) bad = 1;
    }
    return bad ? -1 : 0;
}

// The same rule on fp64 masses (used by the oracle's own self-checks).
int oracle_select_f64(int nk, int n_rows, const double* mass, double tau, int32_t* counts, int32_t* idx) {
    if (!(tau > 0.0 && tau <= 1.0) || nk <= 0 || n_rows < 0) return -1;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 16) reduction(| : bad)
    for (int r = 0; r < n_rows; ++r) {
        const int s = select_row(mass + (size_t)r * nk, nk, tau, idx + (size_t)r * nk);
        counts[r] = s;
        if (s < 0) bad = 1;
    }
    return bad ? -1 : 0;
}

// Fixed-count selection (the LoSA page's ablation baseline, Experiments Summary, "Retained mass vs. a fixed sparsity
// ratio"): each row keeps its k largest-mass blocks, ties to the lower index (R3), listed ascending (R5).
int oracle_select_topk(int nk, int n_rows, const float* mass, int k, int32_t* counts, int32_t* idx) {
    if (nk <= 0 || n_rows < 0 || k < 1) return -1;
    const int s = std::min(k, nk);
#pragma omp parallel for schedule(dynamic, 16)
    for (int r = 0; r < n_rows; ++r) {
        const float* m = mass + (size_t)r * nk;
        std::vector<int> ord(nk);
        std::iota(ord.begin(), ord.end(), 0);
        std::sort(ord.begin(), ord.end(), [&](int a, int b) { return m[a] > m[b] || (m[a] == m[b] && a < b); });
        std::vector<int> kept(ord.begin(), ord.begin() + s);
        std::sort(kept.begin(), kept.end());
        for (int t = 0; t < s; ++t) idx[(size_t)r * nk + t] = kept[t];
        counts[r] = s;
    }
    return 0;
}

// Longest-first work order (R6): item ids sorted by count descending, ties by ascending id.
int oracle_lpt_order(int n, const int32_t* counts, int32_t* order) {
    if (n < 0) return -1;
    std::vector<int> ids(n);
    std::iota(ids.begin(), ids.end(), 0);
    std::stable_sort(ids.begin(), ids.end(), [&](int a, int b) { return counts[a] > counts[b]; });
    for (int t = 0; t < n; ++t) order[t] = ids[t];
    return 0;
}

// Attention restricted to the retained key blocks (Methodology Summary, sparse attention with a frozen
// pattern): for a query of block i of head h, K(q) = the real keys (R1) of the blocks listed in
// kv_idx[indptr[h*nq+i] .. indptr[h*nq+i+1]); the softmax denominator runs over K(q) only.
// Output layout as oracle_dense. Returns 0, or -1 on bad arguments / an out-of-range block index.
int oracle_sparse(int H, int N, int Np, int d, int R, int C, double scale, const float* q, const float* k,
                  const float* v, const int32_t* indptr, const int32_t* kv_idx, int n_items,
                  const int32_t* items, double* o, double* lse) {
    if (bad_shape(H, N, Np, d, R) || C <= 0 || Np % C != 0 || n_items < 0) return -1;
    const int nq = Np / R, nk = Np / C;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int it = 0; it < n_items; ++it) {
        const int item = items[it], h = item / nq, i = item % nq;
        std::vector<int> keys;
        for (int t = indptr[item]; t < indptr[item + 1]; ++t) {
            const int j = kv_idx[t];
            if (j < 0 || j >= nk) { bad = 1; continue; }
            for (int kk = j * C; kk < (j + 1) * C && kk < N; ++kk) keys.push_back(kk);
        }
        const size_t head = (size_t)h * Np * d;
        std::vector<double> s;
        for (int r = 0; r < R; ++r) {
            const int qi = i * R + r;
            const size_t row = (size_t)it * R + r;
            if (qi >= N || keys.empty()) {
                for (int c = 0; c < d; ++c) o[row * d + c] = kNaN;
                lse[row] = kNaN;
                continue;
            }
            logits(q + head + (size_t)qi * d, k + head, d, scale, keys, s);
            lse[row] = log_sum_exp(s);
            weighted_values(s, lse[row], v + head, d, keys, o + row * d);
        }
    }
    return bad ? -1 : 0;
}

// Recall of a pattern under masses M (Motivation Summary): sum of retained mass over the listed rows divided
// by their total mass. mass is [n_rows][nk] fp64; the CSR rows are indptr[rows[t]] .. for t < n_rows.
double oracle_recall(int nk, int n_rows, const double* mass, const int32_t* indptr, const int32_t* kv_idx,
                     const int32_t* rows) {
    double kept = 0.0, total = 0.0;
    for (int t = 0; t < n_rows; ++t) {
        const double* m = mass + (size_t)t * nk;
        for (int j = 0; j < nk; ++j) total += m[j];
        const int r = rows[t];
        for (int e = indptr[r]; e < indptr[r + 1]; ++e) kept += m[kv_idx[e]];
    }
    return total > 0.0 ? kept / total : 0.0;
}

}  // extern "C"
