"""Pins of the fp64 oracle to things other than itself (CPU only).

Every check is a closed form, an invariant the method guarantees, a hand-worked example from
tests/golden/, brute force on tiny inputs, or a special case that reduces to a library routine
(torch's float64 scaled-dot-product attention and logsumexp). A plausible mistake in the oracle —
a transposed operand, a wrong scale, an unmasked padded key, a wrong tail normalisation, a wrong
tie-break or an off-by-one in the prefix cut — fails at least one of them.

Definitions: "LoSA: Near-Lossless Sparse Attention for Training-Free Video Diffusion Acceleration",
Motivation Summary (A, M, Recall, Coverage) and Methodology Summary (selection rule; attention over
the frozen pattern).
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from losa_synth import CONFIGS, make_layer, round_to_bf16, f32_to_bf16_bits, bf16_bits_to_f32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_qkv(rng, H, N, Np, d, q_scale=1.0, k_scale=1.0):
    q = np.zeros((H, Np, d), np.float32)
    k = np.zeros((H, Np, d), np.float32)
    v = np.zeros((H, Np, d), np.float32)
    q[:, :N] = rng.standard_normal((H, N, d)) * q_scale
    k[:, :N] = rng.standard_normal((H, N, d)) * k_scale
    v[:, :N] = rng.standard_normal((H, N, d))
    return q, k, v


# Tolerance against the library's float64 attention. That reference (torch on the CPU) is not bitwise reproducible
# from run to run under CPU load: 1 run in 160 measured here changed its log-sum-exp by up to 5.3e-10 (relative
# 7e-11), while the oracle's output bits never changed. 1e-9 still sits many orders of magnitude below what a dropped
# term, a wrong sign or a transposed operand produces (1e-3 and up); comparisons with closed forms stay at 1e-12.
LIB_ATOL = 1e-9


def _torch_attention(q, k, v, N, scale, key_mask=None):
    """Library routine: torch float64 SDPA over the first N keys (optionally a per-query key mask)."""
    qt = torch.from_numpy(q.astype(np.float64))
    kt = torch.from_numpy(k[:, :N].astype(np.float64))
    vt = torch.from_numpy(v[:, :N].astype(np.float64))
    mask = None
    if key_mask is not None:
        mask = torch.from_numpy(key_mask[..., :N])
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    logits = scale * qt @ kt.transpose(-1, -2)
    if mask is not None:
        logits = logits.masked_fill(~mask, float("-inf"))
    lse = torch.logsumexp(logits, dim=-1)
    return o.numpy(), lse.numpy()


def _rows(o, R, nq, H, N):
    """Flatten oracle output [items][R][...] for all items into [H][Np][...] and keep the real rows."""
    shp = o.shape[2:]
    return o.reshape((H, nq * R) + shp)[:, :N]


# ----------------------------------------------------------------------------------------------- dense

def test_dense_matches_library_sdpa():
    rng = np.random.default_rng(1)
    H, N, R, d, scale = 3, 150, 32, 24, 0.37
    Np = 160
    q, k, v = _rand_qkv(rng, H, N, Np, d, q_scale=1.5, k_scale=0.8)
    import oracle
    o, lse = oracle.dense(q, k, v, N, R, scale)
    ro, rl = _torch_attention(q[:, :N], k, v, N, scale)
    np.testing.assert_allclose(_rows(o, R, Np // R, H, N), ro, rtol=0, atol=LIB_ATOL)
    np.testing.assert_allclose(_rows(lse, R, Np // R, H, N), rl, rtol=0, atol=LIB_ATOL)
    # padded query rows carry no output
    assert np.isnan(o.reshape(H, Np, d)[:, N:]).all()


def test_dense_zero_query_closed_form():
    """q = 0: every real key gets weight 1/N, so O = mean of the real V rows and lse = ln N."""
    rng = np.random.default_rng(2)
    H, N, Np, R, d = 2, 200, 256, 64, 16
    q, k, v = _rand_qkv(rng, H, N, Np, d)
    q[:] = 0
    v[:, N:] = 1e6  # padded value rows must not leak in
    import oracle
    o, lse = oracle.dense(q, k, v, N, R, 0.25)
    o = _rows(o, R, Np // R, H, N)
    lse = _rows(lse, R, Np // R, H, N)
    want = v[:, :N].astype(np.float64).mean(axis=1)
    np.testing.assert_allclose(o, np.broadcast_to(want[:, None, :], o.shape), atol=1e-12)
    np.testing.assert_allclose(lse, math.log(N), atol=1e-12)


def test_dense_one_dominant_key():
    """Each query's logit to one key exceeds all others by > 60: O equals that key's V row."""
    rng = np.random.default_rng(3)
    N, d = 32, 32
    q = np.zeros((1, N, d), np.float32)
    k = np.zeros((1, N, d), np.float32)
    v = rng.standard_normal((1, N, d)).astype(np.float32)
    perm = rng.permutation(N)
    for i in range(N):
        q[0, i, i] = 10.0
        k[0, perm[i], i] = 10.0  # query i sees key perm[i] with logit 100 * scale
    import oracle
    o, lse = oracle.dense(q, k, v, N, 8, 1.0)
    o = o.reshape(N, d)
    np.testing.assert_allclose(o, v[0, perm], atol=1e-12)
    np.testing.assert_allclose(lse.reshape(N), 100.0, atol=1e-12)


def test_dense_golden_worked_examples():
    with open(os.path.join(GOLDEN, "attention_worked_examples.json")) as f:
        g = json.load(f)
    import oracle
    for c in g["cases"]:
        q = np.asarray(c["q"], np.float32)[None]
        k = np.asarray(c["k"], np.float32)[None]
        v = np.asarray(c["v"], np.float32)[None]
        nq, nk = q.shape[1], k.shape[1]
        Np = max(nq, nk)
        qp = np.zeros((1, Np, 1), np.float32); qp[0, :nq] = q[0]
        o, lse = oracle.dense(qp, k, v, nk, Np, 1.0)
        # inputs are fp32-rounded (ln 3 is not exact), hence 1e-6 rather than exact
        np.testing.assert_allclose(o[0, :nq, 0], np.asarray(c["o"])[:, 0], rtol=1e-6, err_msg=c["name"])
        np.testing.assert_allclose(lse[0, :nq], c["lse"], rtol=1e-6, err_msg=c["name"])


# ------------------------------------------------------------------------------------------------ mass

def test_mass_rows_sum_to_one_including_tail():
    rng = np.random.default_rng(4)
    H, N, Np, R, d = 2, 300, 320, 64, 16
    q, k, _ = _rand_qkv(rng, H, N, Np, d, q_scale=2.0, k_scale=2.0)
    import oracle
    m = oracle.mass(q, k, N, R, R, 0.5)
    assert m.shape == (H * (Np // R), Np // R)
    np.testing.assert_allclose(m.sum(axis=1), 1.0, atol=1e-12)
    assert (m >= 0).all()


def test_mass_zero_query_closed_form():
    """q = 0: M(i, j) = (real keys in block j) / N for every query block, tail block included."""
    rng = np.random.default_rng(5)
    H, N, Np, R, d = 1, 150, 192, 64, 8
    q, k, _ = _rand_qkv(rng, H, N, Np, d)
    q[:] = 0
    import oracle
    m = oracle.mass(q, k, N, R, R, 1.0)
    real = np.array([min(R, max(0, N - j * R)) for j in range(Np // R)], np.float64)
    np.testing.assert_allclose(m, np.broadcast_to(real / N, m.shape), atol=1e-14)


def test_mass_block_diagonal():
    """Keys of different blocks are orthogonal and queries of block i align with keys of block i with a
    logit of 60: M is the identity up to exp(-60)."""
    nb, R, d = 4, 16, 4
    N = nb * R
    q = np.zeros((1, N, d), np.float32)
    k = np.zeros((1, N, d), np.float32)
    for t in range(N):
        q[0, t, t // R] = 1.0
        k[0, t, t // R] = 1.0
    import oracle
    m = oracle.mass(q, k, N, R, R, 60.0)
    np.testing.assert_allclose(m, np.eye(nb), atol=1e-20)


def test_mass_ragged_tail_dominant_keys():
    """Real query r sees one key perm[r] with a logit 100 above all others, so A(r, .) is that key up to e^-100:
    M(i, j) = (real rows of block i whose key lies in block j) / R_i, also for the ragged tail block, whose zero
    padded query rows must not count."""
    N, Np, R, C = 100, 128, 32, 16
    rng = np.random.default_rng(17)
    perm = rng.permutation(N)
    q = np.zeros((1, Np, N), np.float32)
    k = np.zeros((1, Np, N), np.float32)
    for r in range(N):
        q[0, r, r] = 10.0
        k[0, perm[r], r] = 10.0
    import oracle
    m = oracle.mass(q, k, N, R, C, 1.0)
    want = np.zeros((Np // R, Np // C))
    for r in range(N):
        want[r // R, perm[r] // C] += 1.0
    want /= np.array([min(R, N - i * R) for i in range(Np // R)], np.float64)[:, None]
    np.testing.assert_allclose(m, want, atol=1e-30)


def test_mass_from_library_attention_probabilities():
    """A is recovered from the library's attention with V = identity (O = A I = A); block sums of A,
    divided by the real rows, must equal the oracle's M. Uneven R != C and a ragged tail."""
    rng = np.random.default_rng(6)
    H, N, Np, R, C, d = 2, 90, 96, 32, 16, 12
    q, k, _ = _rand_qkv(rng, H, N, Np, d, q_scale=1.7, k_scale=1.3)
    eye = np.zeros((H, Np, N), np.float32)
    eye[:, np.arange(N), np.arange(N)] = 1.0
    A, _ = _torch_attention(q[:, :N], k, eye[:, :, :], N, 0.6)  # [H][N][N]
    import oracle
    m = oracle.mass(q, k, N, R, C, 0.6).reshape(H, Np // R, Np // C)
    for h in range(H):
        for i in range(Np // R):
            rows = slice(i * R, min(N, (i + 1) * R))
            nr = rows.stop - rows.start
            for j in range(Np // C):
                want = A[h, rows, j * C:min(N, (j + 1) * C)].sum() / nr
                assert abs(m[h, i, j] - want) < LIB_ATOL


def test_mass_golden_worked_examples():
    with open(os.path.join(GOLDEN, "attention_worked_examples.json")) as f:
        g = json.load(f)
    import oracle
    for c in g["mass_cases"]:
        q = np.asarray(c["q"], np.float32)[None]
        k = np.asarray(c["k"], np.float32)[None]
        n = c.get("n_tokens", q.shape[1])
        m = oracle.mass(q, k, n, c["block"], c["block"], 1.0)
        np.testing.assert_allclose(m, np.asarray(c["mass"]), rtol=1e-6, err_msg=c["name"])


# ---------------------------------------------------------------------------------------------- select

def test_select_golden_worked_examples():
    with open(os.path.join(GOLDEN, "select_worked_examples.json")) as f:
        g = json.load(f)
    import oracle
    for c in g["cases"]:
        for dt in (np.float64, np.float32):
            m = np.asarray([c["mass"]], dt)
            counts, idx = oracle.select(m, c["tau"])
            assert list(idx[0, :counts[0]]) == c["kept"], (c, dt)


def _units(m):
    return np.ceil(np.ldexp(np.asarray(m, np.float64), 52)).astype(np.uint64)


def _check_minimal(m_row, tau, kept):
    """prefix(s-1) < T <= prefix(s) in integer units, with the kept set the s largest masses."""
    u = _units(m_row)
    T = int(math.ceil(tau * float(int(u.sum()))))
    s = len(kept)
    assert s >= 1
    ku = sorted((int(u[j]) for j in kept), reverse=True)
    assert sum(ku) >= T
    assert sum(ku[:-1]) < T or s == 1 and T == 0
    dropped = [j for j in range(len(m_row)) if j not in set(kept)]
    if dropped:
        assert max(m_row[j] for j in dropped) <= min(m_row[j] for j in kept)


@pytest.mark.parametrize("dtype", [np.float64, np.float32])
def test_select_minimality_random(dtype):
    rng = np.random.default_rng(7)
    import oracle
    for nk in (1, 2, 3, 7, 64, 300):
        m = rng.exponential(size=(40, nk)) ** 3
        m /= m.sum(axis=1, keepdims=True)
        m = m.astype(dtype)
        for tau in (0.3, 0.9, 0.99, 1.0):
            counts, idx = oracle.select(m, tau)
            for r in range(m.shape[0]):
                kept = list(idx[r, :counts[r]])
                assert kept == sorted(kept)
                _check_minimal(m[r].astype(np.float64) if dtype == np.float64 else m[r], tau, kept)


def test_select_tau_one_keeps_nonzero():
    rng = np.random.default_rng(8)
    import oracle
    m = rng.random((50, 40))
    m[m < 0.4] = 0.0
    m[:, 0] = np.maximum(m[:, 0], 1e-300)  # denormal-scale but non-zero masses still count
    m /= m.sum(axis=1, keepdims=True)
    for dt in (np.float64, np.float32):
        mm = m.astype(dt)
        counts, idx = oracle.select(mm, 1.0)
        for r in range(len(mm)):
            assert list(idx[r, :counts[r]]) == list(np.nonzero(mm[r] > 0)[0])


def test_select_equal_masses_first_by_index():
    import oracle
    for nk in (4, 8, 16, 33):
        m = np.full((1, nk), 1.0 / nk)
        for tau in (0.25, 0.5, 0.7, 0.9):
            counts, idx = oracle.select(m, tau)
            s = math.ceil(tau * nk - 1e-9)
            assert counts[0] == s and list(idx[0, :s]) == list(range(s))


def test_select_brute_force_tiny():
    """All 2^nk subsets: s is the minimum size of any subset whose integer mass reaches T; with distinct
    masses the kept set is the unique subset of that size with the largest mass."""
    rng = np.random.default_rng(9)
    import oracle
    for trial in range(120):
        nk = int(rng.integers(1, 11))
        kind = trial % 3
        if kind == 0:
            m = rng.random(nk)
        elif kind == 1:  # ties and zeros
            m = rng.integers(0, 4, nk).astype(np.float64)
            if m.sum() == 0:
                m[0] = 1
        else:
            m = rng.exponential(size=nk) ** 4
        m = m / m.sum()
        tau = float(rng.choice([0.2, 0.5, 0.8, 0.9, 0.99, 1.0]))
        counts, idx = oracle.select(m[None], tau)
        kept = list(idx[0, :counts[0]])
        u = [int(x) for x in _units(m)]
        T = int(math.ceil(tau * float(sum(u))))
        best = None
        for size in range(1, nk + 1):
            sums = [(sum(u[j] for j in c), c) for c in itertools.combinations(range(nk), size)]
            ok = [x for x in sums if x[0] >= T]
            if ok:
                best = (size, max(x[0] for x in ok), [x[1] for x in ok])
                break
        assert counts[0] == best[0]
        assert sum(u[j] for j in kept) == best[1]
        if len(set(m)) == nk:
            winners = [c for c in best[2] if sum(u[j] for j in c) == best[1]]
            assert len(winners) == 1 and list(winners[0]) == kept


def test_select_brute_force_nk_up_to_16():
    """The same two facts for nk = 11..16, with the 2^nk subsets enumerated as bit masks."""
    rng = np.random.default_rng(10)
    import oracle
    for trial, nk in enumerate((11, 12, 13, 14, 15, 16, 16, 16, 16)):
        kind = trial % 3
        if kind == 0:
            m = rng.random(nk)
        elif kind == 1:  # ties and zeros
            m = rng.integers(0, 4, nk).astype(np.float64)
            m[0] += 1
        else:
            m = rng.exponential(size=nk) ** 4
        m = m / m.sum()
        tau = float(rng.choice([0.5, 0.9, 0.99, 1.0]))
        counts, idx = oracle.select(m[None], tau)
        kept = [int(j) for j in idx[0, :counts[0]]]
        u = _units(m).astype(np.int64)
        T = int(math.ceil(tau * float(int(u.sum()))))
        masks = np.arange(1 << nk, dtype=np.int64)
        bits = (masks[:, None] >> np.arange(nk, dtype=np.int64)) & 1
        sums = bits @ u
        sizes = bits.sum(axis=1)
        reach = sums >= T
        best_size = int(sizes[reach].min())
        best = reach & (sizes == best_size)
        best_sum = int(sums[best].max())
        assert counts[0] == best_size
        assert int(u[kept].sum()) == best_sum
        if len(set(m)) == nk:
            winners = masks[best & (sums == best_sum)]
            assert len(winners) == 1 and int(winners[0]) == sum(1 << j for j in kept)


def test_select_topk_keeps_k_largest_with_index_ties():
    """Brute force: the kept set is the k largest masses, ties resolved toward lower indices; equal masses keep
    the first k indices; k >= nk keeps everything."""
    rng = np.random.default_rng(21)
    import oracle
    for trial in range(60):
        nk = int(rng.integers(1, 40))
        m = rng.integers(0, 6, nk).astype(np.float32) if trial % 2 else rng.random(nk).astype(np.float32)
        k = int(rng.integers(1, nk + 3))
        counts, idx = oracle.select_topk(m[None], k)
        kept = list(idx[0, :counts[0]])
        want = sorted(sorted(range(nk), key=lambda j: (-float(m[j]), j))[:min(k, nk)])
        assert kept == want
    counts, idx = oracle.select_topk(np.full((1, 8), 0.125, np.float32), 3)
    assert list(idx[0, :counts[0]]) == [0, 1, 2]


def test_select_tiny_tau_keeps_the_heaviest_block():
    """Any tau > 0 keeps at least one block, and a tau below the largest mass keeps exactly the heaviest block
    (the lowest index among equal maxima); a row of all-equal masses keeps block 0."""
    rng = np.random.default_rng(12)
    import oracle
    m = rng.exponential(size=(40, 25)) ** 3
    m[5] = 1.0
    m[6, 3] = m[6, 17] = m[6].max() * 2.0
    m /= m.sum(axis=1, keepdims=True)
    for tau in (1e-300, 1e-12, 1e-3):
        counts, idx = oracle.select(m, tau)
        assert (counts == 1).all()
        assert idx[:, 0].tolist() == np.argmax(m, axis=1).tolist()
    assert idx[5, 0] == 0 and idx[6, 0] == 3


def test_select_rejects_bad_tau():
    import oracle
    m = np.full((1, 4), 0.25)
    for tau in (0.0, -0.1, 1.0000001, float("nan")):
        with pytest.raises(ValueError):
            oracle.select(m, tau)


def test_select_refuses_rows_outside_the_normalised_domain():
    """The selection reads rows of masses normalised to one (the LoSA page's "theta R" rule divided by R): a row
    summing to more than 2 (here one scaled by 1e4, whose integer units would leave 64 bits) is refused, while a row
    whose sum is one up to rounding, or a single block holding all the mass, is accepted."""
    import oracle
    rng = np.random.default_rng(13)
    m = rng.exponential(size=(3, 50))
    m /= m.sum(axis=1, keepdims=True)
    for dt in (np.float64, np.float32):
        oracle.select(m.astype(dt), 0.99)
        big = m.copy()
        big[1] *= 1e4
        with pytest.raises(ValueError):
            oracle.select(big.astype(dt), 0.99)
        one = np.zeros((1, 5), dt)
        one[0, 3] = 1.0
        counts, idx = oracle.select(one, 0.99)
        assert counts[0] == 1 and idx[0, 0] == 3
        over = np.full((1, 4), 0.5000001, dt)  # sums to 2.0000004
        with pytest.raises(ValueError):
            oracle.select(over, 0.5)


def test_lpt_order_definition():
    rng = np.random.default_rng(10)
    import oracle
    counts = rng.integers(1, 9, 500).astype(np.int32)
    order = oracle.lpt_order(counts)
    assert sorted(order.tolist()) == list(range(500))
    want = sorted(range(500), key=lambda i: (-int(counts[i]), i))
    assert order.tolist() == want


# ---------------------------------------------------------------------------------------------- sparse

def test_sparse_all_blocks_equals_dense():
    rng = np.random.default_rng(11)
    H, N, Np, R, d = 2, 120, 128, 32, 16
    q, k, v = _rand_qkv(rng, H, N, Np, d, 1.3, 1.3)
    nq = Np // R
    indptr = np.arange(0, H * nq * nq + 1, nq, dtype=np.int32)
    kv = np.tile(np.arange(nq, dtype=np.int32), H * nq)
    import oracle
    od, ld = oracle.dense(q, k, v, N, R, 0.3)
    os_, ls = oracle.sparse(q, k, v, N, R, R, 0.3, indptr, kv)
    np.testing.assert_array_equal(np.isnan(od), np.isnan(os_))
    np.testing.assert_allclose(os_[~np.isnan(os_)], od[~np.isnan(od)], atol=1e-12)
    np.testing.assert_allclose(ls[~np.isnan(ls)], ld[~np.isnan(ld)], atol=1e-12)


def test_sparse_matches_library_masked_sdpa():
    """Random block lists (unsorted, R != C): the library's masked attention over the same keys."""
    rng = np.random.default_rng(12)
    H, N, Np, R, C, d = 2, 100, 128, 32, 16, 8
    q, k, v = _rand_qkv(rng, H, N, Np, d, 1.5, 1.5)
    nq, nk = Np // R, Np // C
    lists = []
    for _ in range(H * nq):
        s = int(rng.integers(1, nk + 1))
        lists.append(rng.permutation(nk)[:s].astype(np.int32))
    # every list must reach at least one real key
    for L in lists:
        if (L * C >= N).all():
            L[0] = 0
    indptr = np.zeros(H * nq + 1, np.int32)
    indptr[1:] = np.cumsum([len(L) for L in lists])
    kv = np.concatenate(lists)
    mask = np.zeros((H, Np, Np), bool)
    for h in range(H):
        for i in range(nq):
            for j in lists[h * nq + i]:
                mask[h, i * R:(i + 1) * R, j * C:(j + 1) * C] = True
    import oracle
    o, lse = oracle.sparse(q, k, v, N, R, C, 0.9, indptr, kv)
    ro, rl = _torch_attention(q[:, :N], k, v, N, 0.9, key_mask=mask[:, :N])
    np.testing.assert_allclose(_rows(o, R, nq, H, N), ro, atol=LIB_ATOL)
    np.testing.assert_allclose(_rows(lse, R, nq, H, N), rl, atol=LIB_ATOL)


def test_sparse_single_block_lists():
    rng = np.random.default_rng(13)
    H, N, Np, R, d = 1, 96, 96, 32, 8
    q, k, v = _rand_qkv(rng, H, N, Np, d)
    nq = Np // R
    import oracle
    for j in range(nq):
        indptr = np.arange(nq + 1, dtype=np.int32)
        kv = np.full(nq, j, np.int32)
        o, _ = oracle.sparse(q, k, v, N, R, R, 0.5, indptr, kv)
        sl = slice(j * R, (j + 1) * R)
        ro, _ = _torch_attention(q, k[:, sl], v[:, sl], R, 0.5)
        np.testing.assert_allclose(o.reshape(1, Np, d), ro, atol=LIB_ATOL)


def test_sparse_tau_one_reproduces_dense():
    """theta = 1 keeps every block of non-zero mass; with all masses non-zero the pattern is dense."""
    rng = np.random.default_rng(14)
    H, N, Np, R, d = 2, 180, 192, 64, 16
    q, k, v = _rand_qkv(rng, H, N, Np, d)
    import oracle
    m = oracle.mass(q, k, N, R, R, 0.25)
    assert (m > 0).all()
    counts, idx = oracle.select(m, 1.0)
    indptr, kv = oracle.to_csr(counts, idx)
    od, ld = oracle.dense(q, k, v, N, R, 0.25)
    os_, ls = oracle.sparse(q, k, v, N, R, R, 0.25, indptr, kv)
    ok = ~np.isnan(od)
    np.testing.assert_allclose(os_[ok], od[ok], atol=1e-12)


def test_recall_at_construction_reaches_tau():
    """Selection on exact masses retains at least theta of every row's mass (by construction)."""
    layer = make_layer("tiny")
    cfg = layer.cfg
    import oracle
    q, k = layer.all_f32("q"), layer.all_f32("k")
    m = oracle.mass(q, k, cfg.n_tokens, cfg.block, cfg.block, 1 / math.sqrt(cfg.head_dim))
    for tau in cfg.taus:
        counts, idx = oracle.select(m, tau)
        indptr, kv = oracle.to_csr(counts, idx)
        for r in range(m.shape[0]):
            kept = m[r, idx[r, :counts[r]]].sum()
            assert kept >= tau * m[r].sum() - 1e-12
        assert oracle.recall(m, indptr, kv) >= tau - 1e-12


def test_recall_closed_forms():
    """Recall (Motivation Summary: retained mass over total mass of the rows) of patterns whose value is known:
    every block gives 1, block j alone gives column j's share, and a subset of rows counts only those rows."""
    rng = np.random.default_rng(16)
    import oracle
    m = rng.random((6, 5))
    full = np.tile(np.arange(5, dtype=np.int32), 6)
    assert abs(oracle.recall(m, np.arange(0, 31, 5, dtype=np.int32), full) - 1.0) < 1e-15
    for j in range(5):
        one = np.full(6, j, np.int32)
        assert abs(oracle.recall(m, np.arange(7, dtype=np.int32), one) - m[:, j].sum() / m.sum()) < 1e-14
    # rows 4 and 1 of a pattern where row r keeps blocks 0..r-1 (row 0 keeps block 0)
    lists = [np.arange(max(r, 1), dtype=np.int32) for r in range(6)]
    indptr = np.zeros(7, np.int32)
    indptr[1:] = np.cumsum([len(x) for x in lists])
    kv = np.concatenate(lists)
    sub = m[[4, 1]]
    want = (sub[0, :4].sum() + sub[1, :1].sum()) / sub.sum()
    assert abs(oracle.recall(sub, indptr, kv, rows=[4, 1]) - want) < 1e-14


# ------------------------------------------------------------------------------------------- generator

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(15)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    ours = f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    np.testing.assert_array_equal(bf16_bits_to_f32(ours), round_to_bf16(x))


def test_generator_is_seeded_and_padded():
    a, b = make_layer("tiny"), make_layer("tiny")
    np.testing.assert_array_equal(a.q, b.q)
    np.testing.assert_array_equal(a.k, b.k)
    cfg = CONFIGS["tiny"]
    assert a.q.shape == (cfg.heads, cfg.n_padded, cfg.head_dim)
    # Wan2.1-1.3B-480p geometry: 21*30*52 = 32760 tokens, padded to 32768 with zero rows
    c1 = CONFIGS["wan1.3b480"]
    assert (c1.n_tokens, c1.n_padded, c1.n_blocks) == (32760, 32768, 256)
    assert CONFIGS["hunyuan720"].n_padded == 118912 and CONFIGS["wan14b720"].n_padded == 75648


def test_sample_items_is_seeded_and_keeps_the_forced_items():
    """Sampled items are distinct, sorted, in range, reproducible from the seed, and always include the tail query
    block of head 0 and the requested ids."""
    from losa_synth import sample_items
    cfg = CONFIGS["hunyuan720"]
    total = cfg.heads * cfg.n_blocks
    a = sample_items(cfg, 64, seed=3, must_include=[5, 700])
    assert len(a) == 64 and len(set(a.tolist())) == 64 and (np.diff(a) > 0).all()
    assert a.min() >= 0 and a.max() < total
    assert {cfg.n_blocks - 1, 5, 700} <= set(a.tolist())
    np.testing.assert_array_equal(a, sample_items(cfg, 64, seed=3, must_include=[5, 700]))
    assert not np.array_equal(a, sample_items(cfg, 64, seed=4, must_include=[5, 700]))
    small = CONFIGS["tiny"]
    np.testing.assert_array_equal(sample_items(small, 1000), np.arange(small.heads * small.n_blocks))


def test_drift_walk_on_the_host():
    """The reuse loop's drift: each step adds amount * rms(step-0 head) * N(0, 1) to the real rows only, padded rows
    stay zero, and the walk is reproducible from its seed."""
    from losa_synth import Drift
    cfg = CONFIGS["tiny"]
    layer = make_layer(cfg)
    d1 = Drift(cfg, [layer], device="cpu", amount=0.1, seed=7)
    d2 = Drift(cfg, [layer], device="cpu", amount=0.1, seed=7)
    q0 = d1.tokens(0)[0].clone()
    d1.advance()
    d2.advance()
    q1 = d1.tokens(0)[0]
    torch.testing.assert_close(q1, d2.tokens(0)[0], rtol=0, atol=0)
    n = cfg.n_tokens
    assert torch.count_nonzero(q1[:, n:]) == 0
    step = (q1 - q0)[:, :n]
    rms0 = q0[:, :n].pow(2).mean(dim=(1, 2)).sqrt()
    ratio = step.pow(2).mean(dim=(1, 2)).sqrt() / (0.1 * rms0)
    assert torch.allclose(ratio, torch.ones_like(ratio), atol=0.05), ratio
    np.testing.assert_array_equal(layer.q, make_layer(cfg).q)  # the walk leaves the generated layer untouched


def test_lpt_order_invariants():
    """The work order is a permutation along which list lengths never increase, and items of equal length appear in
    increasing id order (many ties)."""
    rng = np.random.default_rng(18)
    import oracle
    for n in (1, 2, 7, 300):
        counts = rng.integers(1, 4, n).astype(np.int32)
        order = oracle.lpt_order(counts)
        assert sorted(order.tolist()) == list(range(n))
        c = counts[order]
        assert (np.diff(c) <= 0).all()
        for v in np.unique(c):
            ids = order[c == v]
            assert (np.diff(ids) > 0).all()


def test_select_topk_boundary_invariants():
    """Top-k keeps min(k, nk) blocks, every kept mass is at least every dropped one, and where equal masses straddle
    the cut the kept ones have the lower indices."""
    rng = np.random.default_rng(19)
    import oracle
    for trial in range(200):
        nk = int(rng.integers(1, 30))
        m = rng.integers(0, 4, nk).astype(np.float32)  # many ties
        k = int(rng.integers(1, nk + 2))
        counts, idx = oracle.select_topk(m[None], k)
        kept = set(idx[0, :counts[0]].tolist())
        assert counts[0] == min(k, nk) and len(kept) == counts[0]
        dropped = [j for j in range(nk) if j not in kept]
        if dropped and kept:
            assert min(m[j] for j in kept) >= max(m[j] for j in dropped)
            cut = min(m[j] for j in kept)
            tied_kept = [j for j in kept if m[j] == cut]
            tied_dropped = [j for j in dropped if m[j] == cut]
            if tied_dropped:
                assert max(tied_kept) < min(tied_dropped)
