"""GPU parity of losa_select against the oracle fed the same fp32 masses: CSR lists and the longest-first
work order must match bit for bit (LoSA page, Methodology Summary, "One-time pattern construction")."""
import numpy as np
import pytest
import torch

import free_block_sparse_losa_b200 as L
from tests.gpu_util import compare_select, require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _masses(rng, rows, nk, kind):
    if kind == "exp":
        m = rng.exponential(size=(rows, nk)) ** 4
    elif kind == "ties":
        m = rng.integers(0, 5, size=(rows, nk)).astype(np.float64)
        m[:, 0] += 1.0
    elif kind == "peaked":  # few dominant blocks, long tail spanning many decades (like real attention)
        m = np.exp(rng.standard_normal((rows, nk)) * 8.0)
    elif kind == "uniform":
        m = np.ones((rows, nk))
    m = m / m.sum(axis=1, keepdims=True)
    return m.astype(np.float32)


def _run(shape_args, m, tau, oracle):
    H, nq, nk, R, C = shape_args
    Np = nk * C
    shape = L.make_shape(H, Np - 1, Np, 128, R, C, "bf16")
    dev = torch.from_numpy(m.reshape(H * nq * nk)).cuda()
    rows = H * nq
    indptr = torch.full((rows + 1,), -7, dtype=torch.int32, device="cuda")
    idx = torch.full((rows * nk,), -7, dtype=torch.int32, device="cuda")
    order = torch.full((rows,), -7, dtype=torch.int32, device="cuda")
    ws = torch.empty(L.losa_select_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    L.losa_select(shape, dev, tau, indptr, idx, order, ws)
    assert L.losa_get_device_error() == 0
    gi = indptr.cpu().numpy()
    nnz = int(gi[-1])
    gk = idx.cpu().numpy()
    # nothing written past nnz
    assert (gk[nnz:] == -7).all()
    return compare_select(gi, gk[:nnz], order.cpu().numpy(), m.reshape(rows, nk), tau, oracle)


@pytest.mark.parametrize("H,nb", [(1, 1), (1, 2), (3, 4), (2, 31), (2, 64), (4, 256), (1, 929), (2, 1024)])
@pytest.mark.parametrize("kind", ["exp", "ties", "peaked", "uniform"])
def test_select_matches_oracle(H, nb, kind, oracle_mod):
    rng = np.random.default_rng(H * 1000 + nb)
    m = _masses(rng, H * nb, nb, kind)
    for tau in (0.5, 0.9, 0.99, 1.0):
        counts = _run((H, nb, nb, 128, 128), m, tau, oracle_mod)
        assert counts.min() >= 1


def test_select_uneven_blocks(oracle_mod):
    """R = 64, C = 32: more key blocks than query blocks per row."""
    rng = np.random.default_rng(3)
    H, nq, nk = 3, 20, 40
    m = _masses(rng, H * nq, nk, "peaked")
    for tau in (0.9, 0.99):
        _run((H, nq, nk, 64, 32), m, tau, oracle_mod)


def test_select_full_size_hunyuan_rows(oracle_mod):
    """22296 rows x 929 blocks (the HunyuanVideo-720p-shaped layer), peaked masses."""
    rng = np.random.default_rng(4)
    H, nb = 24, 929
    m = _masses(rng, H * nb, nb, "peaked")
    _run((H, nb, nb, 128, 128), m, 0.99, oracle_mod)


def test_select_two_branch_hunyuan_rows(oracle_mod):
    """Classifier-free guidance at the HunyuanVideo-720p shape: the conditional and unconditional branches stacked as
    48 heads, 44592 rows x 929 blocks, each branch with its own pattern (LoSA page, Methodology Summary)."""
    rng = np.random.default_rng(5)
    H, nb = 48, 929
    m = _masses(rng, H * nb, nb, "peaked")
    counts = _run((H, nb, nb, 128, 128), m, 0.99, oracle_mod)
    assert counts.min() >= 1


@pytest.mark.parametrize("kind", ["exp", "ties", "peaked", "uniform"])
def test_select_wide_rows_c32(kind, oracle_mod):
    """3716 key blocks per row (the HunyuanVideo shape with 32-key blocks): the shared-memory pick path, and the
    one-CTA sort for rows whose cut lies beyond the pick path's reach (uniform rows, tau = 1)."""
    rng = np.random.default_rng(6)
    H, nk = 1, 3716
    nq = nk * 32 // 128  # 929 query blocks of 128 rows
    m = _masses(rng, H * nq, nk, kind)
    for tau in (0.9, 0.99, 1.0):
        _run((H, nq, nk, 128, 32), m, tau, oracle_mod)


def test_select_reports_rows_outside_the_domain():
    """Rows of masses are normalised to one; a row scaled by 1e4 (its integer units would leave 64 bits) is reported
    through the device error word instead of being cut with undefined arithmetic."""
    shape = L.make_shape(1, 1023, 1024, 128, 128, 128, "bf16")
    rows, nk = 8, 8
    rng = np.random.default_rng(14)
    mm = _masses(rng, rows, nk, "exp")
    mm[3] *= 1e4
    dev = torch.from_numpy(mm.ravel()).cuda()
    indptr = torch.empty(rows + 1, dtype=torch.int32, device="cuda")
    idx = torch.empty(rows * nk, dtype=torch.int32, device="cuda")
    order = torch.empty(rows, dtype=torch.int32, device="cuda")
    ws = torch.empty(L.losa_select_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    L.losa_select(shape, dev, 0.99, indptr, idx, order, ws)
    assert L.losa_get_device_error() == -5
    assert L.losa_get_device_error() == 0


@pytest.mark.parametrize("H,nb,k", [(1, 1, 1), (2, 31, 4), (4, 256, 12), (1, 929, 40), (2, 64, 64), (2, 64, 100),
                                    (1, 929, 100), (1, 1500, 80)])
def test_select_topk_matches_oracle(H, nb, k, oracle_mod):
    rng = np.random.default_rng(H * 7 + nb)
    m = _masses(rng, H * nb, nb, "peaked" if nb > 4 else "ties")
    shape = L.make_shape(H, nb * 128 - 1, nb * 128, 128, 128, 128, "bf16")
    rows = H * nb
    dev = torch.from_numpy(m.ravel()).cuda()
    indptr = torch.empty(rows + 1, dtype=torch.int32, device="cuda")
    idx = torch.empty(rows * nb, dtype=torch.int32, device="cuda")
    order = torch.empty(rows, dtype=torch.int32, device="cuda")
    ws = torch.empty(L.losa_select_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    L.losa_select_topk(shape, dev, k, indptr, idx, order, ws)
    assert L.losa_get_device_error() == 0
    counts, ref = oracle_mod.select_topk(m, k)
    ri, rk = oracle_mod.to_csr(counts, ref)
    gi = indptr.cpu().numpy()
    np.testing.assert_array_equal(gi, ri)
    np.testing.assert_array_equal(idx.cpu().numpy()[:gi[-1]], rk)
    np.testing.assert_array_equal(order.cpu().numpy(), oracle_mod.lpt_order(counts))


def test_select_reports_bad_mass():
    shape = L.make_shape(1, 1023, 1024, 128, 128, 128, "bf16")
    rows, nk = 8, 8
    mm = np.full((rows, nk), 1.0 / 8, np.float32)
    mm[5, 2] = np.nan
    dev = torch.from_numpy(mm.ravel()).cuda()
    indptr = torch.empty(rows + 1, dtype=torch.int32, device="cuda")
    idx = torch.empty(rows * nk, dtype=torch.int32, device="cuda")
    order = torch.empty(rows, dtype=torch.int32, device="cuda")
    ws = torch.empty(L.losa_select_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    L.losa_select(shape, dev, 0.9, indptr, idx, order, ws)
    assert L.losa_get_device_error() == -5
    assert L.losa_get_device_error() == 0  # cleared by the read
