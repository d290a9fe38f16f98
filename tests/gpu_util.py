"""Shared helpers of the GPU parity tests: generation, device transfer, oracle comparison and tolerances.

Tolerances (written here once, used by every GPU test):
  * block masses: |M_gpu - M_ref| <= 1e-4 * M_ref + 1e-30 per entry (the floor covers fp32 exp underflow);
  * outputs: max-abs 2e-2 and relative L2 (||dO|| / ||O_ref|| over the compared real rows) 1e-2;
  * log-sum-exp: abs 1e-3;
  * selection, CSR, work order: bit-exact.
"""
from __future__ import annotations

import math

import numpy as np
import pytest

MASS_RTOL, MASS_ATOL = 1e-4, 1e-30
O_MAXABS, O_RELL2 = 2e-2, 1e-2
LSE_ATOL = 1e-3


def require_gpu():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from free_block_sparse_losa_b200 import build
    build.build()


def device_inputs(layer):
    from free_block_sparse_losa_b200.harness import host_tokens_to_device
    dt = layer.cfg.dtype
    return tuple(host_tokens_to_device(getattr(layer, n), dt) for n in ("q", "k", "v"))


def scale_of(cfg):
    return 1.0 / math.sqrt(cfg.head_dim)


def check_mass(gpu_rows: np.ndarray, ref_rows: np.ndarray, what=""):
    gpu_rows = gpu_rows.astype(np.float64)
    err = np.abs(gpu_rows - ref_rows)
    bound = MASS_RTOL * ref_rows + MASS_ATOL
    bad = err > bound
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what} mass mismatch at {tuple(i)}: gpu={gpu_rows[tuple(i)]!r} "
                             f"ref={ref_rows[tuple(i)]!r} ({int(bad.sum())} entries)")


def check_output(gpu_o: np.ndarray, ref_o: np.ndarray, what=""):
    """gpu_o / ref_o: [rows][d] real rows only."""
    d = np.abs(gpu_o.astype(np.float64) - ref_o)
    maxabs = float(d.max()) if d.size else 0.0
    rel = float(np.linalg.norm(d) / max(np.linalg.norm(ref_o), 1e-300))
    assert maxabs <= O_MAXABS, f"{what} max-abs {maxabs:.3e} > {O_MAXABS}"
    assert rel <= O_RELL2, f"{what} rel-L2 {rel:.3e} > {O_RELL2}"
    return maxabs, rel


def check_lse(gpu_l: np.ndarray, ref_l: np.ndarray, what=""):
    d = float(np.abs(gpu_l.astype(np.float64) - ref_l).max()) if gpu_l.size else 0.0
    assert d <= LSE_ATOL, f"{what} lse abs err {d:.3e} > {LSE_ATOL}"


def item_rows(cfg, items, arr):
    """Gather the real rows of the listed items from a [H][Np][...] array -> ([n_real][...], mask [n][R])."""
    R, nq = cfg.block, cfg.n_blocks
    out, valid = [], np.zeros((len(items), R), bool)
    for t, it in enumerate(items):
        h, i = divmod(int(it), nq)
        rows = np.arange(i * R, (i + 1) * R)
        valid[t] = rows < cfg.n_tokens
        out.append(arr[h, rows])
    return np.stack(out), valid


def compare_select(gpu_indptr, gpu_idx, gpu_order, mass_f32_rows, tau, oracle):
    """Bit-exact comparison of the GPU CSR and work order with the oracle fed the same fp32 masses."""
    counts, idx = oracle.select(mass_f32_rows, tau)
    indptr, kv = oracle.to_csr(counts, idx)
    np.testing.assert_array_equal(gpu_indptr, indptr)
    np.testing.assert_array_equal(gpu_idx, kv)
    np.testing.assert_array_equal(gpu_order, oracle.lpt_order(counts))
    return counts
