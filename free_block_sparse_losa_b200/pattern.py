"""Saving and loading a frozen sparsity pattern (LoSA page, Methodology Summary: the pattern is built once, at step t0,
and reused unchanged for the remaining denoising steps, so it is the method's only state worth keeping between runs).

A pattern is the selection's output for one layer: indptr (H*nq + 1 int32, a monotone prefix of the list lengths),
kv_block_idx (indptr[-1] int32 key-block indices, ascending within each list) and the longest-first work order (H*nq
int32, a permutation of the items), plus the shape it was built for. The file is a NumPy .npz archive; loading checks
the shape against the caller's and the three arrays against each other, so that a pattern is never handed to the
sparse kernel for a layer it does not describe. Host-side only: no device work happens here."""
from __future__ import annotations

import numpy as np

FORMAT = "losa-pattern-v1"
_SHAPE_KEYS = ("heads", "n_tokens", "n_padded", "head_dim", "block_q", "block_k")


def _shape(shape) -> dict:
    """The shape fields a pattern depends on, from a dict or from the C ABI's shape struct."""
    if isinstance(shape, dict):
        return {k: int(shape[k]) for k in _SHAPE_KEYS}
    return {k: int(getattr(shape, k)) for k in _SHAPE_KEYS}


def check_pattern(shape, indptr: np.ndarray, kv_block_idx: np.ndarray, order: np.ndarray) -> None:
    """Raises ValueError unless (indptr, kv_block_idx, order) is a valid pattern for `shape`, with every list strictly
    ascending as the selection writes it (which also rules out a block listed twice)."""
    shape = _shape(shape)
    rows = shape["heads"] * (shape["n_padded"] // shape["block_q"])
    nkb = shape["n_padded"] // shape["block_k"]
    indptr = np.asarray(indptr)
    if indptr.shape != (rows + 1,) or indptr[0] != 0:
        raise ValueError(f"indptr: expected {rows + 1} entries starting at 0")
    counts = np.diff(indptr.astype(np.int64))
    if (counts < 1).any() or (counts > nkb).any():
        raise ValueError("indptr: every list holds between 1 and nk blocks")
    nnz = int(indptr[-1])
    idx = np.asarray(kv_block_idx)
    if idx.shape[0] < nnz:
        raise ValueError(f"kv_block_idx: holds {idx.shape[0]} entries, indptr needs {nnz}")
    idx = idx[:nnz].astype(np.int64)
    if (idx < 0).any() or (idx >= nkb).any():
        raise ValueError("kv_block_idx: block index out of range")
    # ascending within each list: a decrease is allowed only where a new list starts
    drops = np.flatnonzero(np.diff(idx) <= 0) + 1
    if not np.isin(drops, indptr[1:-1]).all():
        raise ValueError("kv_block_idx: a list is not strictly ascending")
    order = np.asarray(order)
    if order.shape != (rows,) or not np.array_equal(np.sort(order.astype(np.int64)), np.arange(rows)):
        raise ValueError("order: expected a permutation of the items")


def save_pattern(path: str, shape, tau: float, indptr, kv_block_idx, order) -> None:
    """Writes a checked pattern; the arrays may be NumPy arrays or host/device tensors."""
    def host(a):
        return a.cpu().numpy() if hasattr(a, "cpu") else np.asarray(a)

    shape = _shape(shape)
    indptr, kv_block_idx, order = host(indptr), host(kv_block_idx), host(order)
    check_pattern(shape, indptr, kv_block_idx, order)
    nnz = int(indptr[-1])
    np.savez(path, format=np.array(FORMAT), shape=np.array([shape[k] for k in _SHAPE_KEYS], dtype=np.int64),
             tau=np.array(float(tau)), indptr=indptr.astype(np.int32),
             kv_block_idx=kv_block_idx[:nnz].astype(np.int32), order=order.astype(np.int32))


def load_pattern(path: str, shape):
    """Reads a pattern saved for `shape`; returns (tau, indptr, kv_block_idx, order) as int32 NumPy arrays."""
    with np.load(path, allow_pickle=False) as z:
        if str(z["format"]) != FORMAT:
            raise ValueError(f"{path}: not a {FORMAT} file")
        saved = dict(zip(_SHAPE_KEYS, (int(x) for x in z["shape"])))
        want = _shape(shape)
        if saved != want:
            raise ValueError(f"{path}: pattern built for {saved}, not {want}")
        tau = float(z["tau"])
        indptr, idx, order = z["indptr"], z["kv_block_idx"], z["order"]
    check_pattern(want, indptr, idx, order)
    return tau, indptr.astype(np.int32), idx.astype(np.int32), order.astype(np.int32)
