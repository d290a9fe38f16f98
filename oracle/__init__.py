"""ctypes wrapper of the fp64 CPU oracle (losa_oracle.cpp) — TEST INFRASTRUCTURE ONLY.

Only the tests, `__graft_entry__.smoke()` and the benchmark's two CPU legs (`cpu_baseline` and `--impl reference`)
may import this package.
It is independent of the CUDA library: it neither imports nor loads anything from it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "losa_oracle.cpp")
_LIB = os.path.join(_HERE, "liblosa_oracle.so")
_lib = None


def compile_command(src: str, out: str) -> list:
    return ["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", "-o", out, src]


def build(force: bool = False) -> str:
    """Compile the oracle with the system C++ compiler (portable flags: it may run on another host)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.run(compile_command(_SRC, _LIB + ".tmp"), check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def bind(path: str):
    """Load a compiled oracle library and declare its entry points."""
    L = ctypes.CDLL(path)
    i32, f64, vp = ctypes.c_int, ctypes.c_double, ctypes.c_void_p
    L.oracle_num_threads.restype = i32
    L.oracle_dense.argtypes = [i32, i32, i32, i32, i32, f64, vp, vp, vp, i32, vp, vp, vp]
    L.oracle_mass.argtypes = [i32, i32, i32, i32, i32, i32, f64, vp, vp, i32, vp, vp]
    L.oracle_select_f32.argtypes = [i32, i32, vp, f64, vp, vp]
    L.oracle_select_f64.argtypes = [i32, i32, vp, f64, vp, vp]
    L.oracle_select_topk.argtypes = [i32, i32, vp, i32, vp, vp]
    L.oracle_lpt_order.argtypes = [i32, vp, vp]
    L.oracle_sparse.argtypes = [i32, i32, i32, i32, i32, i32, f64, vp, vp, vp, vp, vp, i32, vp, vp, vp]
    L.oracle_recall.argtypes = [i32, i32, vp, vp, vp, vp]
    L.oracle_recall.restype = f64
    for name in ("oracle_dense", "oracle_mass", "oracle_select_f32", "oracle_select_f64", "oracle_select_topk",
                 "oracle_lpt_order", "oracle_sparse"):
        getattr(L, name).restype = i32
    return L


def lib():
    global _lib
    if _lib is None:
        _lib = bind(build())
    return _lib


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"{what}: oracle rejected its arguments (rc={rc})")


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def _items(H, Np, R, items):
    if items is None:
        return np.arange(H * (Np // R), dtype=np.int32)
    return _i32(items)


def dense(q, k, v, n_tokens: int, block_q: int, scale: float, items=None):
    """Dense attention. q/k/v: [H][Np][d] fp32 (rounded inputs). Returns (o [n][R][d], lse [n][R]) fp64."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    H, Np, d = q.shape
    it = _items(H, Np, block_q, items)
    o = np.empty((len(it), block_q, d), dtype=np.float64)
    lse = np.empty((len(it), block_q), dtype=np.float64)
    _check(lib().oracle_dense(H, n_tokens, Np, d, block_q, scale, _p(q), _p(k), _p(v), len(it), _p(it), _p(o),
                              _p(lse)), "oracle_dense")
    return o, lse


def mass(q, k, n_tokens: int, block_q: int, block_k: int, scale: float, items=None):
    """Row-normalised block masses [n][nk] fp64 of the listed items."""
    q, k = _f32(q), _f32(k)
    H, Np, d = q.shape
    it = _items(H, Np, block_q, items)
    out = np.empty((len(it), Np // block_k), dtype=np.float64)
    _check(lib().oracle_mass(H, n_tokens, Np, d, block_q, block_k, scale, _p(q), _p(k), len(it), _p(it),
                             _p(out)), "oracle_mass")
    return out


def select(m, tau: float):
    """Selection on a [rows][nk] mass matrix (fp32 or fp64 rule by dtype). Returns (counts, idx[rows][nk]);
    idx[r, :counts[r]] are the kept blocks ascending, the rest is undefined."""
    m = np.ascontiguousarray(m)
    rows, nk = m.shape
    counts = np.empty(rows, dtype=np.int32)
    idx = np.full((rows, nk), -1, dtype=np.int32)
    if m.dtype == np.float32:
        rc = lib().oracle_select_f32(nk, rows, _p(m), tau, _p(counts), _p(idx))
    else:
        m = np.ascontiguousarray(m, dtype=np.float64)
        rc = lib().oracle_select_f64(nk, rows, _p(m), tau, _p(counts), _p(idx))
    _check(rc, "oracle_select")
    return counts, idx


def select_topk(m, k: int):
    """Fixed-count selection on fp32 masses [rows][nk]: (counts, idx) as select()."""
    m = np.ascontiguousarray(m, dtype=np.float32)
    rows, nk = m.shape
    counts = np.empty(rows, dtype=np.int32)
    idx = np.full((rows, nk), -1, dtype=np.int32)
    _check(lib().oracle_select_topk(nk, rows, _p(m), int(k), _p(counts), _p(idx)), "oracle_select_topk")
    return counts, idx


def to_csr(counts, idx):
    """Pack (counts, idx) into CSR (indptr int32 [rows+1], kv_block_idx int32 [nnz])."""
    counts = _i32(counts)
    indptr = np.zeros(len(counts) + 1, dtype=np.int64)
    np.cumsum(counts, out=indptr[1:])
    flat = np.concatenate([idx[r, :counts[r]] for r in range(len(counts))]) if len(counts) else np.zeros(0)
    return indptr.astype(np.int32), _i32(flat)


def lpt_order(counts):
    counts = _i32(counts)
    order = np.empty_like(counts)
    _check(lib().oracle_lpt_order(len(counts), _p(counts), _p(order)), "oracle_lpt_order")
    return order


def sparse(q, k, v, n_tokens: int, block_q: int, block_k: int, scale: float, indptr, kv_idx, items=None):
    """Attention restricted to the listed key blocks. Returns (o [n][R][d], lse [n][R]) fp64."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    indptr, kv_idx = _i32(indptr), _i32(kv_idx)
    H, Np, d = q.shape
    it = _items(H, Np, block_q, items)
    o = np.empty((len(it), block_q, d), dtype=np.float64)
    lse = np.empty((len(it), block_q), dtype=np.float64)
    _check(lib().oracle_sparse(H, n_tokens, Np, d, block_q, block_k, scale, _p(q), _p(k), _p(v), _p(indptr),
                               _p(kv_idx), len(it), _p(it), _p(o), _p(lse)), "oracle_sparse")
    return o, lse


def recall(m, indptr, kv_idx, rows=None):
    """Recall of a CSR pattern under fp64 masses m[t] of CSR rows `rows[t]` (all rows if None)."""
    m = np.ascontiguousarray(m, dtype=np.float64)
    n, nk = m.shape
    rows = np.arange(n, dtype=np.int32) if rows is None else _i32(rows)
    indptr, kv_idx = _i32(indptr), _i32(kv_idx)
    return float(lib().oracle_recall(nk, n, _p(m), _p(indptr), _p(kv_idx), _p(rows)))
