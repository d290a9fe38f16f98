"""Python binding of the LoSA C ABI (include/losa.h): argument marshalling only.

Every function has the name of its C entry point, takes torch CUDA tensors (or raw device pointers as ints)
and passes their pointers, sizes and the current CUDA stream to the library. All computation happens in the
library's CUDA kernels; there is no fallback. Importing this module does not load the library; the first call
does, and raises if liblosa.so is missing (build it with `python -m free_block_sparse_losa_b200.build`).
"""
from __future__ import annotations

import ctypes
import os

__all__ = ["LosaShape", "LosaError", "make_shape", "losa_dense_profile", "losa_select", "losa_select_noalloc",
           "losa_select_topk", "losa_sparse_attn",
           "losa_select_workspace_bytes", "losa_get_device_error", "losa_selftest_wait_timeout",
           "losa_set_wait_limit_ns", "losa_status_string", "losa_version", "library_path", "load",
           "DTYPE_F32", "DTYPE_BF16", "STATUS"]

DTYPE_F32 = 0
DTYPE_BF16 = 1
STATUS = {0: "LOSA_OK", -1: "LOSA_ERR_INVALID_ARG", -2: "LOSA_ERR_UNSUPPORTED", -3: "LOSA_ERR_CAPACITY",
          -4: "LOSA_ERR_CUDA", -5: "LOSA_ERR_DEVICE_FAULT", -6: "LOSA_ERR_TIMEOUT"}

_HERE = os.path.dirname(os.path.abspath(__file__))
_lib = None


class LosaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}")
        self.status = status


class LosaShape(ctypes.Structure):
    _fields_ = [("heads", ctypes.c_int32), ("n_tokens", ctypes.c_int32), ("n_padded", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("block_q", ctypes.c_int32), ("block_k", ctypes.c_int32),
                ("dtype", ctypes.c_int32)]


def make_shape(heads, n_tokens, n_padded, head_dim, block_q, block_k, dtype) -> LosaShape:
    if isinstance(dtype, str):
        dtype = {"f32": DTYPE_F32, "bf16": DTYPE_BF16}[dtype]
    return LosaShape(heads, n_tokens, n_padded, head_dim, block_q, block_k, dtype)


def library_path() -> str:
    return os.environ.get("LOSA_LIBRARY", os.path.join(_HERE, "liblosa.so"))


def load():
    """Load liblosa.so (once). Raises if it is missing: there is no other implementation."""
    global _lib
    if _lib is not None:
        return _lib
    path = library_path()
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library not built: {path} is missing")
    L = ctypes.CDLL(path)
    vp, i32, f32, f64, i64, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_double,
                                  ctypes.c_int64, ctypes.c_size_t)
    sp = ctypes.POINTER(LosaShape)
    L.losa_dense_profile.argtypes = [sp, vp, vp, vp, f32, vp, vp, vp, vp]
    L.losa_dense_profile_ws.argtypes = [sp, vp, vp, vp, f32, vp, vp, vp, vp, sz, vp]
    L.losa_dense_profile_workspace_bytes.argtypes = [sp]
    L.losa_dense_profile_workspace_bytes.restype = sz
    L.losa_select.argtypes = [sp, vp, f64, vp, vp, i64, vp, vp, sz, vp]
    L.losa_select_noalloc.argtypes = [sp, vp, f64, vp, vp, i64, vp, vp]
    L.losa_select_topk.argtypes = [sp, vp, i32, vp, vp, i64, vp, vp, sz, vp]
    L.losa_select_workspace_bytes.argtypes = [sp]
    L.losa_select_workspace_bytes.restype = sz
    L.losa_sparse_attn.argtypes = [sp, vp, vp, vp, f32, vp, vp, vp, vp, vp, vp]
    L.losa_get_device_error.argtypes = [vp]
    L.losa_selftest_wait_timeout.argtypes = [ctypes.c_uint32, vp]
    L.losa_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    L.losa_set_wait_limit_ns.restype = None
    L.losa_status_string.argtypes = [i32]
    L.losa_status_string.restype = ctypes.c_char_p
    L.losa_version.restype = ctypes.c_int
    for name in ("losa_dense_profile", "losa_dense_profile_ws", "losa_select", "losa_select_noalloc", "losa_select_topk",
                 "losa_sparse_attn",
                 "losa_get_device_error",
                 "losa_selftest_wait_timeout"):
        getattr(L, name).restype = i32
    _lib = L
    return L


def _dims(shape):
    """(H, Np, d, nq, nk) of a shape; 0 for a block count whose block size is not positive."""
    nq = shape.n_padded // shape.block_q if shape.block_q > 0 else 0
    nk = shape.n_padded // shape.block_k if shape.block_k > 0 else 0
    return max(shape.heads, 0), max(shape.n_padded, 0), max(shape.head_dim, 0), max(nq, 0), max(nk, 0)


def _token_dtype(shape):
    return {DTYPE_F32: "float32", DTYPE_BF16: "bfloat16"}.get(shape.dtype)


def _ptrs(*specs):
    """Device pointers of arguments given as (value, name, dtype, numel). None stays NULL and an int is taken as a raw
    device pointer (the caller vouches for its size). A tensor must have the expected dtype (if given), hold at least
    `numel` elements (if given), be contiguous and live on the current CUDA device, so that a wrong buffer is refused
    here instead of being read or written out of bounds. The dtype, size and layout of every argument are checked
    before any argument's device."""
    tensors = [(t, name) for t, name, _, _ in specs if t is not None and not isinstance(t, int)]
    if tensors:
        import torch
    for t, name, dtype, numel in specs:
        if t is None or isinstance(t, int):
            continue
        if dtype is not None and t.dtype != getattr(torch, dtype):
            raise ValueError(f"{name}: expected torch.{dtype}, got {t.dtype}")
        if numel is not None and t.numel() < numel:
            raise ValueError(f"{name}: holds {t.numel()} elements, the shape needs {numel}")
        if not t.is_contiguous():
            raise ValueError(f"{name}: expected a contiguous tensor")
    for t, name in tensors:
        if not t.is_cuda:
            raise ValueError(f"{name}: expected a CUDA tensor")
        if t.device.index != torch.cuda.current_device():
            raise ValueError(f"{name}: lives on {t.device}, the current device is cuda:{torch.cuda.current_device()}")
    return tuple(t if (t is None or isinstance(t, int)) else t.data_ptr() for t, _, _, _ in specs)


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str, raise_on_error: bool):
    if status != 0 and raise_on_error:
        raise LosaError(status, where)
    return status


def losa_dense_profile(shape, q, k, v, scale, o, lse=None, mass=None, stream=None, raise_on_error=True):
    H, Np, d, nq, nk = _dims(shape)
    tdt = _token_dtype(shape)
    pq, pk, pv, po, pl, pm = _ptrs((q, "q", tdt, H * Np * d), (k, "k", tdt, H * Np * d), (v, "v", tdt, H * Np * d),
                                   (o, "o", tdt, H * Np * d), (lse, "lse", "float32", H * Np),
                                   (mass, "mass", "float32", H * nq * nk))
    st = load().losa_dense_profile(ctypes.byref(shape), pq, pk, pv, float(scale), po, pl, pm, _stream(stream))
    return _check(st, "losa_dense_profile", raise_on_error)


def losa_dense_profile_workspace_bytes(shape) -> int:
    return int(load().losa_dense_profile_workspace_bytes(ctypes.byref(shape)))


def losa_dense_profile_ws(shape, q, k, v, scale, o, lse, mass, workspace, ws_bytes=None, stream=None,
                          raise_on_error=True):
    """losa_dense_profile with the masses taken in the forward pass (needs a workspace of
    losa_dense_profile_workspace_bytes(shape) bytes)."""
    H, Np, d, nq, nk = _dims(shape)
    tdt = _token_dtype(shape)
    if isinstance(workspace, int):
        if ws_bytes is None:
            raise ValueError("workspace: a raw pointer needs ws_bytes")
        wsb = int(ws_bytes)
    else:
        have = workspace.numel() * workspace.element_size()
        wsb = have if ws_bytes is None else int(ws_bytes)
        if have < wsb:
            raise ValueError(f"workspace: holds {have} bytes, ws_bytes says {wsb}")
    pq, pk, pv, po, pl, pm, pw = _ptrs((q, "q", tdt, H * Np * d), (k, "k", tdt, H * Np * d),
                                       (v, "v", tdt, H * Np * d), (o, "o", tdt, H * Np * d),
                                       (lse, "lse", "float32", H * Np), (mass, "mass", "float32", H * nq * nk),
                                       (workspace, "workspace", None, None))
    st = load().losa_dense_profile_ws(ctypes.byref(shape), pq, pk, pv, float(scale), po, pl, pm, pw, wsb,
                                      _stream(stream))
    return _check(st, "losa_dense_profile_ws", raise_on_error)


def losa_select_workspace_bytes(shape) -> int:
    return int(load().losa_select_workspace_bytes(ctypes.byref(shape)))


def _select_args(shape, mass, indptr, kv_block_idx, order, idx_capacity, workspace=None, ws_bytes=None):
    """Pointers of the selection calls' arguments, the index capacity and the workspace size."""
    H, _, _, nq, nk = _dims(shape)
    if idx_capacity is None:
        if isinstance(kv_block_idx, int):
            raise ValueError("kv_block_idx: a raw pointer needs idx_capacity")
        cap, idx_numel = kv_block_idx.numel(), None
    else:
        cap = idx_numel = int(idx_capacity)
    wsb = None
    if workspace is not None:
        if isinstance(workspace, int):
            if ws_bytes is None:
                raise ValueError("workspace: a raw pointer needs ws_bytes")
            wsb = int(ws_bytes)
        else:
            have = workspace.numel() * workspace.element_size()
            wsb = have if ws_bytes is None else int(ws_bytes)
            if have < wsb:
                raise ValueError(f"workspace: holds {have} bytes, ws_bytes says {wsb}")
    ptrs = _ptrs((mass, "mass", "float32", H * nq * nk), (indptr, "indptr", "int32", H * nq + 1),
                 (kv_block_idx, "kv_block_idx", "int32", idx_numel), (order, "order", "int32", H * nq),
                 (workspace, "workspace", None, None))
    return ptrs, cap, wsb


def losa_select(shape, mass, tau, indptr, kv_block_idx, order, workspace, idx_capacity=None, ws_bytes=None,
                stream=None, raise_on_error=True):
    (pm, pi, pk, po, pw), cap, wsb = _select_args(shape, mass, indptr, kv_block_idx, order, idx_capacity, workspace,
                                                  ws_bytes)
    st = load().losa_select(ctypes.byref(shape), pm, float(tau), pi, pk, cap, po, pw, wsb, _stream(stream))
    return _check(st, "losa_select", raise_on_error)


def losa_select_topk(shape, mass, k_blocks, indptr, kv_block_idx, order, workspace, idx_capacity=None, ws_bytes=None,
                     stream=None, raise_on_error=True):
    (pm, pi, pk, po, pw), cap, wsb = _select_args(shape, mass, indptr, kv_block_idx, order, idx_capacity, workspace,
                                                  ws_bytes)
    st = load().losa_select_topk(ctypes.byref(shape), pm, int(k_blocks), pi, pk, cap, po, pw, wsb, _stream(stream))
    return _check(st, "losa_select_topk", raise_on_error)


def losa_select_noalloc(shape, mass, tau, indptr, kv_block_idx, order, idx_capacity=None, stream=None,
                        raise_on_error=True):
    """losa_select with the library's fixed device scratch instead of a caller workspace (see include/losa.h)."""
    (pm, pi, pk, po, _), cap, _ = _select_args(shape, mass, indptr, kv_block_idx, order, idx_capacity)
    st = load().losa_select_noalloc(ctypes.byref(shape), pm, float(tau), pi, pk, cap, po, _stream(stream))
    return _check(st, "losa_select_noalloc", raise_on_error)


def losa_sparse_attn(shape, q, k, v, scale, indptr, kv_block_idx, order, o, lse=None, stream=None,
                     raise_on_error=True):
    H, Np, d, nq, _ = _dims(shape)
    tdt = _token_dtype(shape)
    pq, pk, pv, pi, px, po, pout, pl = _ptrs(
        (q, "q", tdt, H * Np * d), (k, "k", tdt, H * Np * d), (v, "v", tdt, H * Np * d),
        (indptr, "indptr", "int32", H * nq + 1), (kv_block_idx, "kv_block_idx", "int32", None),
        (order, "order", "int32", H * nq), (o, "o", tdt, H * Np * d), (lse, "lse", "float32", H * Np))
    st = load().losa_sparse_attn(ctypes.byref(shape), pq, pk, pv, float(scale), pi, px, po, pout, pl,
                                 _stream(stream))
    return _check(st, "losa_sparse_attn", raise_on_error)


def losa_get_device_error(stream=None) -> int:
    return int(load().losa_get_device_error(_stream(stream)))


def losa_selftest_wait_timeout(limit_ns: int, stream=None, raise_on_error=True):
    st = load().losa_selftest_wait_timeout(int(limit_ns), _stream(stream))
    return _check(st, "losa_selftest_wait_timeout", raise_on_error)


def losa_set_wait_limit_ns(limit_ns: int):
    load().losa_set_wait_limit_ns(int(limit_ns))


def losa_status_string(status: int) -> str:
    return load().losa_status_string(int(status)).decode()


def losa_version() -> int:
    return int(load().losa_version())
