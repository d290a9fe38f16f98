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
    for name in ("losa_dense_profile", "losa_select", "losa_select_noalloc", "losa_select_topk", "losa_sparse_attn",
                 "losa_get_device_error",
                 "losa_selftest_wait_timeout"):
        getattr(L, name).restype = i32
    _lib = L
    return L


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


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
    st = load().losa_dense_profile(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), float(scale), _ptr(o), _ptr(lse),
                                   _ptr(mass), _stream(stream))
    return _check(st, "losa_dense_profile", raise_on_error)


def losa_select_workspace_bytes(shape) -> int:
    return int(load().losa_select_workspace_bytes(ctypes.byref(shape)))


def losa_select(shape, mass, tau, indptr, kv_block_idx, order, workspace, idx_capacity=None, ws_bytes=None,
                stream=None, raise_on_error=True):
    cap = kv_block_idx.numel() if idx_capacity is None else idx_capacity
    wsb = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    st = load().losa_select(ctypes.byref(shape), _ptr(mass), float(tau), _ptr(indptr), _ptr(kv_block_idx), int(cap),
                            _ptr(order), _ptr(workspace), int(wsb), _stream(stream))
    return _check(st, "losa_select", raise_on_error)


def losa_select_topk(shape, mass, k_blocks, indptr, kv_block_idx, order, workspace, idx_capacity=None, ws_bytes=None,
                     stream=None, raise_on_error=True):
    cap = kv_block_idx.numel() if idx_capacity is None else idx_capacity
    wsb = workspace.numel() * workspace.element_size() if ws_bytes is None else ws_bytes
    st = load().losa_select_topk(ctypes.byref(shape), _ptr(mass), int(k_blocks), _ptr(indptr), _ptr(kv_block_idx),
                                 int(cap), _ptr(order), _ptr(workspace), int(wsb), _stream(stream))
    return _check(st, "losa_select_topk", raise_on_error)


def losa_select_noalloc(shape, mass, tau, indptr, kv_block_idx, order, idx_capacity=None, stream=None,
                        raise_on_error=True):
    """losa_select with the library's fixed device scratch instead of a caller workspace (see include/losa.h)."""
    cap = kv_block_idx.numel() if idx_capacity is None else idx_capacity
    st = load().losa_select_noalloc(ctypes.byref(shape), _ptr(mass), float(tau), _ptr(indptr), _ptr(kv_block_idx),
                                    int(cap), _ptr(order), _stream(stream))
    return _check(st, "losa_select_noalloc", raise_on_error)


def losa_sparse_attn(shape, q, k, v, scale, indptr, kv_block_idx, order, o, lse=None, stream=None,
                     raise_on_error=True):
    st = load().losa_sparse_attn(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), float(scale), _ptr(indptr),
                                 _ptr(kv_block_idx), _ptr(order), _ptr(o), _ptr(lse), _stream(stream))
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
