"""CPU checks of the C-ABI library: it loads, exports every entry point include/losa.h declares, and its
host-side argument checks reject bad calls before anything is launched (no GPU needed: none of these calls
reaches the CUDA runtime)."""
import ctypes
import os
import re

import pytest

import free_block_sparse_losa_b200 as L
from free_block_sparse_losa_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load()


def _declared():
    names = set()
    for h in os.listdir(os.path.join(ROOT, "include")):
        if h.endswith(".h"):
            text = open(os.path.join(ROOT, "include", h)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(losa_[a-z0-9_]+)\s*\(", text))
    return names


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert {"losa_dense_profile", "losa_select", "losa_sparse_attn", "losa_select_workspace_bytes",
            "losa_get_device_error", "losa_status_string"} <= names
    raw = ctypes.CDLL(L.library_path())
    for n in sorted(names):
        assert hasattr(raw, n), n


def test_every_exported_symbol_is_declared(lib):
    """The reverse direction: the library exports no losa_* entry point that the header does not declare (read from
    the dynamic symbol table with nm; skipped where nm is missing)."""
    import shutil
    import subprocess
    if not shutil.which("nm"):
        pytest.skip("nm not available")
    out = subprocess.run(["nm", "-D", "--defined-only", L.library_path()], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.split() and line.split()[-1].startswith("losa_")}
    assert exported and exported <= _declared(), exported - _declared()


def test_status_strings(lib):
    for code, name in L.STATUS.items():
        assert L.losa_status_string(code) == name
    assert L.losa_version() >= 100


FAKE = 0x10000  # aligned, never dereferenced: every call below fails its host checks first


def test_shape_validation(lib):
    good = L.make_shape(2, 1000, 1024, 128, 128, 128, "bf16")
    assert L.losa_select_workspace_bytes(good) > 0
    bad = [
        L.make_shape(0, 1000, 1024, 128, 128, 128, "bf16"),      # no heads
        L.make_shape(2, 1100, 1024, 128, 128, 128, "bf16"),      # N > Np
        L.make_shape(2, 1000, 1000, 128, 128, 128, "bf16"),      # Np not a multiple of the block
        L.make_shape(2, 800, 1024, 128, 128, 128, "bf16"),       # an all-padding block
        L.make_shape(2, 1000, 1024, 128, 128, 128, 7),           # unknown dtype
    ]
    for s in bad:
        assert L.losa_select_workspace_bytes(s) == 0
        assert L.losa_dense_profile(s, FAKE, FAKE, FAKE, 0.1, FAKE, FAKE, FAKE, stream=0,
                                    raise_on_error=False) == -1
        assert L.losa_sparse_attn(s, FAKE, FAKE, FAKE, 0.1, FAKE, FAKE, None, FAKE, stream=0,
                                  raise_on_error=False) == -1
    assert lib.losa_dense_profile(None, None, None, None, 0.1, None, None, None, None) == -1


def test_pointer_and_tau_validation(lib):
    s = L.make_shape(2, 1000, 1024, 128, 128, 128, "bf16")
    # misaligned / null pointers
    assert L.losa_dense_profile(s, FAKE + 2, FAKE, FAKE, 0.1, FAKE, FAKE, None, stream=0, raise_on_error=False) == -1
    assert L.losa_dense_profile(s, FAKE, FAKE, None, 0.1, FAKE, FAKE, None, stream=0, raise_on_error=False) == -1
    # mass requested without lse
    assert L.losa_dense_profile(s, FAKE, FAKE, FAKE, 0.1, FAKE, None, FAKE, stream=0, raise_on_error=False) == -1
    assert L.losa_dense_profile(s, FAKE, FAKE, FAKE, float("nan"), FAKE, FAKE, None, stream=0,
                                raise_on_error=False) == -1
    # the sparse call's int32 arrays must be 4-byte aligned (order may be NULL)
    for ip, kv, od in ((FAKE + 2, FAKE, None), (FAKE, FAKE + 1, None), (FAKE, FAKE, FAKE + 2)):
        assert L.losa_sparse_attn(s, FAKE, FAKE, FAKE, 0.1, ip, kv, od, FAKE, stream=0, raise_on_error=False) == -1
    ws = L.losa_select_workspace_bytes(s)
    for tau in (0.0, -1.0, 1.5, float("nan")):
        assert L.losa_select(s, FAKE, tau, FAKE, FAKE, FAKE, FAKE, idx_capacity=2 * 8 * 8, ws_bytes=ws, stream=0,
                             raise_on_error=False) == -1


def test_one_pass_profile_host_checks(lib):
    """losa_dense_profile_ws refuses bad arguments on the host, before it asks the device for its SM count: bad
    shapes, null or misaligned pointers (the workspace included) and a non-finite scale. The workspace size is 0 for
    a bad shape and for the fp32 path, which takes no workspace."""
    for s in (L.make_shape(0, 1000, 1024, 128, 128, 128, "bf16"), L.make_shape(2, 1100, 1024, 128, 128, 128, "bf16"),
              L.make_shape(2, 1000, 1024, 128, 128, 128, 7), L.make_shape(2, 1000, 1024, 64, 128, 128, "f32")):
        assert L.losa_dense_profile_workspace_bytes(s) == 0
    for s in (L.make_shape(0, 1000, 1024, 128, 128, 128, "bf16"), L.make_shape(2, 1100, 1024, 128, 128, 128, "bf16")):
        assert L.losa_dense_profile_ws(s, FAKE, FAKE, FAKE, 0.1, FAKE, FAKE, FAKE, FAKE, ws_bytes=1 << 30, stream=0,
                                       raise_on_error=False) == -1
    s = L.make_shape(2, 1000, 1024, 128, 128, 128, "bf16")
    for args in ((FAKE + 2, FAKE, FAKE, 0.1, FAKE, FAKE, FAKE, FAKE),       # misaligned q
                 (FAKE, FAKE, FAKE, 0.1, FAKE, FAKE, FAKE, FAKE + 4),       # misaligned workspace
                 (FAKE, FAKE, FAKE, 0.1, FAKE, FAKE, FAKE, 0),              # null workspace
                 (FAKE, FAKE, FAKE, 0.1, FAKE, 0, FAKE, FAKE),              # masses without lse
                 (FAKE, FAKE, FAKE, float("nan"), FAKE, FAKE, FAKE, FAKE)):  # non-finite scale
        assert L.losa_dense_profile_ws(s, *args, ws_bytes=1 << 30, stream=0, raise_on_error=False) == -1
    with pytest.raises(ValueError):  # a raw workspace pointer needs its size
        L.losa_dense_profile_ws(s, FAKE, FAKE, FAKE, 0.1, FAKE, FAKE, FAKE, FAKE, stream=0)


def test_capacity_and_unsupported(lib):
    s = L.make_shape(2, 1000, 1024, 128, 128, 128, "bf16")
    ws = L.losa_select_workspace_bytes(s)
    rows, nk = 2 * 8, 8
    assert L.losa_select(s, FAKE, 0.99, FAKE, FAKE, FAKE, FAKE, idx_capacity=rows * nk - 1, ws_bytes=ws, stream=0,
                         raise_on_error=False) == -3
    assert L.losa_select(s, FAKE, 0.99, FAKE, FAKE, FAKE, FAKE, idx_capacity=rows * nk, ws_bytes=ws - 1, stream=0,
                         raise_on_error=False) == -3
    # bf16 is implemented for head_dim 128, block_q 128 and block_k 128 or 32, up to 1024 blocks of 128 per head
    for s_bad in (L.make_shape(2, 1000, 1024, 64, 128, 128, "bf16"),
                  L.make_shape(2, 1000, 1024, 128, 128, 64, "bf16"),
                  L.make_shape(2, 1000, 1024, 128, 64, 64, "bf16"),
                  L.make_shape(1, 131100, 131200, 128, 128, 128, "bf16")):
        assert L.losa_dense_profile(s_bad, FAKE, FAKE, FAKE, 0.1, FAKE, FAKE, None, stream=0,
                                    raise_on_error=False) == -2
        assert L.losa_sparse_attn(s_bad, FAKE, FAKE, FAKE, 0.1, FAKE, FAKE, None, FAKE, stream=0,
                                  raise_on_error=False) == -2
    # more than 8192 key blocks per selection row
    wide = L.make_shape(1, 262200, 262272, 128, 128, 32, "bf16")
    assert L.losa_select(wide, FAKE, 0.99, FAKE, FAKE, FAKE, FAKE, idx_capacity=1 << 40,
                         ws_bytes=L.losa_select_workspace_bytes(wide), stream=0, raise_on_error=False) == -2
    # more than 2^20 items in one selection call, and lists whose offsets could leave int32
    for big in (L.make_shape(1100, 130000, 130048, 128, 128, 128, "bf16"),
                L.make_shape(600, 131000, 131072, 128, 128, 32, "bf16")):
        wsb = L.losa_select_workspace_bytes(big)
        assert L.losa_select(big, FAKE, 0.99, FAKE, FAKE, FAKE, FAKE, idx_capacity=1 << 40, ws_bytes=wsb, stream=0,
                             raise_on_error=False) == -2
    # two guidance branches at the HunyuanVideo shape (44592 items) are supported: the call gets as far as the
    # workspace check, which comes after the size limits (one byte short, so nothing is launched)
    cfg2 = L.make_shape(48, 118800, 118912, 128, 128, 128, "bf16")
    wsb = L.losa_select_workspace_bytes(cfg2)
    assert L.losa_select(cfg2, FAKE, 0.99, FAKE, FAKE, FAKE, FAKE, idx_capacity=1 << 40, ws_bytes=wsb - 1, stream=0,
                         raise_on_error=False) == -3


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setenv("LOSA_LIBRARY", "/nonexistent/liblosa.so")
    monkeypatch.setattr(L, "_lib", None)
    with pytest.raises(RuntimeError):
        L.load()


def test_binding_refuses_wrong_tensors_before_the_call(lib):
    """The binding checks each tensor against the shape (dtype, element count, layout, device) and raises before
    anything reaches the library, so a wrong buffer is never read or written out of bounds."""
    import torch
    H, N, Np, d, R = 2, 1000, 1024, 128, 128
    s = L.make_shape(H, N, Np, d, R, R, "bf16")
    tok = lambda n=H * Np * d, dt=torch.bfloat16: torch.empty(n, dtype=dt)  # noqa: E731
    i32 = lambda n: torch.empty(n, dtype=torch.int32)  # noqa: E731
    f32 = lambda n: torch.empty(n, dtype=torch.float32)  # noqa: E731
    rows, nk = H * (Np // R), Np // R
    with pytest.raises(ValueError, match="q: expected torch.bfloat16"):
        L.losa_dense_profile(s, tok(dt=torch.float16), tok(), tok(), 0.1, tok(), f32(H * Np), None)
    with pytest.raises(ValueError, match="v: holds"):
        L.losa_dense_profile(s, tok(), tok(), tok(H * Np * d - 1), 0.1, tok(), f32(H * Np), None)
    with pytest.raises(ValueError, match="mass: holds"):
        L.losa_dense_profile(s, tok(), tok(), tok(), 0.1, tok(), f32(H * Np), f32(rows * nk - 1))
    with pytest.raises(ValueError, match="o: expected a contiguous"):
        L.losa_dense_profile(s, tok(), tok(), tok(), 0.1, tok(2 * H * Np * d)[::2], f32(H * Np), None)
    with pytest.raises(ValueError, match="q: expected a CUDA tensor"):
        L.losa_dense_profile(s, tok(), tok(), tok(), 0.1, tok(), f32(H * Np), None)
    with pytest.raises(ValueError, match="indptr: expected torch.int32"):
        L.losa_select(s, f32(rows * nk), 0.99, torch.empty(rows + 1, dtype=torch.int64), i32(rows * nk), i32(rows),
                      torch.empty(64, dtype=torch.uint8))
    with pytest.raises(ValueError, match="order: holds"):
        L.losa_select(s, f32(rows * nk), 0.99, i32(rows + 1), i32(rows * nk), i32(rows - 1),
                      torch.empty(64, dtype=torch.uint8))
    with pytest.raises(ValueError, match="kv_block_idx: holds"):
        L.losa_select(s, f32(rows * nk), 0.99, i32(rows + 1), i32(rows * nk), i32(rows),
                      torch.empty(64, dtype=torch.uint8), idx_capacity=rows * nk + 1)
    with pytest.raises(ValueError, match="workspace: holds"):
        L.losa_select(s, f32(rows * nk), 0.99, i32(rows + 1), i32(rows * nk), i32(rows),
                      torch.empty(64, dtype=torch.uint8), ws_bytes=65)
    with pytest.raises(ValueError, match="a raw pointer needs idx_capacity"):
        L.losa_select_noalloc(s, FAKE, 0.99, FAKE, FAKE, FAKE)
    with pytest.raises(ValueError, match="lse: expected torch.float32"):
        L.losa_sparse_attn(s, tok(), tok(), tok(), 0.1, i32(rows + 1), i32(1), None, tok(),
                           torch.empty(H * Np, dtype=torch.float64))


C_CALLER = r"""
#include <stdio.h>
#include <string.h>
#include "losa.h"
int main(void) {
    losa_shape good = {2, 1000, 1024, 128, 128, 128, LOSA_DTYPE_BF16};
    losa_shape bad = good;
    bad.n_padded = 1000;
    if (losa_version() < 100) return 1;
    if (strcmp(losa_status_string(LOSA_ERR_CAPACITY), "LOSA_ERR_CAPACITY") != 0) return 2;
    if (losa_select_workspace_bytes(&good) == 0 || losa_select_workspace_bytes(&bad) != 0) return 3;
    if (losa_dense_profile(&bad, 0, 0, 0, 0.1f, 0, 0, 0, 0) != LOSA_ERR_INVALID_ARG) return 4;
    if (losa_sparse_attn(&good, 0, 0, 0, 0.1f, 0, 0, 0, 0, 0, 0) != LOSA_ERR_INVALID_ARG) return 5;
    printf("ok\n");
    return 0;
}
"""


def test_plain_c_caller(lib, tmp_path):
    """The boundary is a C ABI: a C99 program that includes only include/losa.h, links liblosa.so and calls the
    host-side entry points runs without Python or torch (none of these calls reaches the CUDA runtime)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    cuda_inc = "/usr/local/cuda/include"
    if not gcc or not os.path.isdir(cuda_inc):
        pytest.skip("gcc or the CUDA headers are not available")
    src = tmp_path / "caller.c"
    src.write_text(C_CALLER)
    exe = tmp_path / "caller"
    libdir = os.path.dirname(L.library_path())
    subprocess.run([gcc, "-std=c99", "-Wall", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc, str(src),
                    "-L", libdir, "-llosa", f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    run = subprocess.run([str(exe)], capture_output=True, text=True)
    assert run.returncode == 0 and run.stdout.strip() == "ok", (run.returncode, run.stdout, run.stderr)
