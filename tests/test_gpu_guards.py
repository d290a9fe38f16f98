"""Guard regions after every output buffer, and a saved-and-reloaded frozen pattern, on the GPU path.

- Every output of the three calls (dense profile: O, lse, M; selection: indptr, kv_block_idx, order; sparse: O, lse)
  goes into a buffer longer than the call needs, its tail filled with a sentinel; after the calls the tails must be
  untouched, and kv_block_idx must be untouched past the retained entries.
- The selection's pattern, saved with `pattern.save_pattern` and loaded back (LoSA page, Methodology Summary: the
  pattern built at step t0 is reused unchanged), gives the same sparse output, bit for bit."""
import math

import numpy as np
import pytest
import torch

import free_block_sparse_losa_b200 as L
from free_block_sparse_losa_b200.pattern import load_pattern, save_pattern
from losa_synth import LayerConfig, make_layer
from tests.gpu_util import device_inputs, require_gpu

pytestmark = pytest.mark.gpu
GUARD = 4096

CASES = {
    "C128-ragged": LayerConfig("guards-c128", heads=3, grid=(5, 13, 31), head_dim=128, block=128, dtype="bf16",
                               amplitude=4.0, ell_range=(1.0, 8.0), n_sinks=2, seed=201, taus=(0.99,)),
    "C32-ragged": LayerConfig("guards-c32", heads=3, grid=(5, 13, 31), head_dim=128, block=128, block_k=32,
                              dtype="bf16", amplitude=4.0, ell_range=(1.0, 8.0), n_sinks=2, seed=202, taus=(0.99,)),
}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _guarded(n, dtype, fill):
    t = torch.empty(n + GUARD, dtype=dtype, device="cuda")
    t.fill_(fill)
    return t


def _tail_intact(t, n, fill, what):
    tail = t[n:].cpu()
    ref = torch.full_like(tail, fill)
    same = torch.equal(tail.view(torch.int16), ref.view(torch.int16)) if t.dtype == torch.bfloat16 else \
        torch.equal(tail, ref)
    assert same, f"{what}: a write landed past the end of the buffer"


@pytest.mark.parametrize("case", sorted(CASES))
def test_outputs_stay_inside_their_buffers_and_patterns_reload(case, tmp_path):
    cfg = CASES[case]
    layer = make_layer(cfg)
    q, k, v = device_inputs(layer)
    bk = cfg.kblock
    shape = L.make_shape(cfg.heads, cfg.n_tokens, cfg.n_padded, cfg.head_dim, cfg.block, bk, cfg.dtype)
    H, Np, d = cfg.heads, cfg.n_padded, cfg.head_dim
    nq, nk = Np // cfg.block, Np // bk
    rows = H * nq
    scale = 1.0 / math.sqrt(d)
    bf, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    o1, lse1, mass = _guarded(H * Np * d, bf, -1234.0), _guarded(H * Np, f32, -7.5e30), _guarded(rows * nk, f32, -3.25)
    L.losa_dense_profile(shape, q, k, v, scale, o1, lse1, mass)
    indptr, idx, order = _guarded(rows + 1, i32, -123456), _guarded(rows * nk, i32, -654321), _guarded(rows, i32, -7)
    ws_bytes = L.losa_select_workspace_bytes(shape)
    ws = torch.empty((ws_bytes + 15) // 16 * 16, dtype=torch.uint8, device="cuda")
    L.losa_select(shape, mass, 0.99, indptr, idx, order, ws, idx_capacity=rows * nk)
    o2, lse2 = _guarded(H * Np * d, bf, -1234.0), _guarded(H * Np, f32, -7.5e30)
    L.losa_sparse_attn(shape, q, k, v, scale, indptr, idx, order, o2, lse2)
    torch.cuda.synchronize()
    assert L.losa_get_device_error() == 0
    for t, n, fill, what in ((o1, H * Np * d, -1234.0, "dense O"), (lse1, H * Np, -7.5e30, "dense lse"),
                             (mass, rows * nk, -3.25, "M"), (indptr, rows + 1, -123456, "indptr"),
                             (order, rows, -7, "order"), (o2, H * Np * d, -1234.0, "sparse O"),
                             (lse2, H * Np, -7.5e30, "sparse lse")):
        _tail_intact(t, n, fill, what)
    nnz = int(indptr[rows].item())
    _tail_intact(idx, nnz, -654321, "kv_block_idx past the retained entries")

    # the same pattern through a file
    path = str(tmp_path / f"{case}.npz")
    save_pattern(path, shape, 0.99, indptr[:rows + 1], idx[:nnz], order[:rows])
    tau, p_indptr, p_idx, p_order = load_pattern(path, shape)
    assert tau == 0.99 and np.array_equal(p_indptr, indptr[:rows + 1].cpu().numpy())
    o3 = torch.empty(H * Np * d, dtype=bf, device="cuda")
    L.losa_sparse_attn(shape, q, k, v, scale, torch.from_numpy(p_indptr).cuda(), torch.from_numpy(p_idx).cuda(),
                       torch.from_numpy(p_order).cuda(), o3)
    torch.cuda.synchronize()
    assert L.losa_get_device_error() == 0
    assert torch.equal(o3.view(torch.int16), o2[:H * Np * d].view(torch.int16))
