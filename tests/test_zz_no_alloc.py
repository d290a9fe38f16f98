"""losa_select_noalloc: selection with the library's fixed device scratch, for callers that cannot allocate
device memory when they call (a server whose memory pool already holds the GPU's memory, a plugin without a
workspace, a path where cudaMalloc would synchronise). Its output must equal losa_select's, bit for bit, on
consecutive calls that reuse the same scratch. This file is collected last on purpose."""
import numpy as np
import pytest
import torch

import free_block_sparse_losa_b200 as L
from tests.gpu_util import require_gpu


def _masses(seed, rows, nk):
    rng = np.random.default_rng(seed)
    m = np.exp(rng.standard_normal((rows, nk)) * 8.0)
    return (m / m.sum(axis=1, keepdims=True)).astype(np.float32)


def _outputs(rows, nk):
    return (torch.full((rows + 1,), -1, dtype=torch.int32, device="cuda"),
            torch.full((rows * nk,), -1, dtype=torch.int32, device="cuda"),
            torch.full((rows,), -1, dtype=torch.int32, device="cuda"))


@pytest.mark.gpu
def test_noalloc_matches_workspace_select_on_consecutive_calls():
    require_gpu()
    H, nb = 12, 256  # the Wan2.1-480p-shaped layer's block grid: 3.2 MB of scratch
    shape = L.make_shape(H, nb * 128 - 8, nb * 128, 128, 128, 128, "bf16")
    rows = H * nb
    ws = torch.empty(L.losa_select_workspace_bytes(shape), dtype=torch.uint8, device="cuda")
    for call, (seed, tau) in enumerate([(1, 0.99), (2, 0.9)]):
        mass = torch.from_numpy(_masses(seed, rows, nb).ravel()).cuda()
        ref = _outputs(rows, nb)
        got = _outputs(rows, nb)
        L.losa_select(shape, mass, tau, *ref, ws)
        L.losa_select_noalloc(shape, mass, tau, *got)
        assert L.losa_get_device_error() == 0
        nnz = int(ref[0][-1].item())
        assert torch.equal(ref[0], got[0]), f"indptr differs on call {call}"
        assert torch.equal(ref[1][:nnz], got[1][:nnz]), f"block lists differ on call {call}"
        assert torch.equal(ref[2], got[2]), f"work order differs on call {call}"


@pytest.mark.gpu
def test_noalloc_rejects_shapes_beyond_its_scratch():
    require_gpu()
    big = L.make_shape(24, 118800, 118912, 128, 128, 128, "bf16")  # needs 83 MB of scratch
    rows, nk = 24 * 929, 929
    mass = torch.zeros(rows * nk, dtype=torch.float32, device="cuda")
    indptr, idx, order = _outputs(rows, nk)
    st = L.losa_select_noalloc(big, mass, 0.99, indptr, idx, order, raise_on_error=False)
    assert st == -3
