"""Host-side helpers around the C ABI, checked on the CPU: the token upload keeps the generator's bits, and the
buffer harness allocates every caller-owned buffer with the layout and size include/losa.h states."""
import numpy as np
import pytest
import torch

import free_block_sparse_losa_b200 as L
from free_block_sparse_losa_b200 import build as B
from free_block_sparse_losa_b200.harness import LayerBuffers, host_tokens_to_device
from losa_synth import CONFIGS, LayerConfig, make_layer


@pytest.fixture(scope="module", autouse=True)
def _lib():
    B.build()
    L.load()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_token_upload_keeps_the_generated_values(dtype):
    cfg = LayerConfig("upload", heads=2, grid=(2, 5, 7), head_dim=64, block=64, dtype=dtype, amplitude=3.0,
                      ell_range=(1.0, 4.0), n_sinks=1, seed=11)
    layer = make_layer(cfg)
    t = host_tokens_to_device(layer.q, dtype, device="cpu")
    assert t.dtype == (torch.bfloat16 if dtype == "bf16" else torch.float32)
    assert t.shape == (cfg.heads, cfg.n_padded, cfg.head_dim) and t.is_contiguous()
    np.testing.assert_array_equal(t.float().numpy(), layer.all_f32("q"))


@pytest.mark.parametrize("block_k", [0, 32])
def test_layer_buffers_follow_the_header_layout(block_k):
    cfg = CONFIGS["wan1.3b480"]
    buf = LayerBuffers(cfg.heads, cfg.n_tokens, cfg.n_padded, cfg.head_dim, cfg.block, cfg.dtype, device="cpu",
                       block_k=block_k)
    H, Np, d = cfg.heads, cfg.n_padded, cfg.head_dim
    nq, nk = Np // 128, Np // (block_k or 128)
    assert (buf.shape.heads, buf.shape.n_tokens, buf.shape.n_padded, buf.shape.head_dim) == (H, cfg.n_tokens, Np, d)
    assert (buf.shape.block_q, buf.shape.block_k, buf.shape.dtype) == (128, block_k or 128, L.DTYPE_BF16)
    assert buf.o.shape == (H, Np, d) and buf.o.dtype == torch.bfloat16
    assert buf.lse.shape == (H, Np) and buf.lse.dtype == torch.float32
    assert buf.mass.shape == (H, nq, nk) and buf.mass.dtype == torch.float32
    assert buf.indptr.shape == (H * nq + 1,) and buf.indptr.dtype == torch.int32
    assert buf.kv_idx.shape == (H * nq * nk,) and buf.kv_idx.dtype == torch.int32  # the worst case: every block
    assert buf.order.shape == (H * nq,) and buf.order.dtype == torch.int32
    ws = L.losa_select_workspace_bytes(buf.shape)
    assert ws > 0 and buf.workspace.numel() >= ws and buf.workspace.numel() % 16 == 0


def test_csr_host_reads_only_the_filled_lists():
    cfg = CONFIGS["tiny"]
    buf = LayerBuffers.for_config(cfg, device="cpu")
    rows = buf.rows
    counts = np.arange(rows) % 3 + 1
    indptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    buf.indptr.copy_(torch.from_numpy(indptr))
    buf.kv_idx.fill_(-9)
    buf.kv_idx[: indptr[-1]] = torch.arange(int(indptr[-1]), dtype=torch.int32) % buf.nk
    buf.order.copy_(torch.arange(rows, dtype=torch.int32).flip(0))
    gi, gk, go = buf.csr_host()
    np.testing.assert_array_equal(gi, indptr)
    assert len(gk) == indptr[-1] and (gk >= 0).all()
    np.testing.assert_array_equal(go, np.arange(rows)[::-1])
