"""Device-buffer harness around the C ABI: allocates the caller-owned buffers of one attention layer with
PyTorch (device memory and streams only) and calls the three entry points in order. No computation happens
here; every step runs in the library's kernels."""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

from . import (DTYPE_BF16, DTYPE_F32, losa_dense_profile, losa_dense_profile_workspace_bytes, losa_dense_profile_ws,
               losa_select, losa_select_topk, losa_select_workspace_bytes, losa_sparse_attn, make_shape)


def host_tokens_to_device(a: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """[H][Np][d] host tokens (fp32 values, or uint16 bf16 bit patterns) -> contiguous device tensor."""
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(device)


def device_tokens_to_f32(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy()


@dataclass
class LayerBuffers:
    heads: int
    n_tokens: int
    n_padded: int
    head_dim: int
    block: int
    dtype: str
    device: str = "cuda"
    block_k: int = 0  # key block size when it differs from the query block size

    def __post_init__(self):
        bk = self.block_k or self.block
        self.shape = make_shape(self.heads, self.n_tokens, self.n_padded, self.head_dim, self.block, bk, self.dtype)
        self.nq = self.n_padded // self.block
        self.nk = self.n_padded // bk
        self.rows = self.heads * self.nq
        tdt = torch.bfloat16 if self.dtype == "bf16" else torch.float32
        dev = self.device
        self.o = torch.empty((self.heads, self.n_padded, self.head_dim), dtype=tdt, device=dev)
        self.lse = torch.empty((self.heads, self.n_padded), dtype=torch.float32, device=dev)
        self.mass = torch.empty((self.heads, self.nq, self.nk), dtype=torch.float32, device=dev)
        self.indptr = torch.empty(self.rows + 1, dtype=torch.int32, device=dev)
        self.kv_idx = torch.empty(self.rows * self.nk, dtype=torch.int32, device=dev)
        self.order = torch.empty(self.rows, dtype=torch.int32, device=dev)
        ws = losa_select_workspace_bytes(self.shape)
        self.workspace = torch.empty((ws + 15) // 16 * 16, dtype=torch.uint8, device=dev)
        pws = losa_dense_profile_workspace_bytes(self.shape)  # 0 on the fp32 path
        self.profile_workspace = torch.empty(max(16, (pws + 15) // 16 * 16), dtype=torch.uint8, device=dev)

    @classmethod
    def for_config(cls, cfg, device="cuda"):
        return cls(cfg.heads, cfg.n_tokens, cfg.n_padded, cfg.head_dim, cfg.block, cfg.dtype, device,
                   getattr(cfg, "block_k", 0))

    def profile(self, q, k, v, scale, with_mass=True, stream=None, one_pass=True):
        """The dense step; with_mass adds the block masses, in the forward pass (one_pass, the default) or in a
        second pass that needs no workspace."""
        if with_mass and one_pass:
            losa_dense_profile_ws(self.shape, q, k, v, scale, self.o, self.lse, self.mass, self.profile_workspace,
                                  stream=stream)
        else:
            losa_dense_profile(self.shape, q, k, v, scale, self.o, self.lse, self.mass if with_mass else None,
                               stream=stream)

    def select(self, tau, mass=None, stream=None):
        losa_select(self.shape, self.mass if mass is None else mass, tau, self.indptr, self.kv_idx, self.order,
                    self.workspace, stream=stream)

    def select_topk(self, k_blocks, mass=None, stream=None):
        losa_select_topk(self.shape, self.mass if mass is None else mass, k_blocks, self.indptr, self.kv_idx,
                         self.order, self.workspace, stream=stream)

    def sparse(self, q, k, v, scale, out=None, lse=None, stream=None, order=True):
        losa_sparse_attn(self.shape, q, k, v, scale, self.indptr, self.kv_idx, self.order if order else None,
                         self.o if out is None else out, lse, stream=stream)

    def csr_host(self):
        indptr = self.indptr.cpu().numpy()
        nnz = int(indptr[-1])
        return indptr, self.kv_idx[:nnz].cpu().numpy(), self.order.cpu().numpy()
