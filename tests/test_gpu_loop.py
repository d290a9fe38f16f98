"""GPU check of the reuse loop (LoSA page, Methodology Summary: dense steps until the construction step, then the
frozen block indices for every later step, with Q/K/V recomputed each step): the pattern selected at step 0 is reused
on drifted inputs, and the sparse output of a later step matches the oracle's restricted attention over that same
frozen pattern on the drifted inputs."""
import math

import numpy as np
import pytest
import torch

import free_block_sparse_losa_b200 as L
from free_block_sparse_losa_b200.harness import LayerBuffers
from losa_synth import CONFIGS, Drift, make_layer, sample_items
from tests.gpu_util import check_lse, check_output, item_rows, require_gpu

pytestmark = pytest.mark.gpu


def test_frozen_pattern_reused_on_drifted_inputs(oracle_mod):
    require_gpu()
    cfg = CONFIGS["loop"]  # Wan2.1-480p-shaped layers; 2 of its 30 layers, 4 steps
    layers = [make_layer(cfg, li) for li in range(2)]
    drift = Drift(cfg, layers, seed=cfg.seed)
    scale = 1.0 / math.sqrt(cfg.head_dim)
    bufs = [LayerBuffers.for_config(cfg) for _ in layers]
    for li, b in enumerate(bufs):
        q, k, v = drift.tokens(li)
        b.profile(q, k, v, scale)
        b.select(0.99)
    frozen = [b.csr_host() for b in bufs]
    for _ in range(3):
        drift.advance()
        for li, b in enumerate(bufs):
            b.sparse(*drift.tokens(li), scale)
    assert L.losa_get_device_error() == 0
    for li, b in enumerate(bufs):
        gi, gk, go = b.csr_host()
        assert np.array_equal(gi, frozen[li][0]) and np.array_equal(gk, frozen[li][1])  # lists untouched
        q, k, v = drift.tokens(li)
        qf, kf, vf = (x.float().cpu().numpy() for x in (q, k, v))
        items = sample_items(cfg, 16, seed=li)
        ref_o, ref_l = oracle_mod.sparse(qf, kf, vf, cfg.n_tokens, cfg.block, cfg.block, scale, gi, gk, items)
        lse = torch.empty_like(b.lse)
        b.sparse(q, k, v, scale, lse=lse)
        got, valid = item_rows(cfg, items, b.o.float().cpu().numpy())
        gl, _ = item_rows(cfg, items, lse.cpu().numpy())
        check_output(got[valid], ref_o[valid], f"loop layer {li}")
        check_lse(gl[valid], ref_l[valid], f"loop layer {li}")
