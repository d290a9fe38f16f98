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


def test_construction_at_step_three_and_cross_step_recall(oracle_mod):
    """The LoSA page's schedule (Methodology Summary): dense steps 0, 1, 2, the pattern built at the dense step t0 = 3,
    frozen afterwards; and its measurement of cross-step stability (Motivation Summary, "Near-lossless patterns are
    stable across denoising"): the recall of the frozen pattern under a later step's exact masses. At construction
    every row keeps at least tau of its own mass; at step 6 the recall the benchmark reports (from the GPU's masses)
    equals the oracle's recall fed the same masses and lists, and agrees with the oracle's recall under its own fp64
    masses on sampled rows; the sparse output at step 6 matches the oracle over the frozen lists."""
    require_gpu()
    import bench

    cfg = CONFIGS["loop"]
    layers = [make_layer(cfg, li) for li in range(2)]
    drift = Drift(cfg, layers, seed=cfg.seed)
    scale = 1.0 / math.sqrt(cfg.head_dim)
    tau, t0, t_probe = 0.99, 3, 6
    bufs = [LayerBuffers.for_config(cfg) for _ in layers]
    probe = LayerBuffers.for_config(cfg)
    frozen = []
    for step in range(t_probe + 1):
        if step > 0:
            drift.advance()
        for li, b in enumerate(bufs):
            q, k, v = drift.tokens(li)
            if step < t0:
                L.losa_dense_profile(b.shape, q, k, v, scale, b.o, b.lse, None)
            elif step == t0:
                b.profile(q, k, v, scale)
                b.select(tau)
                gi, gk, _ = b.csr_host()
                m = b.mass.cpu().numpy().reshape(b.rows, b.nk).astype(np.float64)
                # by construction: every row keeps >= tau of its own (GPU) mass, up to fp32 rounding of the masses
                for r in range(b.rows):
                    assert oracle_mod.recall(m[r:r + 1], gi[r:r + 2] - gi[r], gk[gi[r]:gi[r + 1]]) >= tau - 1e-5
                frozen.append((gi, gk))
            else:
                b.sparse(q, k, v, scale)
    assert L.losa_get_device_error() == 0
    items = sample_items(cfg, 16, seed=5)
    for li, b in enumerate(bufs):
        gi, gk = frozen[li]
        q, k, v = drift.tokens(li)
        probe.profile(q, k, v, scale)
        m = probe.mass.cpu().numpy().reshape(probe.rows, probe.nk).astype(np.float64)
        r_bench = bench.pattern_recall(m, gi, gk)
        r_oracle = oracle_mod.recall(m, gi, gk)
        assert abs(r_bench - r_oracle) <= 1e-10 * r_oracle, (r_bench, r_oracle)
        assert 0.0 < r_oracle <= 1.0 + 1e-6
        qf, kf, vf = (x.float().cpu().numpy() for x in (q, k, v))
        om = oracle_mod.mass(qf, kf, cfg.n_tokens, cfg.block, cfg.block, scale, items)
        r_exact = oracle_mod.recall(om, gi, gk, rows=items)
        r_gpu_rows = oracle_mod.recall(m[items], gi, gk, rows=items)
        assert abs(r_exact - r_gpu_rows) <= 1e-4, (r_exact, r_gpu_rows)
        ref_o, ref_l = oracle_mod.sparse(qf, kf, vf, cfg.n_tokens, cfg.block, cfg.block, scale, gi, gk, items)
        got, valid = item_rows(cfg, items, b.o.float().cpu().numpy())
        check_output(got[valid], ref_o[valid], f"step {t_probe} layer {li}")
    assert L.losa_get_device_error() == 0
