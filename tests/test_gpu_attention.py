"""GPU parity of losa_dense_profile and losa_sparse_attn against the fp64 oracle on the same rounded inputs.

Full comparison on the tiny fp32 configuration and on small bf16 layers that span several tiles and a ragged
tail; at the full sizes of the Wan2.1 / HunyuanVideo-shaped layers, in the launch configuration the benchmark
times, 64 seeded (head, query block) items per call including the tail block and a block holding a sink token.
Definitions: "LoSA: Near-Lossless Sparse Attention for Training-Free Video Diffusion Acceleration", Motivation
Summary (A, M) and Methodology Summary (selection; attention restricted to the retained blocks).
"""
import math

import numpy as np
import pytest
import torch

import free_block_sparse_losa_b200 as L
from free_block_sparse_losa_b200.harness import LayerBuffers
from losa_synth import CONFIGS, LayerConfig, make_layer, sample_items
from tests.gpu_util import (check_lse, check_mass, check_output, compare_select, device_inputs, item_rows,
                            require_gpu, scale_of)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


SMALL = {
    "bf16-2x(4x16x16)": LayerConfig("small-bf16", heads=2, grid=(4, 16, 16), head_dim=128, block=128, dtype="bf16",
                                    amplitude=4.0, ell_range=(1.0, 8.0), n_sinks=2, seed=100,
                                    taus=(0.5, 0.9, 0.99, 1.0)),
    "bf16-3x(5x13x31)-ragged": LayerConfig("ragged-bf16", heads=3, grid=(5, 13, 31), head_dim=128, block=128,
                                           dtype="bf16", amplitude=4.0, ell_range=(1.0, 8.0), n_sinks=2, seed=101,
                                           taus=(0.9, 0.99, 1.0)),
    "bf16-1x(1x1x77)-one-block": LayerConfig("one-block", heads=1, grid=(1, 1, 77), head_dim=128, block=128,
                                             dtype="bf16", amplitude=4.0, ell_range=(1.0, 8.0), n_sinks=1,
                                             seed=102, taus=(0.99,)),
    "f32-tiny": CONFIGS["tiny"],
    # the LoSA page's block shape: 128-row query blocks, 32-key blocks
    "bf16-C32-2x(4x16x16)": LayerConfig("small-bf16-c32", heads=2, grid=(4, 16, 16), head_dim=128, block=128,
                                        block_k=32, dtype="bf16", amplitude=4.0, ell_range=(1.0, 8.0), n_sinks=2,
                                        seed=103, taus=(0.5, 0.9, 0.99, 1.0)),
    # 2015 tokens padded to 2048: the last 32-key block is all padding
    "bf16-C32-3x(5x13x31)-ragged": LayerConfig("ragged-bf16-c32", heads=3, grid=(5, 13, 31), head_dim=128,
                                               block=128, block_k=32, dtype="bf16", amplitude=4.0,
                                               ell_range=(1.0, 8.0), n_sinks=2, seed=104, taus=(0.9, 0.99, 1.0)),
}


def _pipeline(cfg, items, oracle, layer=None):
    layer = make_layer(cfg) if layer is None else layer
    q, k, v = device_inputs(layer)
    scale = scale_of(cfg)
    buf = LayerBuffers.for_config(cfg)
    buf.profile(q, k, v, scale)
    assert L.losa_get_device_error() == 0
    qf, kf, vf = layer.all_f32("q"), layer.all_f32("k"), layer.all_f32("v")
    if items is None:
        items = np.arange(buf.rows, dtype=np.int32)
    R, C, N = cfg.block, cfg.kblock, cfg.n_tokens

    # dense forward
    od, ld = oracle.dense(qf, kf, vf, N, R, scale, items)
    go, valid = item_rows(cfg, items, buf.o.float().cpu().numpy())
    gl, _ = item_rows(cfg, items, buf.lse.cpu().numpy())
    check_output(go[valid], od[valid], f"{cfg.name} dense O")
    check_lse(gl[valid], ld[valid], f"{cfg.name} dense lse")

    # block masses
    gm_all = buf.mass.cpu().numpy().reshape(buf.rows, buf.nk)
    om = oracle.mass(qf, kf, N, R, C, scale, items)
    check_mass(gm_all[items], om, f"{cfg.name}")
    np.testing.assert_allclose(gm_all.sum(axis=1), 1.0, atol=1e-3)

    for tau in cfg.taus:
        buf.select(tau)
        assert L.losa_get_device_error() == 0
        gi, gk, gord = buf.csr_host()
        # every row, bit-exact against the oracle fed the GPU's fp32 masses
        compare_select(gi, gk, gord, gm_all, tau, oracle)
        # the retained set of every compared row keeps >= tau of its exact (oracle) mass, up to fp32 rounding
        for t, it in enumerate(items):
            kept = om[t, gk[gi[it]:gi[it + 1]]].sum()
            assert kept >= tau * om[t].sum() - 2e-4, (tau, it, kept)
        o2 = torch.empty_like(buf.o)
        l2 = torch.empty_like(buf.lse)
        buf.sparse(q, k, v, scale, out=o2, lse=l2)
        assert L.losa_get_device_error() == 0
        os_, ls_ = oracle.sparse(qf, kf, vf, N, R, C, scale, gi, gk, items)
        go2, _ = item_rows(cfg, items, o2.float().cpu().numpy())
        gl2, _ = item_rows(cfg, items, l2.cpu().numpy())
        check_output(go2[valid], os_[valid], f"{cfg.name} sparse O tau={tau}")
        check_lse(gl2[valid], ls_[valid], f"{cfg.name} sparse lse tau={tau}")
    return buf, layer


@pytest.mark.parametrize("name", list(SMALL))
def test_small_full_comparison(name, oracle_mod):
    _pipeline(SMALL[name], None, oracle_mod)


@pytest.mark.parametrize("workload,block_k", [("wan1.3b480", 128), ("wan14b720", 128), ("hunyuan720", 128),
                                              ("wan1.3b480", 32), ("hunyuan720", 32)])
def test_full_size_sampled(workload, block_k, oracle_mod):
    import dataclasses
    cfg = dataclasses.replace(CONFIGS[workload], block_k=block_k)
    layer = make_layer(cfg)
    # 64 seeded items, including the tail block of head 0 and the query blocks holding head 0's sink tokens
    sink_items = [int(t) // cfg.block for t in layer.sinks[0]]
    items = sample_items(cfg, 64, seed=cfg.seed, must_include=sink_items)
    _pipeline(cfg, items, oracle_mod, layer=layer)


def test_sparse_with_every_block_equals_dense():
    cfg = SMALL["bf16-3x(5x13x31)-ragged"]
    layer = make_layer(cfg)
    q, k, v = device_inputs(layer)
    buf = LayerBuffers.for_config(cfg)
    scale = scale_of(cfg)
    buf.profile(q, k, v, scale, with_mass=False)
    nb = buf.nk
    buf.indptr.copy_(torch.arange(0, buf.rows * nb + 1, nb, dtype=torch.int32))
    buf.kv_idx.copy_(torch.arange(nb, dtype=torch.int32).repeat(buf.rows))
    o2 = torch.empty_like(buf.o)
    buf.sparse(q, k, v, scale, out=o2, order=False)
    assert L.losa_get_device_error() == 0
    # Two different kernels (256-key tiles vs 128-key tiles, different running-max references) each round O to bf16;
    # they must agree within the output tolerance both meet against the fp64 oracle.
    n = cfg.n_tokens
    a = buf.o[:, :n].float().cpu().numpy().reshape(-1, cfg.head_dim)
    b = o2[:, :n].float().cpu().numpy().reshape(-1, cfg.head_dim)
    check_output(b, a.astype(np.float64), "full-list sparse vs dense")


def test_sparse_random_lists_and_orders(oracle_mod):
    """Unsorted lists of every length 1..nk, any work order (or none)."""
    cfg = SMALL["bf16-3x(5x13x31)-ragged"]
    layer = make_layer(cfg)
    q, k, v = device_inputs(layer)
    scale = scale_of(cfg)
    buf = LayerBuffers.for_config(cfg)
    rng = np.random.default_rng(7)
    nb = buf.nk
    lists = [rng.permutation(nb)[: 1 + (r % nb)].astype(np.int32) for r in range(buf.rows)]
    indptr = np.zeros(buf.rows + 1, np.int32)
    indptr[1:] = np.cumsum([len(x) for x in lists])
    kv = np.concatenate(lists)
    buf.indptr.copy_(torch.from_numpy(indptr))
    buf.kv_idx[: len(kv)].copy_(torch.from_numpy(kv))
    qf, kf, vf = layer.all_f32("q"), layer.all_f32("k"), layer.all_f32("v")
    ref_o, ref_l = oracle_mod.sparse(qf, kf, vf, cfg.n_tokens, cfg.block, cfg.block, scale, indptr, kv)
    items = np.arange(buf.rows)
    for order in (None, rng.permutation(buf.rows).astype(np.int32)):
        o2 = torch.zeros_like(buf.o)
        l2 = torch.zeros_like(buf.lse)
        if order is not None:
            buf.order.copy_(torch.from_numpy(order))
        buf.sparse(q, k, v, scale, out=o2, lse=l2, order=order is not None)
        assert L.losa_get_device_error() == 0
        go, valid = item_rows(cfg, items, o2.float().cpu().numpy())
        gl, _ = item_rows(cfg, items, l2.cpu().numpy())
        check_output(go[valid], ref_o[valid], "random lists")
        check_lse(gl[valid], ref_l[valid], "random lists")


def test_sparse_reports_bad_csr():
    """Out-of-range block indices and empty rows are reported through the device error word; the kernel
    clamps indices before addressing, so nothing outside the inputs is read."""
    cfg = SMALL["bf16-2x(4x16x16)"]
    layer = make_layer(cfg)
    q, k, v = device_inputs(layer)
    buf = LayerBuffers.for_config(cfg)
    nb = buf.nk
    counts = np.ones(buf.rows, np.int32)
    counts[3] = 0
    indptr = np.zeros(buf.rows + 1, np.int32)
    indptr[1:] = np.cumsum(counts)
    kv = np.zeros(int(indptr[-1]), np.int32)
    kv[5] = nb + 3
    buf.indptr.copy_(torch.from_numpy(indptr))
    buf.kv_idx[: len(kv)].copy_(torch.from_numpy(kv))
    buf.sparse(q, k, v, scale_of(cfg), order=False)
    assert L.losa_get_device_error() == -5
    assert L.losa_get_device_error() == 0


@pytest.mark.parametrize("name", ["bf16-2x(4x16x16)", "f32-tiny"])
def test_sparse_reports_bad_work_order(name):
    """A work-order entry outside [0, H*nq) is reported through the device error word and its slot is skipped: the
    entry is checked before it is used, so nothing outside the inputs is read or written. Every other item is still
    computed."""
    cfg = SMALL[name]
    layer = make_layer(cfg)
    q, k, v = device_inputs(layer)
    buf = LayerBuffers.for_config(cfg)
    scale = scale_of(cfg)
    buf.profile(q, k, v, scale)
    buf.select(0.99)
    ref = torch.empty_like(buf.o)
    buf.sparse(q, k, v, scale, out=ref)
    assert L.losa_get_device_error() == 0
    good = buf.order.clone()
    bad = good.clone()
    bad[1] = buf.rows + 5
    bad[2] = -1
    buf.order.copy_(bad)
    got = torch.zeros_like(buf.o)
    buf.sparse(q, k, v, scale, out=got)
    assert L.losa_get_device_error() == -5
    assert L.losa_get_device_error() == 0
    skipped = {int(good[1]), int(good[2])}
    n = cfg.n_tokens
    for it in range(buf.rows):
        if it in skipped:
            continue
        h, i = divmod(it, buf.nq)
        r0, r1 = i * cfg.block, min((i + 1) * cfg.block, n)
        assert torch.equal(got[h, r0:r1], ref[h, r0:r1]), it
    buf.order.copy_(good)


def test_bounded_wait_selftest():
    """A wait on a barrier nothing completes runs out after its limit and reports LOSA_ERR_TIMEOUT; the
    context stays usable."""
    L.losa_selftest_wait_timeout(2_000_000)
    assert L.losa_get_device_error() == -6
    x = torch.ones(4, device="cuda")
    assert float((x * 2).sum().item()) == 8.0
    assert L.losa_get_device_error() == 0
