"""Batches and classifier-free-guidance branches (LoSA page, Methodology Summary: patterns are kept separately for
the conditional and unconditional branches): two branches stacked as heads = 2 * H get their own patterns, and each
branch's results equal the results of running that branch alone."""
import math

import numpy as np
import pytest
import torch

import free_block_sparse_losa_b200 as L
from free_block_sparse_losa_b200.harness import LayerBuffers, host_tokens_to_device
from losa_synth import LayerConfig, make_layer
from tests.gpu_util import require_gpu

pytestmark = pytest.mark.gpu


def test_two_branches_have_independent_patterns():
    require_gpu()
    base = dict(heads=2, grid=(3, 16, 21), head_dim=128, block=128, dtype="bf16", amplitude=4.0,
                ell_range=(1.0, 8.0), n_sinks=2)
    cond = make_layer(LayerConfig("cond", seed=31, **base))
    uncond = make_layer(LayerConfig("uncond", seed=32, **base))
    scale = 1.0 / math.sqrt(128)
    both = LayerConfig("cfg-pair", seed=0, **{**base, "heads": 4})
    stacked = [np.concatenate([getattr(cond, n), getattr(uncond, n)]) for n in ("q", "k", "v")]
    q2, k2, v2 = (host_tokens_to_device(a, "bf16") for a in stacked)
    pair = LayerBuffers.for_config(both)
    pair.profile(q2, k2, v2, scale)
    pair.select(0.99)
    pair.sparse(q2, k2, v2, scale)
    pi, pk, _ = pair.csr_host()
    rows_per_branch = pair.rows // 2
    outs = []
    for li, layer in enumerate((cond, uncond)):
        q, k, v = (host_tokens_to_device(getattr(layer, n), "bf16") for n in ("q", "k", "v"))
        one = LayerBuffers.for_config(layer.cfg)
        one.profile(q, k, v, scale)
        one.select(0.99)
        one.sparse(q, k, v, scale)
        oi, ok_, _ = one.csr_host()
        lo = rows_per_branch * li
        seg = pk[pi[lo]:pi[lo + rows_per_branch]]
        assert np.array_equal(pi[lo:lo + rows_per_branch + 1] - pi[lo], oi)
        assert np.array_equal(seg, ok_)
        assert torch.equal(pair.mass[2 * li:2 * li + 2], one.mass)
        assert torch.equal(pair.o[2 * li:2 * li + 2], one.o)
        outs.append(seg)
    assert L.losa_get_device_error() == 0
    assert not (len(outs[0]) == len(outs[1]) and np.array_equal(outs[0], outs[1]))
