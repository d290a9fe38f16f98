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


def _stacked(base, seeds, heads_each):
    """Layers generated with their own seeds, stacked along the head axis (branch-major), with the stacked config."""
    import dataclasses
    from losa_synth import Layer
    parts = [make_layer(LayerConfig(f"branch{s}", seed=s, **base)) for s in seeds]
    cfg = dataclasses.replace(parts[0].cfg, name="stacked", heads=heads_each * len(seeds))
    arrays = {n: np.concatenate([getattr(p, n) for p in parts]) for n in ("q", "k", "v")}
    return Layer(cfg, arrays["q"], arrays["k"], arrays["v"], np.concatenate([p.lengthscales for p in parts]),
                 np.concatenate([p.sinks for p in parts])), parts


def test_two_branches_match_the_oracle(oracle_mod):
    """Each stacked branch's masses, lists and sparse output against the oracle on that branch's own inputs (every
    item): separate patterns per guidance branch, computed in one call."""
    require_gpu()
    from tests.gpu_util import check_mass, check_output, compare_select, item_rows, check_lse
    base = dict(heads=2, grid=(3, 16, 21), head_dim=128, block=128, dtype="bf16", amplitude=4.0,
                ell_range=(1.0, 8.0), n_sinks=2)
    layer, parts = _stacked(base, (41, 42), 2)
    cfg = layer.cfg
    scale = 1.0 / math.sqrt(128)
    q, k, v = (host_tokens_to_device(getattr(layer, n), "bf16") for n in ("q", "k", "v"))
    buf = LayerBuffers.for_config(cfg)
    buf.profile(q, k, v, scale)
    buf.select(0.99)
    o2, l2 = torch.empty_like(buf.o), torch.empty_like(buf.lse)
    buf.sparse(q, k, v, scale, out=o2, lse=l2)
    assert L.losa_get_device_error() == 0
    gi, gk, gord = buf.csr_host()
    gm = buf.mass.cpu().numpy().reshape(buf.rows, buf.nk)
    compare_select(gi, gk, gord, gm, 0.99, oracle_mod)
    N, R = cfg.n_tokens, cfg.block
    per = buf.rows // 2
    for b, part in enumerate(parts):
        qf, kf, vf = part.all_f32("q"), part.all_f32("k"), part.all_f32("v")
        check_mass(gm[b * per:(b + 1) * per], oracle_mod.mass(qf, kf, N, R, R, scale), f"branch {b}")
        # this branch's lists, re-based to its own rows
        bi = gi[b * per:(b + 1) * per + 1] - gi[b * per]
        bk = gk[gi[b * per]:gi[(b + 1) * per]]
        ref_o, ref_l = oracle_mod.sparse(qf, kf, vf, N, R, R, scale, bi, bk)
        got, valid = item_rows(part.cfg, np.arange(per), o2[2 * b:2 * b + 2].float().cpu().numpy())
        gl, _ = item_rows(part.cfg, np.arange(per), l2[2 * b:2 * b + 2].cpu().numpy())
        check_output(got[valid], ref_o[valid], f"branch {b} sparse O")
        check_lse(gl[valid], ref_l[valid], f"branch {b} sparse lse")


def test_two_branches_at_hunyuan_size(oracle_mod):
    """Two guidance branches of the HunyuanVideo-720p-shaped layer in one call (48 heads: 44592 items x 929 blocks):
    the whole hot path, with every row's selection bit-exact and 64 sampled items per branch against the oracle."""
    require_gpu()
    import dataclasses
    from losa_synth import CONFIGS, Layer, sample_items
    from tests.test_gpu_attention import _pipeline
    h = CONFIGS["hunyuan720"]
    parts = [make_layer(dataclasses.replace(h, seed=s)) for s in (3, 13)]
    cfg = dataclasses.replace(h, name="hunyuan720-two-branches", heads=2 * h.heads)
    layer = Layer(cfg, *(np.concatenate([getattr(p, n) for p in parts]) for n in ("q", "k", "v")),
                  np.concatenate([p.lengthscales for p in parts]), np.concatenate([p.sinks for p in parts]))
    per = h.heads * h.n_blocks
    items = np.concatenate([sample_items(h, 32, seed=20), per + sample_items(h, 32, seed=21)]).astype(np.int32)
    buf, _ = _pipeline(cfg, items, oracle_mod, layer=layer)
    assert buf.rows == 2 * per
