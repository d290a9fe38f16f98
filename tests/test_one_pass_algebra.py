"""The one-pass form of the block masses (LoSA page, Motivation Summary: M(i, j) is the sum of the softmax weights A
over query block i and key block j), checked on the CPU against the oracle's masses.

The dense kernel never has a row's final max or sum while it walks the keys. Per row it keeps a reference max m that
moves only when a 256-key tile's max exceeds it by more than 2^8 (in base-2 units of the scaled logit), forms every
weight as 2^(s c - m c) with c = scale * log2(e), and keeps the exact sum b(j) of each key block's weights, brought to
an anchor max m0 (multiplied by 2^((m - m0) c)). When m moves more than 2^60 above m0, the sums stored so far are
rescaled and m0 moves to m. Once every row of a query block has its final m and l, M(i, j) = sum over rows of
b(j) * 2^((m0 - m) c) / l, divided by the block's real rows.

This file runs that procedure in NumPy, vectorised over rows, in fp64 (the algebra, which must give the masses up to
rounding) and in fp32 (the kernel's arithmetic, which must stay inside the 1e-4 relative bound), on a ragged layer
and on one whose later keys raise every row's max far past the anchor span. A variant that forgets the rescale on
re-anchoring must fail, so the re-anchoring case is exercised, not skipped."""
import dataclasses

import numpy as np
import pytest

from losa_synth import LayerConfig, make_layer

TILE = 256          # keys per forward tile of the dense kernel
LAZY_SPAN = 8.0     # the reference max moves only past 2^8 above itself
ANCHOR_SPAN = 60.0  # stored sums stay within 2^60 of their anchor

CFG = LayerConfig("one-pass-algebra", heads=2, grid=(5, 13, 31), head_dim=128, block=128, dtype="bf16",
                  amplitude=4.0, ell_range=(1.0, 8.0), n_sinks=2, seed=303)
CFG_C32 = dataclasses.replace(CFG, name="one-pass-algebra-c32", block_k=32, seed=304)


def one_pass_masses(q, k, n_tokens, block_q, block_k, scale, dtype, rescale_on_reanchor=True):
    """Row-normalised masses [H * nq][nk] by the one-pass procedure; also returns how many (row, tile) re-anchors
    happened."""
    H, Np, _ = q.shape
    nq, nk = Np // block_q, Np // block_k
    c = dtype(scale * np.log2(np.e))
    out = np.zeros((H * nq, nk), dtype=np.float64)
    reanchors = 0
    n_tiles = -(-n_tokens // TILE)
    for h in range(H):
        s_all = (q[h].astype(np.float64) @ k[h, :n_tokens].astype(np.float64).T).astype(dtype)  # [Np][n_tokens]
        rows = Np
        m = np.zeros(rows, dtype)
        m0 = np.zeros(rows, dtype)
        fac = np.ones(rows, dtype)
        l_run = np.zeros(rows, dtype)
        stored = np.zeros((rows, nk), dtype)
        for t in range(n_tiles):
            k0, k1 = t * TILE, min((t + 1) * TILE, n_tokens)
            s = s_all[:, k0:k1]
            tmax = s.max(axis=1)
            need = np.full(rows, True) if t == 0 else (tmax - m) * c > dtype(LAZY_SPAN)
            alpha = np.where(need & (t > 0), np.exp2(np.minimum((m - tmax) * c, 0)), dtype(1.0)).astype(dtype)
            m = np.where(need, tmax, m).astype(dtype)
            p = np.exp2(s * c - (m * c)[:, None]).astype(dtype)
            l_run = (l_run * alpha + p.sum(axis=1, dtype=dtype)).astype(dtype)
            if t == 0:
                m0 = m.copy()
                fac = np.ones(rows, dtype)
            else:
                far = need & ((m - m0) * c > dtype(ANCHOR_SPAN))
                near = need & ~far
                if far.any():
                    reanchors += int(far.sum())
                    if rescale_on_reanchor:
                        r = np.exp2((m0[far] - m[far]) * c).astype(dtype)
                        stored[far] = (stored[far] * r[:, None]).astype(dtype)
                    m0 = np.where(far, m, m0).astype(dtype)
                    fac = np.where(far, dtype(1.0), fac).astype(dtype)
                fac = np.where(near, np.exp2((m - m0) * c), fac).astype(dtype)
            for j in range(k0 // block_k, -(-k1 // block_k)):
                a, b = j * block_k - k0, min((j + 1) * block_k, k1) - k0
                stored[:, j] = (p[:, a:b].sum(axis=1, dtype=dtype) * fac).astype(dtype)
        w = (np.exp2((m0 - m) * c) / l_run).astype(dtype)  # per-row factor, known only at the end
        for i in range(nq):
            r0, r1 = i * block_q, min((i + 1) * block_q, n_tokens)
            if r1 <= r0:
                continue
            rows_i = slice(r0, r1)
            out[h * nq + i] = (stored[rows_i].astype(np.float64) * w[rows_i, None]).sum(axis=0) / (r1 - r0)
    return out, reanchors


def _scale_keys(layer, t0, t1, log2_factor):
    """The keys of tokens t0 .. t1 - 1 of every head times 2^log2_factor, exactly (the bf16 exponent field)."""
    k = layer.k.astype(np.int32)
    seg = k[:, t0:t1]
    k[:, t0:t1] = np.where((seg & 0x7FFF) != 0, seg + (log2_factor << 7), seg)
    return dataclasses.replace(layer, k=k.astype(np.uint16))


def _real_items(cfg):
    return np.array([h * cfg.n_blocks + i for h in range(cfg.heads) for i in range(cfg.n_blocks)
                     if i * cfg.block < cfg.n_tokens], dtype=np.int32)


def _case(cfg, oracle, far):
    layer = make_layer(cfg)
    if far:  # a middle tile 4x, the last tile 16x: rows move past the anchor span
        layer = _scale_keys(layer, 512, 768, 2)
        layer = _scale_keys(layer, (cfg.n_tokens - 1) // TILE * TILE, cfg.n_tokens, 4)
    q, k = layer.all_f32("q"), layer.all_f32("k")
    scale = 1.0 / np.sqrt(cfg.head_dim)
    items = _real_items(cfg)
    ref = oracle.mass(q, k, cfg.n_tokens, cfg.block, cfg.kblock, scale, items)
    return q, k, scale, items, ref


@pytest.mark.parametrize("cfg", [CFG, CFG_C32], ids=["C128", "C32"])
@pytest.mark.parametrize("far", [False, True], ids=["ragged", "max-grows-far"])
def test_one_pass_masses_in_fp64_equal_the_masses(cfg, far, oracle_mod):
    q, k, scale, items, ref = _case(cfg, oracle_mod, far)
    got, reanchors = one_pass_masses(q, k, cfg.n_tokens, cfg.block, cfg.kblock, scale, np.float64)
    if far:
        assert reanchors > 0
    np.testing.assert_allclose(got[items], ref, rtol=1e-9, atol=1e-300)


@pytest.mark.parametrize("cfg", [CFG, CFG_C32], ids=["C128", "C32"])
def test_one_pass_masses_in_fp32_stay_inside_the_bound(cfg, oracle_mod):
    q, k, scale, items, ref = _case(cfg, oracle_mod, False)
    got, _ = one_pass_masses(q, k, cfg.n_tokens, cfg.block, cfg.kblock, scale, np.float32)
    err = np.abs(got[items] - ref)
    assert (err <= 1e-4 * ref + 1e-30).all(), f"max relative error {float((err / np.maximum(ref, 1e-300)).max())}"


def test_dropping_the_rescale_on_reanchoring_is_caught(oracle_mod):
    q, k, scale, items, ref = _case(CFG, oracle_mod, True)
    got, reanchors = one_pass_masses(q, k, CFG.n_tokens, CFG.block, CFG.kblock, scale, np.float64,
                                     rescale_on_reanchor=False)
    assert reanchors > 0
    assert not np.allclose(got[items], ref, rtol=1e-4, atol=0)
