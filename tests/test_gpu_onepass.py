"""The block masses taken in the forward pass (losa_dense_profile_ws; LoSA page, Motivation Summary, M(i, j) as the
sum of A over a query block and a key block) against the two-pass call and the oracle: on small layers at C = 128
and C = 32, on a layer whose later keys raise each row's max far above its first tile's (the row's anchor moves and
its stored sums are rescaled), and the call's refusals."""
import dataclasses

import numpy as np
import pytest
import torch

import free_block_sparse_losa_b200 as L
from free_block_sparse_losa_b200.harness import LayerBuffers
from losa_synth import make_layer
from tests.gpu_util import check_lse, check_mass, check_output, device_inputs, item_rows, require_gpu, scale_of
from tests.test_gpu_attention import SMALL

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _check_mass_rtol(gpu_rows, ref_rows, rtol, what):
    err = np.abs(gpu_rows.astype(np.float64) - ref_rows)
    bad = err > rtol * ref_rows + 1e-30
    assert not bad.any(), f"{what}: {int(bad.sum())} entries beyond {rtol} relative, first at {np.argwhere(bad)[0]}"


def _both_ways(cfg, layer, oracle, mass_rtol=None, lse_rtol=0.0):
    """Runs the two-pass and the one-pass profile on the same inputs; checks both calls' masses, and the one-pass
    call's O and lse, against the oracle, and O against the two-pass call bit for bit (the forward is the same
    code). mass_rtol replaces the 1e-4 mass tolerance, and lse_rtol widens the lse tolerance by that fraction of
    |lse|, where the inputs make fp32 logits too coarse for the defaults."""
    q, k, v = device_inputs(layer)
    buf = LayerBuffers.for_config(cfg)
    scale = scale_of(cfg)
    buf.profile(q, k, v, scale, one_pass=False)
    m2, o2, l2 = buf.mass.cpu().numpy().copy(), buf.o.clone(), buf.lse.clone()
    buf.profile(q, k, v, scale)
    torch.cuda.synchronize()
    assert L.losa_get_device_error() == 0
    assert torch.equal(buf.o.view(torch.int16), o2.view(torch.int16))
    # lse = m + ln l: with C = 32 the one-pass call sums each row's weights in four quarter accumulators, so l may
    # differ from the two-pass call's by a few fp32 ulps, and lse by a few ulps of its own size (about 900 on the
    # scaled-key layer, where one ulp is 6e-5)
    assert bool(((buf.lse - l2).abs() <= 1e-5 + 4 * 2.0 ** -23 * l2.abs()).all())
    items = np.arange(buf.rows, dtype=np.int32)
    qf, kf, vf = layer.all_f32("q"), layer.all_f32("k"), layer.all_f32("v")
    ref = oracle.mass(qf, kf, cfg.n_tokens, cfg.block, cfg.kblock, scale, items)
    m1 = buf.mass.cpu().numpy().reshape(buf.rows, buf.nk)
    if mass_rtol is None:
        check_mass(m1, ref, f"{cfg.name} one-pass")
        check_mass(m2.reshape(buf.rows, buf.nk), ref, f"{cfg.name} two-pass")
    else:
        _check_mass_rtol(m1, ref, mass_rtol, f"{cfg.name} one-pass")
        _check_mass_rtol(m2.reshape(buf.rows, buf.nk), ref, mass_rtol, f"{cfg.name} two-pass")
    np.testing.assert_allclose(m1.sum(axis=1), 1.0, atol=1e-3)
    od, ld = oracle.dense(qf, kf, vf, cfg.n_tokens, cfg.block, scale, items)
    go, valid = item_rows(cfg, items, buf.o.float().cpu().numpy())
    gl, _ = item_rows(cfg, items, buf.lse.cpu().numpy())
    check_output(go[valid], od[valid], f"{cfg.name} dense O")
    if lse_rtol:
        err = np.abs(gl[valid].astype(np.float64) - ld[valid])
        assert (err <= 1e-3 + lse_rtol * np.abs(ld[valid])).all(), f"{cfg.name} dense lse: max err {err.max():.3e}"
    else:
        check_lse(gl[valid], ld[valid], f"{cfg.name} dense lse")


@pytest.mark.parametrize("name", ["bf16-3x(5x13x31)-ragged", "bf16-C32-3x(5x13x31)-ragged",
                                  "bf16-1x(1x1x77)-one-block"])
def test_one_pass_masses(name, oracle_mod):
    cfg = SMALL[name]
    _both_ways(cfg, make_layer(cfg), oracle_mod)


def _scale_keys(layer, t0, t1, log2_factor):
    """The keys of tokens t0 .. t1 - 1 of every head times 2^log2_factor, exactly (the bf16 exponent field)."""
    k = layer.k.astype(np.int32)
    seg = k[:, t0:t1]
    k[:, t0:t1] = np.where((seg & 0x7FFF) != 0, seg + (log2_factor << 7), seg)
    return dataclasses.replace(layer, k=k.astype(np.uint16))


@pytest.mark.parametrize("name", ["bf16-3x(5x13x31)-ragged", "bf16-C32-3x(5x13x31)-ragged"])
def test_one_pass_masses_when_the_row_max_grows_far(name, oracle_mod):
    cfg = SMALL[name]
    layer = make_layer(cfg)
    n = cfg.n_tokens
    # a middle tile 4x (the reference max moves within the anchor span), the last tile 16x (far past it). The last
    # tile's logits reach about 1000, where one fp32 ulp of the tensor core's accumulation is about 1e-4 of the
    # logit scale times log2(e): both calls then agree with the exact masses to a few 1e-5, at times just above
    # 1e-4, so this case checks the anchor logic at 5e-4 (a wrong anchor factor would be off by 2^60). For the same
    # reason lse (about 900 here) may be off by more than the usual 1e-3: the worst-case rounding bound of a
    # 128-term fp32 dot product, 128 * 2^-24 of its magnitude, is added to that tolerance.
    layer = _scale_keys(layer, 512, 768, 2)
    layer = _scale_keys(layer, (n - 1) // 256 * 256, n, 4)
    _both_ways(cfg, layer, oracle_mod, mass_rtol=5e-4, lse_rtol=128 * 2.0 ** -24)


def test_one_pass_refusals():
    cfg = SMALL["bf16-2x(4x16x16)"]
    q, k, v = device_inputs(make_layer(cfg))
    buf = LayerBuffers.for_config(cfg)
    need = L.losa_dense_profile_workspace_bytes(buf.shape)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert need == sms * buf.nk * 128 * 4
    scale = scale_of(cfg)
    st = L.losa_dense_profile_ws(buf.shape, q, k, v, scale, buf.o, buf.lse, buf.mass, buf.profile_workspace,
                                 ws_bytes=need - 1, raise_on_error=False)
    assert st == -3  # LOSA_ERR_CAPACITY
    st = L.losa_dense_profile_ws(buf.shape, q, k, v, scale, buf.o, buf.lse, buf.mass,
                                 buf.profile_workspace.data_ptr() + 4, ws_bytes=need, raise_on_error=False)
    assert st == -1  # LOSA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert L.losa_get_device_error() == 0
