"""The benchmark's work model and roofline arithmetic, checked against invariants rather than restated formulas:
with every block kept and no padding the sparse call does exactly the dense call's tensor work (at either key block
size); the profile adds one more Q K^T pass over the same pairs; the selection moves the mass matrix plus its CSR
output; a roofline fraction is achieved over peak. Runs without a GPU."""
import dataclasses
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from losa_synth import CONFIGS  # noqa: E402


@pytest.mark.parametrize("block_k", [0, 32])
def test_full_lists_equal_dense_work(block_k):
    cfg = dataclasses.replace(CONFIGS["wan1.3b480"], block_k=block_k)
    H, Np, d = cfg.heads, cfg.n_padded, cfg.head_dim
    nnz = H * (Np // cfg.block) * (Np // cfg.kblock)  # every (item, key block)
    w = bench.work_model(cfg, nnz)
    # the dense-equivalent figure counts the N real tokens; with N = Np the two must agree exactly
    assert w["sparse_flop"] == pytest.approx(w["dense_equiv_flop"] * (Np / cfg.n_tokens) ** 2, rel=1e-12)
    assert w["sparse_flop"] == pytest.approx(4.0 * H * Np * Np * d, rel=1e-12)


def test_profile_is_one_forward_pass():
    cfg = CONFIGS["hunyuan720"]
    w = bench.work_model(cfg, 0)
    # forward: Q K^T and P V (2 flops per multiply-add each); the masses reuse the forward's weights
    assert w["profile_flop"] == pytest.approx(w["dense_equiv_flop"], rel=1e-12)
    assert w["profile_exp"] == pytest.approx(1.0 * cfg.heads * cfg.n_tokens ** 2, rel=1e-12)


def test_select_bytes_are_mass_plus_csr():
    cfg = CONFIGS["hunyuan720"]
    rows = cfg.heads * cfg.n_blocks
    for nnz in (0, 108056):
        w = bench.work_model(cfg, nnz)
        mass = 4 * rows * cfg.n_kblocks                 # fp32 mass matrix read once
        csr = 4 * (nnz + rows + 1) + 4 * rows           # kv_block_idx, indptr, order
        assert w["select_bytes"] == mass + csr


def test_roofline_fraction_is_achieved_over_peak():
    pk = {"bf16_tflops": 1618.0, "bf16_tflops_sustained": 1377.3, "hbm_gbs": 6551.4, "sm_max_mhz": 1965.0,
          "source": "test"}
    r = bench.roofline("k", "tensor", 2.0e12, 2.0e-3, pk, "TFLOP/s")  # 2e12 flop in 2 ms = 1000 TFLOP/s
    assert r["achieved"] == pytest.approx(1000.0)
    assert r["frac"] == pytest.approx(1000.0 / 1377.3, abs=1e-4)
    assert r["frac_of_burst"] == pytest.approx(1000.0 / 1618.0, abs=1e-4)
    assert r["frac_of_sustained"] == pytest.approx(r["frac"])
    r = bench.roofline("k", "tensor", 2.0e12, 2.0e-3, pk, "TFLOP/s", peak_kind="burst")
    assert r["frac"] == pytest.approx(1000.0 / 1618.0, abs=1e-4) and r["peak"] == 1618.0
    r = bench.roofline("k", "hbm", 6.5514e9, 1.0e-3, pk, "GB/s")  # 6.55 GB in 1 ms = the measured peak
    assert r["frac"] == pytest.approx(1.0, abs=1e-4)


def test_clock_summary_reads_nvidia_smi_samples():
    """The clock record of a timed region: median SM clock over loaded samples (idle ones at the start or end are
    left out), the maximum clock, and every throttle reason that was active in any sample; malformed lines are
    skipped."""
    cs = bench.ClockSampler(0)
    cs.lines = [
        "0, 345, 1965, 120.5, 0x0000000000000001, Not Active, Not Active, Not Active, Not Active",  # idle
        "0, 1620, 1965, 998.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1635, 1965, 1001.2, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1650, 1965, 990.7, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "[N/A], garbage",
        "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    s = cs.summary()
    assert s == {"sm_mhz": 1635.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 4}
    cs.lines.append("0, 1500, 1965, 900.0, 0x0000000000000040, Not Active, Active, Not Active, Not Active")
    assert bench.ClockSampler.summary(cs)["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    empty = bench.ClockSampler(0)
    assert empty.summary() == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


def test_traffic_counters_only_for_the_captured_kernels(monkeypatch):
    """roofline.traffic comes from the committed counter summary only while the kernel sources hash to the value
    recorded with it, and only for the workload it was captured on."""
    import json
    with open(os.path.join(ROOT, "profiles", "traffic_hunyuan720.json")) as f:
        rec = json.load(f)
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: rec["source_hash"])
    assert bench.measured_traffic(rec["workload"])["sparse_attn"] == rec["sparse_attn"]
    assert bench.measured_traffic("some-other-layer") == {}
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.measured_traffic(rec["workload"]) == {}


def test_peaks_fall_back_per_missing_entry(tmp_path):
    """The roofline denominators come from the measurement file; an entry it lacks falls back alone, and the source
    names it; without the file every entry is the earlier measurement."""
    import json
    full = {"hbm_gbs": 6551.4, "bf16_tflops": 1618.2, "bf16_tflops_sustained": 1377.3, "sm_max_mhz": 1965.0}
    f = tmp_path / "peaks.json"
    f.write_text(json.dumps(full))
    p = bench.peaks(str(f))
    assert p["source"] == "measured" and p["bf16_tflops_sustained"] == 1377.3 and p["hbm_gbs"] == 6551.4
    f.write_text(json.dumps({k: v for k, v in full.items() if k != "bf16_tflops_sustained"}))
    p = bench.peaks(str(f))
    assert p["bf16_tflops_sustained"] == bench.FALLBACK_PEAKS["bf16_tflops_sustained"]
    assert p["hbm_gbs"] == 6551.4 and "fallback for bf16_tflops_sustained" in p["source"]
    p = bench.peaks(str(tmp_path / "absent.json"))
    assert p["source"] == "fallback" and p["bf16_tflops"] == bench.FALLBACK_PEAKS["bf16_tflops"]


def test_l2_note_matches_the_workload_size():
    assert bench.bench_config(CONFIGS["hunyuan720"], 0.99, 1)["l2"].startswith("inputs larger than L2")
    assert bench.bench_config(CONFIGS["tiny"], 0.99, 1)["l2"].startswith("inputs fit in L2")
