#!/usr/bin/env python
"""Benchmark of the LoSA hot path on B200.

One step = the whole hot path over one synthetic attention layer: losa_dense_profile (dense forward + exact block
masses), losa_select (tau = 0.99 by default) and losa_sparse_attn over the frozen lists. The default workload is the
HunyuanVideo-720p-shaped layer (24 heads, 33x45x80 token grid, N = 118800 padded to 118912, head_dim 128, bf16,
128 x 128 blocks).

Prints ONE JSON line (rank 0). `value` is the dense-equivalent throughput of losa_sparse_attn, 4*H*N^2*d / t_sparse,
summed over ranks (weak scaling: every rank runs its own layer); the per-kernel times, the profile+select time, the
block density, the roofline of each kernel and the oracle's CPU baseline are extra keys.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference] [--workload NAME]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from losa_synth import CONFIGS, make_layer, sample_items  # noqa: E402

METRIC = "sparse-attn ms/call & dense-equiv TFLOP/s at tau=0.99; profile+select ms"
KERNELS_PER_STEP = {"dense_profile": 1, "select": 5, "sparse_attn": 1}


FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}


def peaks(path=None):
    """Roofline denominators: the measured copy bandwidth and bf16 GEMM rates of this GPU model when the measurement
    file is present (any missing entry falls back to the earlier measurement, and the source says so), else the
    earlier measurement."""
    path = path or os.path.join(ROOT, "MEASURED_PEAKS.json")
    if not os.path.exists(path):
        return {**FALLBACK_PEAKS, "source": "fallback"}
    with open(path) as f:
        p = json.load(f)
    out = {k: float(p[k]) if isinstance(p.get(k), (int, float)) else v for k, v in FALLBACK_PEAKS.items()}
    missing = [k for k in FALLBACK_PEAKS if not isinstance(p.get(k), (int, float))]
    out["source"] = "measured" if not missing else "measured, fallback for " + ", ".join(missing)
    return out


L2_MB = 126.0  # B200 L2 capacity


def bench_config(cfg, tau, world):
    """The workload description both arms report (identical dicts for the same run)."""
    elem = 2 if cfg.dtype == "bf16" else 4
    qkv_mb = cfg.heads * cfg.n_padded * cfg.head_dim * elem / 1e6
    return {"workload": cfg.name, "heads": cfg.heads, "n_tokens": cfg.n_tokens, "n_padded": cfg.n_padded,
            "head_dim": cfg.head_dim, "block": cfg.block, "block_k": cfg.kblock, "tau": tau,
            "l2": ("inputs larger than L2 (3 x %.0f MB of Q/K/V per layer)" % qkv_mb if 3 * qkv_mb > L2_MB else
                   "inputs fit in L2 (3 x %.2f MB of Q/K/V), not flushed: a small check workload" % qkv_mb),
            "parallelism": f"replicas x{world} (one independent layer per GPU)"}


def work_model(cfg, nnz):
    """Algorithmic work per call. Tensor FLOPs count 2 per multiply-add; the dense-equivalent figure uses the
    real token count N, kept-block figures count whole 128 x 128 tiles."""
    H, N, Np, d, B = cfg.heads, cfg.n_tokens, cfg.n_padded, cfg.head_dim, cfg.block
    nq, nkb, C = Np // B, Np // cfg.kblock, cfg.kblock
    return {
        "dense_equiv_flop": 4.0 * H * N * N * d,
        # Q K^T + P V of the forward; the block masses come from the forward's own weights (one pass)
        "profile_flop": 4.0 * H * N * N * d,
        "profile_exp": 1.0 * H * N * N,
        "sparse_flop": 4.0 * B * C * d * nnz,         # kept blocks only (R x C each)
        "sparse_exp": float(B * C * nnz),
        "select_bytes": 4.0 * H * nq * nkb + 4.0 * (nnz + 2 * H * nq + 1),  # read M, write CSR + order
    }


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, ValueError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [s for s in sm if s > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def kernel_source_hash():
    import glob
    import hashlib
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "free_block_sparse_losa_b200", "csrc", "*"))):
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(workload_name):
    """Per-launch DRAM bytes from the committed ncu summary, only if the kernels are unchanged since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic_hunyuan720.json")
    if not os.path.exists(path):
        return {}
    with open(path) as f:
        t = json.load(f)
    if t.get("workload") != workload_name or t.get("source_hash") != kernel_source_hash():
        return {}
    return t


def roofline(name, bound, work, seconds, pk, unit, traffic=None, peak_kind="sustained"):
    if bound == "tensor":
        peak = pk["bf16_tflops_sustained"] if peak_kind == "sustained" else pk["bf16_tflops"]
        achieved = work / seconds / 1e12
    elif bound == "hbm":
        peak = pk["hbm_gbs"]
        achieved = work / seconds / 1e9
    else:  # alu (exp unit): 148 SMs x 16 ex2 per clock at the max SM clock
        peak = 148 * 16 * pk["sm_max_mhz"] * 1e6 / 1e12
        achieved = work / seconds / 1e12
    out = {"kernel": name, "bound": bound, "achieved": round(achieved, 3), "peak": peak, "unit": unit,
           "frac": round(achieved / peak, 4), "traffic": traffic, "peak_source": f"{pk['source']} {peak_kind}"
           if bound == "tensor" else pk["source"]}
    if bound == "tensor":  # both measured GEMM rates, whichever the headline fraction uses
        out["frac_of_burst"] = round(achieved / pk["bf16_tflops"], 4)
        out["frac_of_sustained"] = round(achieved / pk["bf16_tflops_sustained"], 4)
    return out


# ------------------------------------------------------------------------------------------------ CPU oracle

def oracle_inputs(layer):
    return layer.all_f32("q"), layer.all_f32("k"), layer.all_f32("v")


def oracle_threads():
    import oracle
    return oracle.num_threads()


def oracle_sample_run(cfg, qkv, tau, n_items, seed=7):
    """The oracle, as it stands, on a seeded sample of (head, query block) items of the workload: dense forward,
    masses, selection and restricted attention. Returns per-item seconds of each stage."""
    import oracle
    q, k, v = qkv
    items = sample_items(cfg, n_items, seed=seed)[:n_items]
    scale = 1.0 / math.sqrt(cfg.head_dim)
    R, C, N = cfg.block, cfg.kblock, cfg.n_tokens
    t0 = time.perf_counter()
    oracle.dense(q, k, v, N, R, scale, items)
    t1 = time.perf_counter()
    m = oracle.mass(q, k, N, R, C, scale, items)
    t2 = time.perf_counter()
    counts, idx = oracle.select(m.astype(np.float32), tau)
    t3 = time.perf_counter()
    # CSR over the sampled items only: rows outside the sample are empty
    rows = cfg.heads * cfg.n_blocks
    full_counts = np.zeros(rows, np.int32)
    full_counts[items] = counts
    indptr = np.zeros(rows + 1, np.int32)
    indptr[1:] = np.cumsum(full_counts)
    kv = np.concatenate([idx[t, :counts[t]] for t in range(len(items))]).astype(np.int32)
    t4 = time.perf_counter()
    oracle.sparse(q, k, v, N, R, C, scale, indptr, kv, items)
    t5 = time.perf_counter()
    n = len(items)
    return {"items": n, "dense_s": (t1 - t0) / n, "mass_s": (t2 - t1) / n, "select_s": (t3 - t2) / n,
            "sparse_s": (t5 - t4) / n, "density": float(counts.sum()) / (n * cfg.n_kblocks),
            "threads": oracle.num_threads()}


def cpu_line(cfg, per_item, sample_desc):
    rows = cfg.heads * cfg.n_blocks
    work = work_model(cfg, 0)
    t_sparse = per_item["sparse_s"] * rows
    return {"value": round(work["dense_equiv_flop"] / t_sparse / 1e12, 6),
            "unit": "TFLOP/s (dense-equivalent, sparse attention)", "cores": per_item["threads"], "kind": "oracle",
            "sample": sample_desc, "sparse_attn_ms_extrapolated": round(t_sparse * 1e3, 1),
            "profile_select_ms_extrapolated": round((per_item["dense_s"] + per_item["mass_s"] +
                                                     per_item["select_s"]) * rows * 1e3, 1)}


def run_reference(args, cfg):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    layer = make_layer(cfg)
    qkv = oracle_inputs(layer)
    n_items = args.ref_items or max(1, oracle_threads() // 2)
    desc = (f"{n_items} seeded (head, query-block) items of {cfg.name} per step (dense forward, masses, "
            f"selection, restricted attention), fp64 oracle, extrapolated linearly to all "
            f"{cfg.heads * cfg.n_blocks} items")
    for _ in range(args.warmup):
        oracle_sample_run(cfg, qkv, args.tau, max(1, n_items // 4), seed=99)
    runs, wall = [], []
    for s in range(args.steps):
        w0 = time.perf_counter()
        runs.append(oracle_sample_run(cfg, qkv, args.tau, n_items, seed=1000 + s))
        wall.append(time.perf_counter() - w0)
    per = {k: float(np.mean([r[k] for r in runs])) for k in ("dense_s", "mass_s", "select_s", "sparse_s",
                                                             "density")}
    per["threads"] = runs[0]["threads"]
    c = cpu_line(cfg, per, desc)
    rows = cfg.heads * cfg.n_blocks
    full_step_ms = (per["dense_s"] + per["mass_s"] + per["select_s"] + per["sparse_s"]) * rows * 1e3
    # ms_per_step is the wall time each timed step really took (one sampled step); the whole-layer figures are
    # extrapolations from the sample's per-item rate and are labelled as such.
    line = {"impl": "reference", "metric": METRIC, "value": c["value"], "unit": c["unit"], "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(float(np.mean(wall)) * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(cfg, args.tau, args.gpus),
            "step_is_sample": f"each step runs {n_items} of the {rows} items; value is the sample's rate",
            "extrapolated": {"full_layer_ms_per_step": round(full_step_ms, 1),
                             "sparse_attn_ms": c["sparse_attn_ms_extrapolated"],
                             "profile_select_ms": c["profile_select_ms_extrapolated"]},
            "cpu_baseline": {"value": c["value"], "unit": c["unit"], "cores": c["cores"], "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": c["value"], "unit": c["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------------- native path

class RankGroup:
    """One process per GPU (RANK / WORLD_SIZE / LOCAL_RANK from the launcher): barriers around the timed region and
    the max over ranks of each device-timed duration. Every rank takes the same collective steps in the same order."""

    def __init__(self, backend="nccl", timeout_s=600):
        import torch
        self.rank = int(os.environ.get("RANK", "0"))
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend
        self.dist = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            kw = {"device_id": torch.device("cuda", self.local)} if backend == "nccl" else {}
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
            self.dist = dist

    def barrier(self):
        if self.dist is not None:
            self.dist.barrier()

    def max(self, x):
        if self.dist is None:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device="cuda" if self.backend == "nccl" else "cpu")
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist is not None:
            self.dist.barrier()
            self.dist.destroy_process_group()
            self.dist = None


def whole_job_value(world, steps, flop_per_step, seconds_max):
    """Whole-job throughput in TFLOP/s: every rank runs `steps` steps of `flop_per_step` (weak scaling), the job
    takes as long as its slowest rank."""
    return world * steps * flop_per_step / seconds_max / 1e12


def run_native(args, cfg):
    import torch
    import free_block_sparse_losa_b200 as L
    from free_block_sparse_losa_b200.harness import LayerBuffers, host_tokens_to_device

    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    group = RankGroup("nccl")
    rank, world, local = group.rank, group.world, group.local
    barrier, max_over_ranks = group.barrier, group.max

    L.load()
    layer = make_layer(cfg)
    q, k, v = (host_tokens_to_device(getattr(layer, n), cfg.dtype) for n in ("q", "k", "v"))
    scale = 1.0 / math.sqrt(cfg.head_dim)
    buf = LayerBuffers.for_config(cfg)
    stream = torch.cuda.current_stream()

    def step(ev):
        ev[0].record(stream)
        buf.profile(q, k, v, scale)
        ev[1].record(stream)
        buf.select(args.tau)
        ev[2].record(stream)
        buf.sparse(q, k, v, scale)
        ev[3].record(stream)

    mk = lambda: [torch.cuda.Event(enable_timing=True) for _ in range(4)]  # noqa: E731
    for _ in range(args.warmup):
        step(mk())
    torch.cuda.synchronize()
    if L.losa_get_device_error() != 0:
        raise RuntimeError("device error during warm-up")
    nnz = int(buf.indptr[-1].item())

    evs = [mk() for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t_start.record(stream)
        for e in evs:
            step(e)
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier()
    total_ms = max_over_ranks(t_start.elapsed_time(t_end))
    prof_ms = [e[0].elapsed_time(e[1]) for e in evs]
    sel_ms = [e[1].elapsed_time(e[2]) for e in evs]
    spa_ms = [e[2].elapsed_time(e[3]) for e in evs]
    t_sparse = max_over_ranks(sum(spa_ms) / 1e3)
    t_prof = max_over_ranks(sum(prof_ms) / 1e3)
    t_sel = max_over_ranks(sum(sel_ms) / 1e3)
    per_sparse, per_prof, per_sel = t_sparse / args.steps, t_prof / args.steps, t_sel / args.steps
    status = L.losa_get_device_error()
    if status != 0:
        raise RuntimeError(f"device error in timed region: {status}")

    work = work_model(cfg, nnz)
    K = args.steps
    value = whole_job_value(world, K, work["dense_equiv_flop"], t_sparse)

    # end to end through the C ABI with host buffers: pinned Q/K/V -> device, sparse attention, O -> pinned host
    e2e = None
    if not args.no_e2e:
        # Two device buffer sets: step s uploads into set s % 2 and computes into its O on the main stream while the
        # O of step s - 1 goes back to the host on a second stream (the host link is full duplex). Step s's call
        # waits until the read-back of step s - 2 has left the O it overwrites.
        hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
        ho = [torch.empty(buf.o.shape, dtype=buf.o.dtype, pin_memory=True) for _ in range(2)]
        dqkv = [tuple(torch.empty_like(x) for x in (q, k, v)) for _ in range(2)]
        do = [torch.empty_like(buf.o) for _ in range(2)]
        d2h_stream = torch.cuda.Stream()
        computed = [torch.cuda.Event() for _ in range(2)]
        read_back = [torch.cuda.Event() for _ in range(2)]
        n_e2e = [0]

        def e2e_step():
            s = n_e2e[0] % 2
            dq, dk, dv = dqkv[s]
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            if n_e2e[0] >= 2:
                stream.wait_event(read_back[s])
            buf.sparse(dq, dk, dv, scale, out=do[s])
            computed[s].record(stream)
            d2h_stream.wait_event(computed[s])
            with torch.cuda.stream(d2h_stream):
                ho[s].copy_(do[s], non_blocking=True)
            read_back[s].record(d2h_stream)
            n_e2e[0] += 1

        def e2e_join():
            stream.wait_stream(d2h_stream)

        for _ in range(max(1, args.warmup)):
            e2e_step()
        e2e_join()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        e0.record(stream)
        for _ in range(K):
            e2e_step()
        e2e_join()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        t_e2e = max_over_ranks(e0.elapsed_time(e1) / 1e3)
        if L.losa_get_device_error() != 0:
            raise RuntimeError("device error in the end-to-end loop")
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
        d2h = ho[0].numel() * ho[0].element_size()
        e2e = {"value": round(whole_job_value(world, K, work["dense_equiv_flop"], t_e2e), 3),
               "unit": "TFLOP/s (dense-equivalent, sparse attention)",
               "includes": "pinned-host Q/K/V -> device, the sparse call, O -> pinned host, every step",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_call": round(t_e2e / K * 1e3, 3)}

    # Outside the timed region: the sparse call's steady state when sparse calls follow each other (every denoising
    # step after construction), here with the step's lists, and the long-list regime (tau = 1: every list holds every
    # block, so per-item overheads vanish), each timed with CUDA events and its own clock record.
    def sparse_series(reps):
        for _ in range(2):
            buf.sparse(q, k, v, scale)
        torch.cuda.synchronize()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
        with ClockSampler(local) as ck:
            ev[0].record(stream)
            for _ in range(reps):
                buf.sparse(q, k, v, scale)
            ev[1].record(stream)
            torch.cuda.synchronize()
        if L.losa_get_device_error() != 0:
            raise RuntimeError("device error in the sparse series")
        return ev[0].elapsed_time(ev[1]) / reps / 1e3, ck.summary()

    extras = {}
    if not args.no_extras:
        t_ss, ck_ss = sparse_series(max(K, 20))
        extras["sparse_attn_steady"] = {"ms": round(t_ss * 1e3, 4), "calls": max(K, 20), "clocks": ck_ss}
        buf.select(1.0)
        nnz_full = int(buf.indptr[-1].item())
        t_full, ck_full = sparse_series(3)
        extras["sparse_attn_tau1"] = {"ms": round(t_full * 1e3, 3), "calls": 3, "nnz_blocks": nnz_full,
                                      "clocks": ck_full}
        buf.select(args.tau)
        torch.cuda.synchronize()

    # Outside the timed region: block density at each tau, and the fixed-count top-k ablation at matched mean
    # coverage (the LoSA page's "retained mass vs. a fixed sparsity ratio"), both on this step's exact masses.
    rows = cfg.heads * cfg.n_blocks
    density = {}
    for tau in (0.9, 0.95, 0.99, 1.0):
        buf.select(tau)
        density[str(tau)] = round(int(buf.indptr[-1].item()) / (rows * cfg.n_kblocks), 6)
    m = buf.mass.cpu().numpy().reshape(rows, cfg.n_kblocks).astype(np.float64)
    buf.select(args.tau)
    gi, gk, _ = buf.csr_host()
    k_match = max(1, int(round(len(gk) / rows)))
    row_tau = np.array([m[r, gk[gi[r]:gi[r + 1]]].sum() for r in range(rows)]) / m.sum(axis=1)
    buf.select_topk(k_match)
    ti, tk, _ = buf.csr_host()
    row_topk = np.array([m[r, tk[ti[r]:ti[r + 1]]].sum() for r in range(rows)]) / m.sum(axis=1)
    buf.select(args.tau)
    ablation = {"k_blocks_matched": k_match, "recall_mass_rule": round(float(row_tau.mean()), 6),
                "recall_topk": round(float(row_topk.mean()), 6),
                "worst_row_recall_mass_rule": round(float(row_tau.min()), 6),
                "worst_row_recall_topk": round(float(row_topk.min()), 6)}

    # Outside the timed region, after everything that reads this step's masses: the dense step alone (no masses),
    # which sets construction against one dense step at this shape, and the two-pass profile call (masses from a
    # second Q K^T pass, no workspace), each timed back to back with CUDA events and its own clock record.
    if not args.no_extras:
        def profile_series(reps, **kw):
            buf.profile(q, k, v, scale, **kw)
            torch.cuda.synchronize()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            with ClockSampler(local) as ck:
                ev[0].record(stream)
                for _ in range(reps):
                    buf.profile(q, k, v, scale, **kw)
                ev[1].record(stream)
                torch.cuda.synchronize()
            if L.losa_get_device_error() != 0:
                raise RuntimeError("device error in the profile series")
            return ev[0].elapsed_time(ev[1]) / reps, ck.summary()

        t_fwd, ck_fwd = profile_series(3, with_mass=False)
        t_two, ck_two = profile_series(3, one_pass=False)
        extras["dense_step_no_mass"] = {"ms": round(t_fwd, 3), "calls": 3, "clocks": ck_fwd,
                                        "profile_select_over_dense_step": round((per_prof + per_sel) * 1e3 / t_fwd,
                                                                                3)}
        extras["dense_profile_two_pass"] = {"ms": round(t_two, 3), "calls": 3, "clocks": ck_two}

    pk = peaks()
    tr = measured_traffic(cfg.name)
    roof = {
        "dense_profile": roofline("attn_dense_kernel<1, 1, 1> (losa_dense_profile_ws: dense forward with the block "
                                  "masses taken in the same pass)", "tensor", work["profile_flop"], per_prof, pk,
                                  "TFLOP/s", tr.get("dense_profile")),
        "select": roofline("select_rows + select_hist + select_order + select_scatter (losa_select)", "hbm",
                           work["select_bytes"], per_sel, pk, "GB/s", tr.get("select")),
        # the kept-block target is stated against the bf16 dense peak: the burst GEMM rate is the denominator
        "sparse_attn": roofline("attn_sparse_kernel over the retained lists (losa_sparse_attn)", "tensor",
                                work["sparse_flop"], per_sparse, pk, "TFLOP/s", tr.get("sparse_attn"),
                                peak_kind="burst"),
    }
    if "sparse_attn_steady" in extras:
        e = extras["sparse_attn_steady"]
        roof["sparse_attn_steady"] = roofline("attn_sparse_kernel, back-to-back sparse calls", "tensor",
                                              work["sparse_flop"], e["ms"] / 1e3, pk, "TFLOP/s", None,
                                              peak_kind="burst")
        e["dense_equiv_tflops"] = round(work["dense_equiv_flop"] / (e["ms"] / 1e3) / 1e12, 3)
        f = extras["sparse_attn_tau1"]
        roof["sparse_attn_tau1"] = roofline("attn_sparse_kernel, every list full (tau = 1)", "tensor",
                                            work_model(cfg, f["nnz_blocks"])["sparse_flop"], f["ms"] / 1e3, pk,
                                            "TFLOP/s", None, peak_kind="burst")
    if "dense_step_no_mass" in extras:
        roof["dense_step_no_mass"] = roofline("attn_dense_kernel<0, 1, 0> (losa_dense_profile without masses: the "
                                              "dense step)", "tensor", work["profile_flop"],
                                              extras["dense_step_no_mass"]["ms"] / 1e3, pk, "TFLOP/s", None)
        roof["dense_profile_two_pass"] = roofline("attn_dense_kernel<1, 1, 0> (losa_dense_profile: forward, then a "
                                                  "second Q K^T pass for the masses)", "tensor",
                                                  1.5 * work["profile_flop"],
                                                  extras["dense_profile_two_pass"]["ms"] / 1e3, pk, "TFLOP/s", None)
    dominant = max(("dense_profile", per_prof), ("select", per_sel), ("sparse_attn", per_sparse),
                   key=lambda x: x[1])[0]
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s (dense-equivalent, sparse attention)",
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": round(total_ms / K, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": cfg.dtype,
        "data": "synthetic: seeded grid-structured Q/K/V (per-head random Fourier locality, sink keys, padded tail)",
        "config": bench_config(cfg, args.tau, world),
        "sparse_attn_ms": round(per_sparse * 1e3, 3),
        "profile_ms": round(per_prof * 1e3, 3),
        "select_ms": round(per_sel * 1e3, 3),
        "profile_select_ms": round((per_prof + per_sel) * 1e3, 3),
        "dense_equiv_tflops": round(K * work["dense_equiv_flop"] / t_sparse / 1e12, 3),
        "kept_block_tflops": round(work["sparse_flop"] / per_sparse / 1e12, 3),
        "block_density": round(nnz / (cfg.heads * cfg.n_blocks * cfg.n_kblocks), 5),
        "block_density_by_tau": density,
        "topk_ablation": ablation,
        "nnz_blocks": nnz,
        "roofline": roof[dominant],
        "rooflines": roof,
        "gpu_launches": K * sum(KERNELS_PER_STEP.values()),
        "clocks": clocks.summary(),
        "e2e": e2e,
        **extras,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_cpu = args.cpu_items or oracle_threads()
        per = oracle_sample_run(cfg, oracle_inputs(layer), args.tau, n_cpu)
        line["cpu_baseline"] = cpu_line(cfg, per, f"{n_cpu} seeded items of {cfg.name} (dense forward, "
                                        f"masses, selection, restricted attention), extrapolated to all "
                                        f"{cfg.heads * cfg.n_blocks} items")
    if rank == 0:
        print(json.dumps(line), flush=True)
    group.close()
    return 0


# ------------------------------------------------------------------------------------------ reuse loop

def dense_reference_fp64(cfg, q, k, v, scale, items):
    """Dense attention of the listed items in float64 with plain torch CPU ops, for the loop's reported
    approximation error (rows t >= N are NaN)."""
    import torch
    R, nq, N = cfg.block, cfg.n_blocks, cfg.n_tokens
    out = np.full((len(items), R, cfg.head_dim), np.nan)
    kf, vf = k.double().cpu(), v.double().cpu()
    qf = q.double().cpu()
    for t, it in enumerate(items):
        h, i = divmod(int(it), nq)
        rows = min(R, N - i * R)
        s = (qf[h, i * R:i * R + rows] @ kf[h, :N].T) * scale
        out[t, :rows] = (torch.softmax(s, dim=-1) @ vf[h, :N]).numpy()
    return out


def pattern_recall(mass, indptr, kv_idx):
    """Recall of a CSR pattern under masses [rows][nk]: retained mass over total mass."""
    kept = sum(float(mass[r, kv_idx[indptr[r]:indptr[r + 1]]].sum()) for r in range(mass.shape[0]))
    return kept / float(mass.sum())


def run_loop(args, cfg):
    """Denoising-loop reuse at the Wan2.1-480p shape: steps before the construction step t0 are dense, step t0
    profiles every layer and selects its pattern (t0 = 0 by default; the LoSA page's setup uses t0 = 3), later steps
    run sparse attention with the frozen lists on Q/K/V that drift each step. Each layer's dense call on the same
    inputs is timed beside it, giving the 50-dense-step baseline. Reports totals, the sampled approximation error
    of the sparse output against fp64 dense attention, and the recall of the frozen pattern under later steps' exact
    masses."""
    import torch
    import free_block_sparse_losa_b200 as L
    from free_block_sparse_losa_b200.harness import LayerBuffers
    from losa_synth import Drift

    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    L.load()
    n_layers = args.loop_layers or cfg.layers
    n_steps = args.loop_steps or cfg.extra["steps"]
    layers = [make_layer(cfg, li) for li in range(n_layers)]
    drift = Drift(cfg, layers, seed=cfg.seed)
    scale = 1.0 / math.sqrt(cfg.head_dim)
    bufs = [LayerBuffers.for_config(cfg) for _ in range(n_layers)]
    dense_o = torch.empty_like(bufs[0].o)
    dense_lse = torch.empty_like(bufs[0].lse)
    probe = LayerBuffers.for_config(cfg)  # dense profile for recall measurements (not timed)
    stream = torch.cuda.current_stream()
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    t_sparse_path, t_dense_path = [], []
    t0 = args.construct_step
    report_steps = sorted({t0 + 1, n_steps // 5, n_steps // 2, n_steps - 1} & set(range(t0 + 1, n_steps)))
    rel_l2, recall = {}, {}
    items = sample_items(cfg, 8, seed=99)
    # warm-up of both call kinds on step-0 inputs
    q, k, v = drift.tokens(0)
    for _ in range(3):
        bufs[0].profile(q, k, v, scale)
        bufs[0].select(args.tau)
        bufs[0].sparse(q, k, v, scale)
        L.losa_dense_profile(bufs[0].shape, q, k, v, scale, dense_o, dense_lse, None)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for step in range(n_steps):
            if step > 0:
                drift.advance()
            step_sparse, step_dense = [], []
            for li in range(n_layers):
                q, k, v = drift.tokens(li)
                b = bufs[li]
                e0, e1, e2 = ev(), ev(), ev()
                e0.record(stream)
                if step < t0:
                    L.losa_dense_profile(b.shape, q, k, v, scale, b.o, b.lse, None)
                elif step == t0:
                    b.profile(q, k, v, scale)
                    b.select(args.tau)
                else:
                    b.sparse(q, k, v, scale)
                e1.record(stream)
                L.losa_dense_profile(b.shape, q, k, v, scale, dense_o, dense_lse, None)
                e2.record(stream)
                step_sparse.append((e0, e1))
                step_dense.append((e1, e2))
                if step in report_steps and li == 0:
                    torch.cuda.synchronize()
                    ref = dense_reference_fp64(cfg, q, k, v, scale, items)
                    got = b.o.float().cpu().numpy().reshape(cfg.heads * cfg.n_blocks, cfg.block, cfg.head_dim)
                    gd = dense_o.float().cpu().numpy().reshape(got.shape)
                    ok = ~np.isnan(ref)
                    rel_l2[step] = {"sparse_vs_dense_fp64": float(np.linalg.norm((got[items] - ref)[ok]) /
                                                                  np.linalg.norm(ref[ok])),
                                    "dense_kernel_vs_dense_fp64": float(np.linalg.norm((gd[items] - ref)[ok]) /
                                                                        np.linalg.norm(ref[ok]))}
                    probe.profile(q, k, v, scale)
                    m = probe.mass.cpu().numpy().reshape(probe.rows, probe.nk).astype(np.float64)
                    gi, gk, _ = b.csr_host()
                    recall[step] = pattern_recall(m, gi, gk)
            torch.cuda.synchronize()
            t_sparse_path.append(sum(a.elapsed_time(z) for a, z in step_sparse))
            t_dense_path.append(sum(a.elapsed_time(z) for a, z in step_dense))
    if L.losa_get_device_error() != 0:
        raise RuntimeError("device error in the reuse loop")
    nnz = [int(b.indptr[-1].item()) for b in bufs]
    loop_ms, dense_ms = sum(t_sparse_path), sum(t_dense_path)
    line = {"metric": f"denoising reuse loop ({n_layers} layers x {n_steps} steps): dense steps, profile+select at "
                      f"step {t0}, then sparse steps, vs dense steps", "value": round(dense_ms / loop_ms, 4),
            "unit": "x (dense loop time / LoSA loop time)", "n_gpus": 1, "steps": n_steps, "warmup": 3,
            "ms_per_step": round(loop_ms / n_steps, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": cfg.dtype, "data": "synthetic, drifted 0.02 rms per step",
            "config": {"workload": cfg.name, "layers": n_layers, "heads": cfg.heads, "n_tokens": cfg.n_tokens,
                       "head_dim": cfg.head_dim, "block": cfg.block, "tau": args.tau},
            "loop_ms": round(loop_ms, 3), "dense_loop_ms": round(dense_ms, 3),
            "construct_step": t0,
            "construct_step_profile_select_ms": round(t_sparse_path[t0], 3),
            "construct_step_dense_ms": round(t_dense_path[t0], 3),
            "sparse_step_ms_mean": round(float(np.mean(t_sparse_path[t0 + 1:])), 3) if n_steps > t0 + 1 else None,
            "dense_step_ms_mean": round(float(np.mean(t_dense_path)), 3),
            "block_density": round(sum(nnz) / (n_layers * cfg.heads * cfg.n_blocks ** 2), 5),
            "rel_l2_layer0_sampled": rel_l2, "recall_of_frozen_pattern_layer0": recall,
            "gpu_launches": n_layers * (t0 + 1 + 3 + (n_steps - 1 - t0) + n_steps),
            "clocks": clocks.summary()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", choices=sorted(CONFIGS), default="hunyuan720")
    ap.add_argument("--tau", type=float, default=0.99)
    ap.add_argument("--block-k", type=int, default=0, choices=[0, 32, 128],
                    help="key block size C (0: the workload's, 128; 32 is the LoSA page's setup)")
    ap.add_argument("--cpu-items", type=int, default=0, help="oracle sample size (0: one item per host thread)")
    ap.add_argument("--ref-items", type=int, default=0, help="reference-arm items per step (0: half the threads)")
    ap.add_argument("--loop-layers", type=int, default=0, help="reuse loop: layers (0: the config's 30)")
    ap.add_argument("--loop-steps", type=int, default=0, help="reuse loop: denoising steps (0: the config's 50)")
    ap.add_argument("--construct-step", type=int, default=0, help="reuse loop: step t0 that builds the pattern")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true", help="skip the steady-state and tau = 1 sparse timings")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    cfg = CONFIGS[args.workload]
    if args.block_k:
        import dataclasses
        cfg = dataclasses.replace(cfg, block_k=args.block_k)
    if args.workload == "loop":
        if args.impl == "reference":
            print(json.dumps({"impl": "reference", "unavailable": "the reuse loop has no CPU-oracle arm; its "
                              "accuracy is checked against the oracle inside the loop"}))
            return 0
        return run_loop(args, cfg)
    if args.impl == "reference":
        return run_reference(args, cfg)
    return run_native(args, cfg)


if __name__ == "__main__":
    sys.exit(main())
