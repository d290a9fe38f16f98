"""Seeded synthetic inputs for the LoSA hot path.

This module is shared by the CPU oracle's tests and by the CUDA path's tests and benchmark. It holds
no part of the method's arithmetic: it only draws Q/K/V tensors with the structure of a video
diffusion transformer's self-attention layer (a 3D token grid flattened row-major over (t, y, x),
attention that is local in space-time, a few "sink" keys) and rounds them to the storage dtype.
Both sides read the same rounded tensors.

Recipe (per head, from its own PCG64 sub-stream, draws in this order):
  1. lengthscale l: fixed per axis (config "tiny") or log l ~ U[ln lo, ln hi], isotropic;
  2. W ~ N(0, I_3) of shape (3, d) and b ~ U[0, 2 pi) of shape (d,);
  3. phi(p) = cos(W^T (p / l) + b), a d-dimensional random Fourier feature map of the token's
     (t, y, x) position with unit amplitude;
  4. q = a * phi + 0.3 * eps_q,  k = a * phi + 0.3 * eps_k  (eps ~ N(0, 1)),  v ~ N(0, 1);
  5. n_sinks distinct valid token indices drawn uniformly; their k rows are multiplied by 3.
Rows N..Np-1 (the padding up to a multiple of the block size) are zero. Generation runs in fp64 and
is rounded once to fp32 (round-to-nearest-even) and, for bf16 configs, from fp32 to bf16 (RNE).
Sub-streams: numpy SeedSequence(seed).spawn(layers * heads); head h of layer l uses child l*H + h.
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

__all__ = ["LayerConfig", "CONFIGS", "Layer", "make_layer", "bf16_bits_to_f32", "f32_to_bf16_bits",
           "round_to_bf16", "pad_to", "sample_items"]


def pad_to(n: int, block: int) -> int:
    return ((n + block - 1) // block) * block


@dataclass(frozen=True)
class LayerConfig:
    """Shape and generator parameters of one synthetic attention layer (batch 1)."""
    name: str
    heads: int
    grid: tuple            # (T, Y, X) token grid; N = T*Y*X, flattened row-major (t, y, x)
    head_dim: int
    block: int             # query block size R (and key/value block size C unless block_k is set)
    dtype: str             # "f32" or "bf16"
    amplitude: float       # a
    ell_fixed: tuple | None = None      # per-axis lengthscale (t, y, x), or None
    ell_range: tuple = (1.0, 8.0)       # log-uniform range for the isotropic lengthscale
    n_sinks: int = 0
    noise: float = 0.3
    sink_gain: float = 3.0
    seed: int = 0
    layers: int = 1
    taus: tuple = (0.99,)
    extra: dict = field(default_factory=dict)
    block_k: int = 0       # key/value block size C when it differs from R (the LoSA page's setup: R = 128, C = 32)

    @property
    def kblock(self) -> int:
        return self.block_k or self.block

    @property
    def n_kblocks(self) -> int:
        return self.n_padded // self.kblock

    @property
    def n_tokens(self) -> int:
        t, y, x = self.grid
        return t * y * x

    @property
    def n_padded(self) -> int:
        return pad_to(self.n_tokens, self.block)

    @property
    def n_blocks(self) -> int:
        return self.n_padded // self.block


CONFIGS = {
    "tiny": LayerConfig("tiny-4x8x8-h2-d64-f32", heads=2, grid=(4, 8, 8), head_dim=64, block=64, dtype="f32",
                   amplitude=3.0, ell_fixed=(2.0, 3.0, 3.0), n_sinks=0, seed=0, taus=(0.9, 0.99, 1.0)),
    "wan1.3b480": LayerConfig("wan2.1-1.3b-480p-21x30x52-h12", heads=12, grid=(21, 30, 52), head_dim=128, block=128,
                   dtype="bf16", amplitude=4.0, ell_range=(1.0, 8.0), n_sinks=2, seed=1,
                   taus=(0.9, 0.95, 0.99, 1.0)),
    "wan14b720": LayerConfig("wan2.1-14b-720p-21x45x80-h40", heads=40, grid=(21, 45, 80), head_dim=128, block=128,
                   dtype="bf16", amplitude=4.0, ell_range=(1.0, 12.0), n_sinks=2, seed=2, taus=(0.99,)),
    "hunyuan720": LayerConfig("hunyuanvideo-720p-33x45x80-h24", heads=24, grid=(33, 45, 80), head_dim=128, block=128,
                   dtype="bf16", amplitude=4.0, ell_range=(1.0, 8.0), n_sinks=2, seed=3, taus=(0.99,)),
    "loop": LayerConfig("wan2.1-1.3b-480p-loop-30layers-h12", heads=12, grid=(21, 30, 52), head_dim=128, block=128,
                   dtype="bf16", amplitude=4.0, ell_range=(1.0, 8.0), n_sinks=2, seed=4, layers=30,
                   taus=(0.99,), extra={"steps": 50, "drift": 0.02}),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round-to-nearest-even) and return the 16-bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    bits = x.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = (bits + 0x7FFF + lsb) >> 16
    nan = np.isnan(x)
    out = rounded.astype(np.uint16)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(f32_to_bf16_bits(np.asarray(x, dtype=np.float32)))


def _positions(grid) -> np.ndarray:
    t, y, x = grid
    tt, yy, xx = np.meshgrid(np.arange(t), np.arange(y), np.arange(x), indexing="ij")
    return np.stack([tt.ravel(), yy.ravel(), xx.ravel()], axis=1).astype(np.float64)


@dataclass
class Layer:
    """One generated layer. q/k/v are [H][Np][d]; fp32 arrays for "f32", uint16 bf16 bits for "bf16"."""
    cfg: LayerConfig
    q: np.ndarray
    k: np.ndarray
    v: np.ndarray
    lengthscales: np.ndarray
    sinks: np.ndarray

    def head_f32(self, name: str, h: int) -> np.ndarray:
        """Rounded values of one head of q, k or v as fp32 [Np][d] (exact)."""
        a = getattr(self, name)[h]
        return a if self.cfg.dtype == "f32" else bf16_bits_to_f32(a)

    def all_f32(self, name: str) -> np.ndarray:
        a = getattr(self, name)
        return a if self.cfg.dtype == "f32" else bf16_bits_to_f32(a)


def _gen_head(cfg: LayerConfig, ss: np.random.SeedSequence, pos: np.ndarray):
    rng = np.random.Generator(np.random.PCG64(ss))
    n, d = cfg.n_tokens, cfg.head_dim
    if cfg.ell_fixed is not None:
        ell = np.asarray(cfg.ell_fixed, dtype=np.float64)
    else:
        lo, hi = cfg.ell_range
        ell = np.full(3, math.exp(rng.uniform(math.log(lo), math.log(hi))))
    w = rng.standard_normal((3, d))
    b = rng.uniform(0.0, 2.0 * math.pi, size=d)
    phi = np.cos((pos / ell) @ w + b)
    q = cfg.amplitude * phi + cfg.noise * rng.standard_normal((n, d))
    k = cfg.amplitude * phi + cfg.noise * rng.standard_normal((n, d))
    v = rng.standard_normal((n, d))
    sinks = np.sort(rng.choice(n, size=cfg.n_sinks, replace=False)) if cfg.n_sinks else np.zeros(0, np.int64)
    if cfg.n_sinks:
        k[sinks] *= cfg.sink_gain
    out = []
    for a in (q, k, v):
        a32 = np.zeros((cfg.n_padded, d), dtype=np.float32)
        a32[:n] = a.astype(np.float32)
        out.append(a32 if cfg.dtype == "f32" else f32_to_bf16_bits(a32))
    return out, float(ell[0]) if cfg.ell_fixed is None else ell.copy(), sinks


def make_layer(cfg: LayerConfig | str, layer: int = 0, threads: int = 8) -> Layer:
    """Generate layer `layer` of a config, given as a LayerConfig or a workload name (layer > 0 only for
    multi-layer configs)."""
    if isinstance(cfg, str):
        cfg = CONFIGS[cfg]
    if not 0 <= layer < cfg.layers:
        raise ValueError("layer out of range")
    children = np.random.SeedSequence(cfg.seed).spawn(cfg.layers * cfg.heads)
    pos = _positions(cfg.grid)
    store = np.uint16 if cfg.dtype == "bf16" else np.float32
    shape = (cfg.heads, cfg.n_padded, cfg.head_dim)
    q, k, v = (np.empty(shape, dtype=store) for _ in range(3))
    ells, sinks = [None] * cfg.heads, [None] * cfg.heads

    def work(h):
        (qh, kh, vh), ell, sk = _gen_head(cfg, children[layer * cfg.heads + h], pos)
        q[h], k[h], v[h] = qh, kh, vh
        ells[h], sinks[h] = ell, sk

    with ThreadPoolExecutor(max_workers=max(1, threads)) as ex:
        list(ex.map(work, range(cfg.heads)))
    return Layer(cfg, q, k, v, np.asarray(ells, dtype=np.float64), np.asarray(sinks))


def sample_items(cfg: LayerConfig, n: int = 64, seed: int = 12345, must_include=()) -> np.ndarray:
    """Seeded sample of (head, q-block) item ids h*nq + qb, sorted, including `must_include` ids
    and always the tail q-block of head 0."""
    nq = cfg.n_blocks
    total = cfg.heads * nq
    rng = np.random.Generator(np.random.PCG64(seed))
    forced = {nq - 1, *[int(i) for i in must_include]}
    n = min(n, total)
    pool = rng.permutation(total)
    chosen = list(forced)
    for i in pool:
        if len(chosen) >= n:
            break
        if int(i) not in forced:
            chosen.append(int(i))
    return np.asarray(sorted(chosen[:max(n, len(forced))]), dtype=np.int32)


class Drift:
    """Per-step drift of a multi-layer config's Q/K/V on the device (the reuse-loop input).

    X_s = X_{s-1} + amount * rms(X_0[layer, head]) * eps_s, eps_s ~ N(0, 1) drawn fresh for every step, layer and tensor
    from a torch generator seeded with (seed, step, layer); rms over the real rows of each head of the step-0 tensor.
    The walk is kept in fp32 master copies; `tokens(layer)` returns the rounded tensors the kernels read (bf16 by
    round-to-nearest-even, the same rounding as the host generator).
    """

    def __init__(self, cfg: "LayerConfig", layers: list, device="cuda", amount: float | None = None, seed: int = 0):
        import torch
        self.torch = torch
        self.cfg = cfg
        self.device = device
        self.amount = cfg.extra.get("drift", 0.02) if amount is None else amount
        self.seed = seed
        self.step = 0
        self.master = []   # per layer: (q, k, v) fp32 [H][Np][d]
        self.rms = []      # per layer: (3, H) fp32
        n = cfg.n_tokens
        for layer in layers:
            # own copies: the walk must not write into the layer's arrays (a same-device .to() would alias them)
            ts = tuple(torch.from_numpy(layer.all_f32(name)).to(device, copy=True) for name in ("q", "k", "v"))
            self.master.append(ts)
            self.rms.append(torch.stack([t[:, :n].pow(2).mean(dim=(1, 2)).sqrt() for t in ts]))

    def advance(self):
        """Apply one drift step to every layer."""
        torch = self.torch
        self.step += 1
        n = self.cfg.n_tokens
        for li, ts in enumerate(self.master):
            g = torch.Generator(device=self.device)
            g.manual_seed((self.seed * 1_000_003 + self.step) * 4099 + li)
            for ti, t in enumerate(ts):
                eps = torch.randn(t[:, :n].shape, generator=g, device=self.device, dtype=torch.float32)
                t[:, :n].add_(eps * (self.amount * self.rms[li][ti]).view(-1, 1, 1))

    def tokens(self, li: int):
        """The current rounded q, k, v of layer li as device tensors of the config dtype."""
        torch = self.torch
        dt = torch.bfloat16 if self.cfg.dtype == "bf16" else torch.float32
        return tuple(t.to(dt) for t in self.master[li])
