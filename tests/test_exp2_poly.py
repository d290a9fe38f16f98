"""Error bound of the kernel's polynomial 2^x (used for part of the softmax exponentials on the FMA pipe).

The coefficients are read from the CUDA source and the kernel's steps are replayed in fp32 (each fused multiply-add
rounded once): the Cody-Waite split x = n + f with n = round(x) by the 1.5 * 2^23 shift, a degree-4 polynomial for
2^f on [-1/2, 1/2], and n added to the exponent field. Against numpy's exp2 the relative error must stay below
4e-6 over the whole range the kernel feeds it (x in [-125, 8]), which is well inside the 1e-4 block-mass tolerance."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "free_block_sparse_losa_b200", "csrc", "attn_tc.cuh")


def _coeffs():
    text = open(SRC).read()
    c = {int(k): float(v) for k, v in re.findall(r"kExp2C(\d) = ([0-9.eE+-]+)f", text)}
    assert sorted(c) == [0, 1, 2, 3, 4]
    return [np.float32(c[i]) for i in range(5)]


def _fma(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly(x):
    c0, c1, c2, c3, c4 = _coeffs()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0)).astype(np.float32)).astype(np.float32)
    p = _fma(np.full_like(f, c4), f, np.full_like(f, c3))
    p = _fma(p, f, np.full_like(f, c2))
    p = _fma(p, f, np.full_like(f, c1))
    p = _fma(p, f, np.full_like(f, c0))
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-125.0, 8.0, 4_000_001).astype(np.float32)
    got = exp2_poly(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 4e-6, rel.max()


def test_integer_points_and_clamp():
    xs = np.arange(-125, 9, dtype=np.float32)
    got = exp2_poly(xs).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(xs.astype(np.float64)) - 1) < 1e-6)
    assert exp2_poly(np.float32(-400.0)) == exp2_poly(np.float32(-125.0))
