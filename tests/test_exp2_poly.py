"""Error bounds of the sparse kernel's polynomial 2^x (used for part of the forward P on the FMA pipe).

The coefficients are read from the CUDA source and the kernel's steps are replayed in fp32 (each fused multiply-add
rounded once): the Cody-Waite split x = n + f with n = round(x) by the 1.5 * 2^23 shift, a polynomial for 2^f on
[-1/2, 1/2], and n added to the exponent field. Against numpy's exp2 over the whole range the kernels feed it
(x in [-125, 8]) the degree-3 form (forward P, rounded to bf16 next) stays below 8e-5 relative error, under a tenth
of bf16's relative half-step 2^-9."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "free_block_sparse_losa_b200", "csrc", "attn_tc.cuh")


def _coeffs(name="D", degree=3):
    text = open(SRC).read()
    c = {int(k): float(v) for k, v in re.findall(r"kExp2%s(\d) = ([0-9.eE+-]+)f" % name, text)}
    assert sorted(c) == list(range(degree + 1))
    return [np.float32(c[i]) for i in range(degree + 1)]


def _fma(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly(x, name="D", degree=3):
    c = _coeffs(name, degree)
    x = np.maximum(np.asarray(x, np.float32), np.float32(-125.0))
    t = (x + np.float32(12582912.0)).astype(np.float32)
    f = (x - (t - np.float32(12582912.0)).astype(np.float32)).astype(np.float32)
    p = _fma(np.full_like(f, c[degree]), f, np.full_like(f, c[degree - 1]))
    for k in range(degree - 2, -1, -1):
        p = _fma(p, f, np.full_like(f, c[k]))
    bits = (p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


def test_integer_points_and_clamp():
    xs = np.arange(-125, 9, dtype=np.float32)
    got = exp2_poly(xs).astype(np.float64)
    assert np.all(np.abs(got / np.exp2(xs.astype(np.float64)) - 1) < 8e-5)
    assert exp2_poly(np.float32(-400.0)) == exp2_poly(np.float32(-125.0))


def test_degree3_relative_error_bound():
    x = np.linspace(-125.0, 8.0, 4_000_001).astype(np.float32)
    got = exp2_poly(x).astype(np.float64)
    rel = np.abs(got / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 8e-5, rel.max()
    assert rel.max() < 0.1 * 2.0 ** -9
