"""The FMA-pipe exp2 used for part of the softmax: its coefficients are the minimax fit that
exp2_poly.py derives, and the whole evaluation (range reduction, polynomial, exponent add),
replayed in float32 arithmetic, stays within its relative error bound of 2^x."""
import os
import re

import numpy as np

from tiled_attention_26_b200 import exp2_poly

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "tiled_attention_26_b200", "csrc", "sm100.cuh")


def kernel_coefficients():
    text = open(HDR).read()
    body = text[text.index("float exp2_fma("):]
    body = body[: body.index("}\n")]
    lits = [float(x) for x in re.findall(r"(?<![\d.])(\d\.\d+)f", body)]
    # fmaf(c3, f, c2); fmaf(p, f, c1); fmaf(p, f, c0)
    return lits[0], lits[1], lits[2], lits[3]


def f32(x):
    return np.float32(x)


def fma32(a, b, c):
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def exp2_fma_model(x):
    x = np.asarray(x, dtype=np.float32)
    c3, c2, c1, c0 = (np.float32(v) for v in kernel_coefficients())
    t = (x + np.float32(12582912.0)).astype(np.float32)
    n = (t - np.float32(12582912.0)).astype(np.float32)
    f = (x - n).astype(np.float32)
    p = fma32(c3, f, c2)
    p = fma32(p, f, c1)
    p = fma32(p, f, c0)
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_coefficients_are_the_derived_minimax():
    c, err = exp2_poly.remez_exp2(3)
    c3, c2, c1, c0 = kernel_coefficients()
    assert np.allclose([c0, c1, c2, c3], c, rtol=1e-6, atol=0)
    assert err < 8e-5


def test_relative_error_over_the_clamped_range():
    x = np.concatenate([np.linspace(-125.0, 64.0, 2_000_003, dtype=np.float32),
                        np.float32([-125.0, -0.5, 0.0, 0.5, 1.0, 8.0, -7.5, 63.5])])
    got = exp2_fma_model(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1e-4, rel.max()
    assert np.all(got > 0)


def test_exact_at_integers():
    # f = 0 -> p = c0, so 2^n comes out as c0 * 2^n: relative error |c0 - 1| < 1e-4
    n = np.arange(-120, 60, dtype=np.float32)
    got = exp2_fma_model(n).astype(np.float64)
    assert np.max(np.abs(got / np.exp2(n.astype(np.float64)) - 1)) < 1e-4
