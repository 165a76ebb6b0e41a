"""The attention kernel's software exp2 (Cody-Waite split + cubic), evaluated
step by step in float32 exactly as the kernel does, against numpy's exp2.

The kernel uses it for one exponential in four; its error must stay far below
the bf16 rounding applied to P (2^-9 relative) and keep LSE within 1e-3.
"""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(__file__)), "sparse_attention_video_b200",
                   "csrc", "sa_exp2_poly.h")


def _coeffs():
    txt = open(HDR).read()
    c = dict(re.findall(r"kExp2C(\d) = ([-0-9.e]+)f;", txt))
    return [np.float32(c[str(i)]) for i in range(4)]


def _exp2_poly(x):
    c0, c1, c2, c3 = _coeffs()
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-125.0))
    magic = f32(12582912.0)
    t = (x + magic).astype(f32)
    f = (x - (t - magic)).astype(f32)
    p = ((c3 * f + c2) * f + c1) * f + c0
    p = p.astype(f32)
    n = t.view(np.int32) - np.array([magic], f32).view(np.int32)[0]
    return (p.view(np.int32) + (n << 23)).view(f32)


def test_relative_error_over_the_kernel_range():
    x = np.concatenate([np.linspace(-125.0, 8.0, 2_000_001), -np.logspace(-8, 0, 10_001),
                        np.arange(-125, 9, dtype=np.float64)]).astype(np.float32)
    got = _exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1.2e-4, rel.max()


def test_minus_infinity_floors_at_a_normal_tiny_value():
    v = _exp2_poly(np.array([-np.inf, -1e30], np.float32))
    assert np.all(v > 0) and np.all(v < 1e-37)


def test_exact_at_integers_within_polynomial_error():
    x = np.arange(-20, 9, dtype=np.float32)
    np.testing.assert_allclose(_exp2_poly(x), np.exp2(x.astype(np.float64)), rtol=1e-4)
