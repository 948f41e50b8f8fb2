"""The FMA-pipe 2^x of the forward kernel (``exp2_poly_pair`` in
``csrc/fa2_forward.cu``), restated step by step in IEEE fp32 on the host and
checked against ``numpy.exp2`` (no GPU).

The kernel computes 2^x for x <= 0 as: clamp at -125; j = round(x) by adding
and subtracting 1.5 * 2^23 (the fp32 adds round to nearest even); f = x - j
in [-1/2, 1/2]; 2^f by a cubic in Horner form with fused multiply-adds; 2^j
by adding j to the exponent field.  The cubic is a minimax (Remez) fit made
for the kernel; its relative error bound is 7.5e-5, well under the 2^-9
rounding of the bf16 probabilities it produces ("FlashAttention 2: Three
Places the Chip Was Still Waiting", section 2.1, on moving scalar work off
the unit that bounds it).

The coefficients are read from the kernel source, so the test checks the
arithmetic the kernel compiles.
"""

import os
import re

import numpy as np
import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "exact_tiled_attention_29_b200", "csrc", "fa2_forward.cu")


def kernel_coefficients():
    text = open(SRC).read()
    coef = {}
    for i in range(4):
        m = re.search(rf"constexpr float kExp2C{i} = ([0-9.eE+-]+)f;", text)
        assert m, f"kExp2C{i} not found in the kernel source"
        coef[i] = np.float32(float(m.group(1)))
    return [coef[i] for i in range(4)]


def f32(x):
    return np.asarray(x, dtype=np.float32)


def fma32(a, b, c):
    """fp32 fused multiply-add: the product of two fp32 values is exact in
    fp64, the sum is rounded once to fp64 and then to fp32 (the double
    rounding can differ from a true fma only in rare last-bit ties)."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly(x, coef):
    c0, c1, c2, c3 = coef
    x = np.maximum(f32(x), np.float32(-125.0))
    rnd = np.float32(12582912.0)  # 1.5 * 2^23
    t = (x + rnd).astype(np.float32)          # low mantissa bits hold j
    jf = (t - rnd).astype(np.float32)         # j as a float
    f = fma32(jf, f32(np.full_like(x, -1.0)), x)
    q = fma32(f32(np.full_like(x, c3)), f, f32(np.full_like(x, c2)))
    q = fma32(q, f, f32(np.full_like(x, c1)))
    q = fma32(q, f, f32(np.full_like(x, c0)))
    bits = q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.int32).view(np.float32), f, jf


def test_reduction_is_exact_and_in_range():
    x = f32(np.linspace(-125.0, 0.0, 400_001))
    _, f, jf = exp2_poly(x, kernel_coefficients())
    assert np.all(np.abs(f) <= 0.5)
    assert np.array_equal(jf, np.round(x))          # ties to even, like the fp32 add
    assert np.array_equal(f.astype(np.float64), x.astype(np.float64) - jf.astype(np.float64))


def test_relative_error_over_the_softmax_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([f32(np.linspace(-125.0, 0.0, 2_000_001)),
                        f32(-rng.random(1_000_000) * 125.0),
                        f32(-rng.random(1_000_000) * 2.0)])
    got, _, _ = exp2_poly(x, kernel_coefficients())
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got.astype(np.float64) - ref) / ref
    assert rel.max() <= 1e-4, rel.max()
    assert got.max() <= 1.0 + 1e-4


@pytest.mark.parametrize("x,expect", [(0.0, 1.0), (-1.0, 0.5), (-10.0, 2.0 ** -10), (-125.0, 2.0 ** -125)])
def test_integer_points(x, expect):
    got, _, _ = exp2_poly(f32([x]), kernel_coefficients())
    assert abs(float(got[0]) / expect - 1.0) <= 1e-4


def test_clamp_below_the_normal_range():
    # anything below -125 becomes 2^-125: small, normal, never a denormal or garbage
    got, _, _ = exp2_poly(f32([-126.0, -200.0, -1e30]), kernel_coefficients())
    assert np.all(got == got[0]) and abs(float(got[0]) / 2.0 ** -125 - 1.0) <= 1e-4
