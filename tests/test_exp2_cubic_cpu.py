"""The states kernel computes a quarter of its softmax exponentials on the FMA
pipe: 2^t = 2^n * 2^f with n = round(t) (taken with the 1.5 * 2^23 shift),
f = t - n in [-1/2, 1/2], 2^f by a cubic, and n added into the exponent
field, all in fp32 (csrc/build_states_tc.cu, exp2_poly_x2).  Its comment
claims a relative error below 7.5e-5 (under a quarter of a bf16 half-unit,
2^-9 / 4 = 4.9e-4).  This test replays the same steps in fp32 with numpy
(fused multiply-adds as an exact product plus one rounding) over a dense grid
of arguments and checks that bound against the exact 2^t.
"""
import math

import numpy as np

# the kernel's coefficients, highest degree first
C3, C2, C1, C0 = np.float32(0.0551716685), np.float32(0.2426111251), np.float32(0.6932609678), np.float32(0.9999280572)
SHIFT = np.float32(12582912.0)  # 1.5 * 2^23


def _fma32(a, b, c):
    """fp32 fused multiply-add: the product is exact in fp64, one rounding to fp32 at the end."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_cubic(t):
    t = np.maximum(np.asarray(t, np.float32), np.float32(-125.0))
    y = (t + SHIFT).astype(np.float32)           # round(t) lands in the low mantissa bits
    n = (y - SHIFT).astype(np.float32)
    f = _fma32(n, np.full_like(n, -1.0), t)      # t - n, exact
    p = _fma32(np.full_like(f, C3), f, np.full_like(f, C2))
    p = _fma32(p, f, np.full_like(f, C1))
    p = _fma32(p, f, np.full_like(f, C0))
    bits = (p.view(np.uint32).astype(np.uint64) + (y.view(np.uint32).astype(np.uint64) << np.uint64(23)))
    return (bits & np.uint64(0xFFFFFFFF)).astype(np.uint32).view(np.float32)


def test_relative_error_bound_over_the_softmax_range():
    # the softmax arguments are s * log2(e) - m <= 0; cover both signs and every fraction
    t = np.linspace(-100.0, 20.0, 1_200_001, dtype=np.float64).astype(np.float32)
    got = exp2_cubic(t).astype(np.float64)
    ref = np.exp2(t.astype(np.float64))
    rel = np.abs(got - ref) / ref
    assert rel.max() < 7.5e-5, rel.max()
    assert rel.max() < (2.0 ** -9) / 4  # under a quarter of a bf16 half-unit


def test_fraction_interval_endpoints_and_integers():
    f = np.array([-0.5, -0.25, 0.0, 0.25, 0.5, 1.0, -1.0, 7.0, -60.0], np.float32)
    got = exp2_cubic(f).astype(np.float64)
    ref = np.exp2(f.astype(np.float64))
    assert (np.abs(got - ref) / ref).max() < 7.5e-5
    # integers: f = 0, the cubic's constant term alone times 2^n
    assert abs(float(exp2_cubic(np.float32(-60.0))) / math.ldexp(1.0, -60) - float(C0)) < 1e-7


def test_clamp_keeps_very_negative_arguments_finite_and_tiny():
    got = exp2_cubic(np.array([-125.0, -200.0, -1e30], np.float32)).astype(np.float64)
    assert np.all(got > 0) and np.all(got < 1e-37)
    assert np.all(got == got[0])  # everything below -125 is clamped to it
