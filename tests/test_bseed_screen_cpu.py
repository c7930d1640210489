"""The screen of the fused batched-seeding round, checked on the host.

The round keeps a point's D2 without computing its exact distance when
    est - 2^-9 (3 |x|^2 + 2 |est|) > D2,     est = |x|^2 - 2 acc,
where acc is the tensor-core fp32 accumulation of <x, c> (bf16 operands,
products exact in fp32) plus a ninth K step adding the three bf16 parts of
-|c|^2 / 2, and |x|^2, |c|^2 are fp32 sums of squares.  That is exact only
if |est - |x - c|^2| stays below the margin.  The accumulation order and
rounding of the tensor cores are not specified, so this emulates two
extremes in numpy (fp32 adds in k order rounded to nearest, and the same
adds rounded toward zero) and checks that the error stays under a twentieth
of the margin: on clustered points and centres drawn from them, on far
points, on a point equal to its centre, and on magnitudes over six orders.
"""
import numpy as np
import pytest


def bf16(x):
    """Round fp32 values to bf16 (nearest even) and back, like the storage."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


def add32(a, b, toward_zero):
    """a + b in fp32, rounded to nearest or toward zero (the fp64 sum of two
    fp32 values of these magnitudes is exact)."""
    s = np.float64(a) + np.float64(b)
    r = np.float32(s)
    if toward_zero and abs(np.float64(r)) > abs(s):
        r = np.nextafter(r, np.float32(0.0))
    return r


def bias_parts(c):
    """The three bf16 parts of -|c|^2 / 2 (fp32 |c|^2), as the pick kernel forms them."""
    cn = np.float32(0.0)
    for v in c:
        cn = np.float32(np.float32(v) * np.float32(v) + cn)
    b = np.float32(-0.5) * cn
    hi = bf16(b)
    r1 = np.float32(b - hi)
    mid = bf16(r1)
    lo = bf16(np.float32(r1 - mid))
    return [hi, mid, lo], cn


def estimate(x, c, toward_zero):
    acc = np.float32(0.0)
    for xi, ci in zip(x, c):
        acc = add32(acc, np.float32(xi) * np.float32(ci), toward_zero)  # bf16 x bf16: exact in fp32
    parts, _ = bias_parts(c)
    for p in parts:
        acc = add32(acc, p, toward_zero)  # the ninth K step: ones x the parts
    xn = np.float32(0.0)
    for v in x:
        xn = np.float32(np.float32(v) * np.float32(v) + xn)
    est = np.float32(xn - np.float32(2.0) * acc)
    margin = np.float32((np.float32(3.0) * xn + np.float32(2.0) * abs(est)) * np.float32(2.0 ** -9))
    return float(est), float(margin)


@pytest.mark.parametrize("toward_zero", [False, True])
@pytest.mark.parametrize("d", [128])
def test_screen_error_is_far_inside_its_margin(d, toward_zero):
    g = np.random.default_rng(17 + int(toward_zero))
    means = g.standard_normal((32, d)).astype(np.float32)
    worst = 0.0
    for trial in range(1500):
        kind = trial % 5
        scale = 10.0 ** g.uniform(-3, 3)
        if kind == 0:      # clustered point and a centre of its own cluster
            m = means[g.integers(32)]
            x = bf16((m + 0.3 * g.standard_normal(d)) * scale)
            c = bf16((m + 0.3 * g.standard_normal(d)) * scale)
        elif kind == 1:    # a centre from another cluster
            x = bf16((means[g.integers(32)] + 0.3 * g.standard_normal(d)) * scale)
            c = bf16((means[g.integers(32)] + 0.3 * g.standard_normal(d)) * scale)
        elif kind == 2:    # the point is the centre
            x = bf16(g.standard_normal(d) * scale)
            c = x.copy()
        elif kind == 3:    # a near-duplicate
            x = bf16(g.standard_normal(d) * scale)
            c = bf16(x + g.standard_normal(d) * 1e-3 * scale)
        else:              # different magnitudes
            x = bf16(g.standard_normal(d) * scale)
            c = bf16(g.standard_normal(d) * scale * 10.0 ** g.uniform(-1, 1))
        exact = float(np.sum((x.astype(np.float64) - c.astype(np.float64)) ** 2))
        est, margin = estimate(x, c, toward_zero)
        err = abs(est - exact)
        assert err <= margin / 20.0, (trial, kind, err, margin)
        worst = max(worst, err / margin)
    assert worst > 0.0  # the emulation did round


def test_screen_keeps_d2_only_when_the_exact_distance_would():
    """Where the screen keeps D2 (est - margin > D2), the exact distance is at
    least D2, for D2 just below, at and above the exact distance."""
    g = np.random.default_rng(5)
    for _ in range(400):
        x = bf16(g.standard_normal(128))
        c = bf16(x + 0.5 * g.standard_normal(128))
        exact = float(np.sum((x.astype(np.float64) - c.astype(np.float64)) ** 2))
        est, margin = estimate(x, c, False)
        for d2 in (exact * (1 - 1e-3), exact, exact * (1 + 1e-3), est - margin * 1.0001):
            if est - margin > d2:
                assert exact >= d2
