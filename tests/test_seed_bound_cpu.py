"""The lower bound behind the exact pruning of the k-means++ update.

A piece of a group is skipped when a lower bound of |c - a| (c the new
centre, a the group's anchor) exceeds R + M.  The bound comes from int8
copies with power-of-two scales:
    |c - a| >= |c' - a'| - |c - c'| - |a - a'|,
where |c' - a'|^2 = s_c^2 |q_c|^2 + s_a^2 |q_a|^2 - 2 s_c s_a <q_c, q_a> is
formed in fp64 from an exact integer dot product and each quantisation error
is computed in fp64 and rounded up.  This checks, with the same arithmetic
steps in numpy, that the bound (minus the slack the test adds) never exceeds
the exact distance: on random pairs, on equal vectors, and on vectors whose
magnitudes span many orders.  It checks the bound's mathematics on the host;
the GPU parity tests check that the pruned update returns the unpruned picks.
"""
import numpy as np
import pytest


def q8(v):
    """Power-of-two scale with max|v| <= 127 s, codes, |codes|^2, error (rounded up)."""
    v = v.astype(np.float32)
    amax = float(np.max(np.abs(v)))
    if not amax > 0:
        s = np.float32(1.0)
    else:
        _, e = np.frexp(np.float32(amax * np.float32(1.0 / 127.0) * np.float32(1.0 + 1e-6)))
        s = np.float32(np.ldexp(np.float32(1.0), int(e)))
    q = np.clip(np.rint(v / s), -127, 127).astype(np.int64)
    err = np.sqrt(np.sum((v.astype(np.float64) - q.astype(np.float64) * float(s)) ** 2)) * (1 + 1e-12)
    err = np.nextafter(np.float32(err), np.float32(np.inf))  # rounded up to float
    return float(s), q, int(np.sum(q * q)), float(err)


def lower_bound(c, a):
    sc, qc, nc, ec = q8(c)
    sa, qa, na, ea = q8(a)
    dot = int(np.sum(qc * qa))
    dc2 = sc * sc * nc + sa * sa * na - 2.0 * sc * sa * dot
    slack = 1e-7 * (sc * np.sqrt(nc) + sa * np.sqrt(na))
    return np.sqrt(max(dc2, 0.0)) - ec - ea - slack


def bf16(x):
    """Round fp32 values to bf16 (nearest even) and back, like the storage."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32)


@pytest.mark.parametrize("d", [64, 128])
def test_bound_never_exceeds_the_exact_distance(d):
    g = np.random.default_rng(11 + d)
    worst = np.inf
    for trial in range(3000):
        scale_c, scale_a = 10.0 ** g.uniform(-3, 3, 2)
        c = bf16(g.standard_normal(d) * scale_c)
        if trial % 5 == 0:
            a = c.copy()                                     # the same point
        elif trial % 5 == 1:
            a = bf16(c + g.standard_normal(d) * 1e-3 * scale_c)  # a close point
        else:
            a = bf16(g.standard_normal(d) * scale_a)
        exact = np.sqrt(np.sum((c.astype(np.float64) - a.astype(np.float64)) ** 2))
        lb = lower_bound(c, a)
        assert lb <= exact, (trial, lb, exact)
        worst = min(worst, exact - lb)
    assert worst >= 0.0


def test_bound_with_clamped_codes_and_zero_vectors():
    d = 128
    c = np.zeros(d, np.float32)
    a = np.zeros(d, np.float32)
    assert lower_bound(c, a) <= 0.0
    a[3] = 1.0
    assert lower_bound(c, a) <= 1.0
    # one huge coordinate and many tiny ones: most codes round to zero
    c = bf16(np.concatenate([[1e4], np.full(d - 1, 1e-3)]))
    a = bf16(np.concatenate([[-1e4], np.full(d - 1, -1e-3)]))
    exact = np.sqrt(np.sum((c.astype(np.float64) - a.astype(np.float64)) ** 2))
    assert lower_bound(c, a) <= exact
