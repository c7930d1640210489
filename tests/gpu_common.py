"""Helpers for the GPU parity tests: device copies and the parity rules.

Parity rule (tolerances of the tests): outputs agree within 2e-2 max abs for
bf16 storage and 1e-4 for fp32; centroid indices agree exactly except where
the oracle's relative top-2 gap is below 1e-4, and at those rows the output
is compared with the oracle re-run on the GPU's index.
"""
import numpy as np
import torch

TOL = {torch.bfloat16: 2e-2, torch.float32: 1e-4}
GAP = 1e-4


def dev(t):
    return t.to("cuda").contiguous()


def host(t):
    return t.detach().to("cpu")


def f64(t):
    return host(t).to(torch.float64).numpy()


def max_abs(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    fin = np.isfinite(a) & np.isfinite(b)
    assert (np.isneginf(a) == np.isneginf(b)).all(), "-inf pattern differs"
    return float(np.abs(a[fin] - b[fin]).max()) if fin.any() else 0.0


def check_indices(gpu_idx, ora_idx, ora_gap):
    """Indices equal except at near-ties; returns the mask of accepted mismatches."""
    gpu_idx, ora_idx, ora_gap = map(np.asarray, (gpu_idx, ora_idx, ora_gap))
    bad = gpu_idx != ora_idx
    assert not (bad & (ora_gap >= GAP)).any(), (
        f"{int((bad & (ora_gap >= GAP)).sum())} index mismatches with gap >= {GAP}")
    return bad
