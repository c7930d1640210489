"""The oracle still reproduces its committed regression fixture (tests/golden)."""
import json
import os

import numpy as np

from long_prefix_attention_b200 import inputs
from oracle import asm_oracle as O

HERE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_oracle_tiny_fp32_fixture():
    with open(os.path.join(HERE, "oracle_tiny_fp32.json")) as f:
        fx = json.load(f)
    b = inputs.build_inputs(inputs.CONFIGS[0], N=256, L=96, K=16)
    A, lz = O.build_states(b["q"], b["k"], b["v"], b["scale"])
    seeds = O.kmeanspp_seed(b["q"], b["u"])
    C, Cq, assign, counts, inertia = O.kmeans(b["q"], seeds, 3, O.L2, O.F32)
    Ab, lzb = O.aggregate(A[0], lz[0], assign[0], 16, O.ZBAR_MEAN)
    np.testing.assert_allclose(lz[0, :8], fx["logz_h0_first8"], atol=1e-12)
    np.testing.assert_allclose(A[1, 5, :8], fx["a_h1_q5_first8"], atol=1e-12)
    assert seeds[0].tolist() == fx["kmeanspp_idx_h0"]
    assert counts[0].tolist() == fx["kmeans_counts_h0"]
    np.testing.assert_allclose(inertia[0], fx["kmeans_inertia_h0"], rtol=1e-12)
    np.testing.assert_allclose(lzb, fx["logz_bar_h0"], atol=1e-12)
