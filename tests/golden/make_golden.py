"""Write the oracle regression fixtures in this folder.

The pages print no worked numeric example, so every stored value here is
written by this script, which calls only the fp64 oracle (``oracle/``) on the
seeded tiny-fp32 workload (Hq=2, Hkv=1, d=64, prefix L=512, N=2048 calibration
queries from a 32-component mixture, K=64, local length 16).  The fixtures
guard the oracle against unintended changes; the pins in
``tests/test_oracle_pins.py`` are what tie it to the method.

Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from long_prefix_attention_b200 import inputs  # noqa: E402  (seeded generators only)
from oracle import asm_oracle as O  # noqa: E402


def main():
    cfg = inputs.CONFIGS[0]
    b = inputs.build_inputs(cfg, N=256, L=96, K=16)
    A, lz = O.build_states(b["q"], b["k"], b["v"], b["scale"])
    seeds = O.kmeanspp_seed(b["q"], b["u"])
    C, Cq, assign, counts, inertia = O.kmeans(b["q"], seeds, 3, O.L2, O.F32)
    Ab, lzb = O.aggregate(A[0], lz[0], assign[0], 16, O.ZBAR_MEAN)
    fx = {
        "source": "Context Memorization for Efficient Long Context Generation, Metodologia "
                  "(attention state, chunk merge, clustering, aggregation); values written by "
                  "tests/golden/make_golden.py from the fp64 oracle on the tiny-fp32 workload "
                  "cut to N=256, L=96, K=16.",
        "shape": {"Hq": 2, "Hkv": 1, "d": 64, "N": 256, "L": 96, "K": 16, "iters": 3},
        "logz_h0_first8": lz[0, :8].tolist(),
        "a_h1_q5_first8": A[1, 5, :8].tolist(),
        "kmeanspp_idx_h0": seeds[0].tolist(),
        "kmeans_counts_h0": counts[0].tolist(),
        "kmeans_inertia_h0": inertia[0].tolist(),
        "logz_bar_h0": lzb.tolist(),
    }
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny_fp32.json"), "w") as f:
        json.dump(fx, f, indent=1)


if __name__ == "__main__":
    main()
