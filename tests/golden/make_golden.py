"""Writes tiny_k5_L2_seed0.json: oracle outputs at sampled indices.

A regression fixture for the oracle itself (the pages print no worked
example for this layer).  Calls only `oracle/` and the seeded input
generator; run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from depthwise_convolution_wtconv_b200.configs import WORKLOADS  # noqa: E402
from depthwise_convolution_wtconv_b200.inputs import make_inputs, as_float64  # noqa: E402


def main():
    wl = WORKLOADS["tiny_k5_L2"]
    p = as_float64(make_inputs(wl, 0))
    Y = oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    g = oracle.backward(p["X"], p["dY"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    outs = dict(Y=Y, **g)
    pick = np.random.default_rng(0)
    tensors = {}
    for key, arr in outs.items():
        flat = arr.reshape(-1)
        idx = sorted(pick.choice(flat.size, size=min(16, flat.size), replace=False).tolist())
        tensors[key] = dict(index=idx, value=[float(flat[i]) for i in idx], sum=float(np.sum(flat)))
    doc = {
        "_source": "Written by tests/golden/make_golden.py from oracle/ only (workload tiny_k5_L2, seed 0).",
        "tensors": tensors,
    }
    with open(os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_k5_L2_seed0.json"), "w") as f:
        json.dump(doc, f, indent=1)


if __name__ == "__main__":
    main()
