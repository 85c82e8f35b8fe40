"""The same-GPU comparator of bench.py (the layer as plain PyTorch ops with
autograd) computes the layer: its forward and every gradient equal the
oracle's in float64 on the CPU, so the time and memory it reports are those
of the same computation."""
import os
import sys

import numpy as np
import pytest
import torch

import oracle
from depthwise_convolution_wtconv_b200.configs import Workload
from depthwise_convolution_wtconv_b200.inputs import as_float64, make_inputs

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402


@pytest.mark.parametrize("shape", [(2, 3, 16, 16, 5, 2), (1, 2, 16, 8, 3, 3), (2, 2, 12, 12, 3, 0)])
def test_torch_cascade_matches_oracle_forward_and_gradients(shape):
    N, C, H, W, k, L = shape
    p = as_float64(make_inputs(Workload("c", N, C, H, W, k, L, "f32"), 2))
    t = {key: torch.tensor(p[key], requires_grad=True) for key in ("X", "W0", "b0", "s0")}
    t["Wl"] = torch.tensor(p["Wl"], requires_grad=True) if L else None
    t["sl"] = torch.tensor(p["sl"], requires_grad=True) if L else None
    Y = bench.torch_cascade(t["X"], t["W0"], t["b0"], t["s0"], t["Wl"], t["sl"])
    Yref = oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    np.testing.assert_allclose(Y.detach().numpy(), Yref, rtol=0, atol=1e-10)
    Y.backward(torch.tensor(p["dY"]))
    g = oracle.backward(p["X"], p["dY"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    pairs = [("dX", "X"), ("dW0", "W0"), ("db0", "b0"), ("ds0", "s0")] + ([("dWl", "Wl"), ("dsl", "sl")] if L else [])
    for gk, tk in pairs:
        np.testing.assert_allclose(t[tk].grad.numpy(), g[gk], rtol=0, atol=1e-10, err_msg=gk)
