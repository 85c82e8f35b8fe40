"""The same-GPU comparators of bench.py compute the layer: the plain
PyTorch cascade (any L) and the diagonalwise-refactorized conv (L = 0) give
the oracle's forward and every gradient in float64 on the CPU, so the times
and memory they report are those of the same computation."""
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


@pytest.mark.parametrize("C,block", [(64, 32), (40, 32), (7, 32), (5, 2), (3, 1)])
def test_diagonalwise_refactorization_matches_oracle_at_level_0(C, block):
    """L = 0 with channel counts that are and are not multiples of the block
    (the last block zero-padded); forward and the input, weight, bias and
    scale gradients."""
    p = as_float64(make_inputs(Workload("d", 2, C, 9, 7, 3, 0, "f32"), 5))
    t = {key: torch.tensor(p[key], requires_grad=True) for key in ("X", "W0", "b0", "s0")}
    Y = bench.diagonalwise_conv(t["X"], t["W0"], t["b0"], t["s0"], block=block)
    np.testing.assert_allclose(Y.detach().numpy(), oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], None, None),
                               rtol=0, atol=1e-10)
    Y.backward(torch.tensor(p["dY"]))
    g = oracle.backward(p["X"], p["dY"], p["W0"], p["b0"], p["s0"], None, None)
    for gk, tk in [("dX", "X"), ("dW0", "W0"), ("db0", "b0"), ("ds0", "s0")]:
        np.testing.assert_allclose(t[tk].grad.numpy(), g[gk], rtol=0, atol=1e-10, err_msg=gk)


def test_diagonalwise_weight_is_block_diagonal():
    """Each dense block weight holds channel c's kernel at (c, c) of its block
    and zeros off the diagonal: a kernel planted on one channel moves only
    that channel's output."""
    X = torch.randn(1, 6, 5, 5, dtype=torch.float64)
    W0 = torch.zeros(6, 3, 3, dtype=torch.float64)
    W0[4, 1, 1] = 1.0
    Y = bench.diagonalwise_conv(X, W0, torch.zeros(6, dtype=torch.float64), torch.ones(6, dtype=torch.float64),
                                block=4)
    assert torch.equal(Y[:, 4], X[:, 4])
    assert torch.count_nonzero(Y[:, [0, 1, 2, 3, 5]]) == 0
