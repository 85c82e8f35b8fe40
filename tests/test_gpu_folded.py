"""The folded-weight entry points (scales folded once, then data passes
without the folding launch): the forward over a forward block equals
wtconv_forward bit for bit, the forward over an adjoint block equals
wtconv_backward_data bit for bit, and both match the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import depthwise_convolution_wtconv_b200 as wt
from depthwise_convolution_wtconv_b200.configs import Workload
from depthwise_convolution_wtconv_b200.inputs import make_inputs, as_float64

pytestmark = pytest.mark.gpu

CASES = [
    Workload("tiny_L2", 1, 8, 16, 16, 5, 2, "f32"),
    Workload("whole_L3", 2, 6, 56, 56, 5, 3, "f32"),
    Workload("whole_L2_bf16", 3, 4, 28, 28, 5, 2, "bf16"),
    Workload("bands_deep_L3_k7", 2, 2, 256, 128, 7, 3, "f32"),
    Workload("bands_deep_L5_bf16", 1, 2, 256, 256, 3, 5, "bf16"),
    Workload("rows_L0_k3", 2, 3, 112, 112, 3, 0, "f32"),
    Workload("small_L0_k5", 4, 5, 14, 14, 5, 0, "f32"),
    Workload("L1_k1", 2, 3, 16, 12, 1, 1, "f32"),
    Workload("ragged_L2", 2, 3, 13, 11, 5, 2, "f32"),
    Workload("recursive_512_L2", 1, 2, 512, 512, 3, 2, "f32"),
]


def _dev(inp, io):
    dt = torch.float32 if io == "f32" else torch.bfloat16
    d = {k: (v.to(dt) if k in ("X", "dY") else v).cuda().contiguous() for k, v in inp.items()}
    if d["Wl"].numel() == 0:
        d["Wl"] = d["sl"] = None
    return d


@pytest.mark.parametrize("wl", CASES, ids=[c.name for c in CASES])
def test_folded_passes_equal_the_unfolded_ones(cuda_ok, wl):
    inp = make_inputs(wl, 3)
    d = _dev(inp, wl.io)
    fw = wt.fold_weights(d["W0"], d["b0"], d["s0"], d["Wl"], d["sl"])
    ad = wt.fold_weights(d["W0"], None, d["s0"], d["Wl"], d["sl"], adjoint=True)
    y_ref = wt.forward(d["X"], d["W0"], d["b0"], d["s0"], d["Wl"], d["sl"])
    dx_ref = wt.backward_data(d["dY"], d["W0"], d["s0"], d["Wl"], d["sl"])
    y = wt.forward_folded(d["X"], fw, wl.k, wl.L)
    dx = wt.forward_folded(d["dY"], ad, wl.k, wl.L)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    assert torch.equal(dx, dx_ref)
    # and against the oracle (fp32 1e-4, bf16 2e-2 of the max-abs)
    p = as_float64(inp)
    Y = oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    tol = 1e-4 if wl.io == "f32" else 2e-2
    err = np.max(np.abs(y.float().cpu().numpy().astype(np.float64) - Y)) / np.max(np.abs(Y))
    assert err <= tol, err


def test_one_block_serves_every_batch(cuda_ok):
    """A block depends on the parameters only: the same block gives the
    forward of batches of different sizes and plane shapes."""
    small = Workload("a", 2, 4, 32, 32, 5, 2, "f32")
    inp = make_inputs(small, 5)
    d = _dev(inp, "f32")
    fw = wt.fold_weights(d["W0"], d["b0"], d["s0"], d["Wl"], d["sl"])
    for N, H, W in ((1, 16, 16), (5, 64, 48), (3, 256, 192)):
        x = torch.randn(N, 4, H, W, device="cuda", generator=torch.Generator("cuda").manual_seed(N))
        y = wt.forward_folded(x, fw, 5, 2)
        assert torch.equal(y, wt.forward(x, d["W0"], d["b0"], d["s0"], d["Wl"], d["sl"]))
