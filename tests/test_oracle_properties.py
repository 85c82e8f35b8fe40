"""Property sweep of the float64 oracle over random small shapes.

The layer (arXiv:2608.10805, abstract: Haar analysis, per-level depthwise
convs with per-channel scales, synthesis cascade, scaled base conv) is, as a
function of each of X, W0, b0, s0, Wl and sl with the others fixed, linear
plus a part that does not depend on it.  So for every parameter p, with
F(p) = <Y(p), dY>:  <p, dF/dp> = F(p) - F(0) exactly (Euler's identity for
a degree-1 function; for X this is the adjoint dot-product test).  The
right side uses the forward pass only, so each identity ties the oracle's
hand-derived backward to its forward on any shape: odd and tiny sides, every
kernel size, up to three levels.  None of this needs a GPU.
"""
import numpy as np
from hypothesis import given, settings, strategies as st

import oracle


@st.composite
def layer_case(draw):
    N = draw(st.integers(1, 2))
    C = draw(st.integers(1, 3))
    H = draw(st.integers(1, 19))
    W = draw(st.integers(1, 19))
    k = draw(st.sampled_from([1, 3, 5, 7]))
    L = draw(st.integers(0, 3))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    return N, C, H, W, k, L, seed


def _euler_errors(case):
    """Per parameter, |<p, dF/dp> - (F(p) - F(0))| over its scale."""
    N, C, H, W, k, L, seed = case
    g = np.random.default_rng(seed)
    p = dict(X=g.standard_normal((N, C, H, W)), W0=g.standard_normal((C, k, k)) / k,
             b0=g.standard_normal(C) * 0.1, s0=g.uniform(0.5, 1.5, C),
             Wl=g.standard_normal((L, C, 4, k, k)) / k if L else None,
             sl=g.uniform(0.5, 1.5, (L, C, 4)) if L else None)
    dY = g.standard_normal((N, C, H, W))

    def F(**over):
        q = dict(p, **over)
        Y = oracle.forward(q["X"], q["W0"], q["b0"], q["s0"], q["Wl"], q["sl"])
        assert Y.shape == (N, C, H, W)
        return float(np.sum(Y * dY))

    grads = oracle.backward(p["X"], dY, p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    pairs = [("X", "dX"), ("W0", "dW0"), ("b0", "db0"), ("s0", "ds0")]
    if L:
        pairs += [("Wl", "dWl"), ("sl", "dsl")]
    F_all = F()
    err = {}
    for name, gname in pairs:
        assert grads[gname].shape == p[name].shape, gname
        lhs = float(np.sum(p[name] * grads[gname]))
        rhs = F_all - F(**{name: np.zeros_like(p[name])})
        scale = 1.0 + abs(lhs) + abs(rhs) + float(np.sum(np.abs(p[name] * grads[gname])))
        err[name] = abs(lhs - rhs) / scale
    return err


@settings(max_examples=150, deadline=None, derandomize=True)
@given(layer_case())
def test_every_gradient_satisfies_eulers_identity(case):
    err = _euler_errors(case)
    assert max(err.values()) <= 1e-11, (case, err)


def test_euler_identity_catches_a_planted_adjoint_mistake(monkeypatch):
    """A transposed weight-gradient correlation in the oracle breaks the
    identity for W0 and Wl and leaves the others intact."""
    good = oracle.wtconv_oracle.dwcorr_weight
    monkeypatch.setattr(oracle.wtconv_oracle, "dwcorr_weight", lambda A, G, k: np.swapaxes(good(A, G, k), -1, -2))
    err = _euler_errors((1, 2, 11, 9, 5, 2, 7))
    assert err["W0"] > 1e-3 and err["Wl"] > 1e-3
    assert err["X"] <= 1e-11 and err["b0"] <= 1e-11


@settings(max_examples=60, deadline=None, derandomize=True)
@given(layer_case())
def test_forward_and_gradients_equal_torch_composition_on_random_shapes(case):
    """The oracle against the layer composed from library routines (per-level
    F.pad, grouped conv2d, conv_transpose2d, cropping; autograd for the
    gradients) on the same random shape and values."""
    import torch
    from test_oracle import torch_wtconv_ragged

    N, C, H, W, k, L, seed = case
    g = np.random.default_rng(seed)
    p = dict(X=g.standard_normal((N, C, H, W)), W0=g.standard_normal((C, k, k)) / k,
             b0=g.standard_normal(C) * 0.1, s0=g.uniform(0.5, 1.5, C),
             Wl=g.standard_normal((L, C, 4, k, k)) / k if L else None,
             sl=g.uniform(0.5, 1.5, (L, C, 4)) if L else None)
    dY = g.standard_normal((N, C, H, W))
    t = {key: (None if v is None else torch.tensor(v, requires_grad=True)) for key, v in p.items()}
    Yt = torch_wtconv_ragged(t["X"], t["W0"], t["b0"], t["s0"], t["Wl"], t["sl"])
    Yt.backward(torch.tensor(dY))
    Y = oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    np.testing.assert_allclose(Y, Yt.detach().numpy(), rtol=0, atol=1e-12 * (1 + np.abs(Y).max()))
    gr = oracle.backward(p["X"], dY, p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    for name, gname in (("X", "dX"), ("W0", "dW0"), ("b0", "db0"), ("s0", "ds0"), ("Wl", "dWl"), ("sl", "dsl")):
        if t[name] is None:
            continue
        want = t[name].grad.numpy()
        np.testing.assert_allclose(gr[gname], want, rtol=0, atol=1e-11 * (1 + np.abs(want).max()), err_msg=gname)
