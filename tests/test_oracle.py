"""Pins for the float64 oracle: each check ties it to something other than itself.

Sources: the layer as described in arXiv:2608.10805 (abstract: Haar analysis
butterfly, per-level depthwise convs and per-channel scales, multi-level
synthesis cascade, scaled base depthwise conv) and the mathematics of the
+-1/2 Haar transform.  None of these tests needs a GPU.
"""
import json
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from depthwise_convolution_wtconv_b200.configs import WORKLOADS, Workload
from depthwise_convolution_wtconv_b200.inputs import make_inputs, as_float64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng = np.random.default_rng(1234)


def _params(N=2, C=3, H=8, W=8, k=3, L=2, seed=0):
    wl = Workload("t", N, C, H, W, k, L, "f32")
    return as_float64(make_inputs(wl, seed))


# ---------------------------------------------------------------- Haar algebra

def test_haar_roundtrip_identity():
    A = rng.standard_normal((2, 3, 8, 12))
    np.testing.assert_allclose(oracle.haar_synthesis(oracle.haar_analysis(A)), A, rtol=0, atol=1e-14)
    B = rng.standard_normal((2, 3, 4, 4, 6))
    np.testing.assert_allclose(oracle.haar_analysis(oracle.haar_synthesis(B)), B, rtol=0, atol=1e-14)


def test_haar_parseval():
    A = rng.standard_normal((3, 10, 6))
    assert np.isclose(np.sum(oracle.haar_analysis(A) ** 2), np.sum(A ** 2), rtol=1e-13)


def test_haar_constant_input_has_no_detail():
    A = np.full((1, 1, 8, 8), 3.5)
    S = oracle.haar_analysis(A)
    assert np.all(S[:, :, 1:] == 0)
    assert np.all(S[:, :, 0] == 7.0)  # (4 * 3.5) / 2


def test_haar_single_block_by_hand():
    # block a=1 b=2 / c=3 d=4
    S = oracle.haar_analysis(np.array([[1.0, 2.0], [3.0, 4.0]]))
    assert S[:, 0, 0].tolist() == [5.0, -2.0, -1.0, 0.0]


def test_ll_chain_is_scaled_block_sum_bruteforce():
    """LL_l = 2^-l * (sum over the aligned 2^l x 2^l block), by explicit loops."""
    X = rng.standard_normal((1, 1, 16, 16))
    cur = X
    for l in range(1, 5):
        cur = oracle.haar_analysis(cur)[:, :, 0]
        b = 1 << l
        for i in range(16 // b):
            for j in range(16 // b):
                tot = 0.0
                for y in range(i * b, (i + 1) * b):
                    for x in range(j * b, (j + 1) * b):
                        tot += X[0, 0, y, x]
                assert abs(cur[0, 0, i, j] - tot / b) < 1e-12


# --------------------------------------------------------- depthwise conv pins

def _direct_dwconv_loops(X, W0):
    """Six nested loops: the textbook depthwise cross-correlation."""
    N, C, H, Wd = X.shape
    k = W0.shape[-1]
    r = k // 2
    out = np.zeros_like(X)
    for n in range(N):
        for c in range(C):
            for i in range(H):
                for j in range(Wd):
                    acc = 0.0
                    for u in range(k):
                        for v in range(k):
                            y, x = i + u - r, j + v - r
                            if 0 <= y < H and 0 <= x < Wd:
                                acc += W0[c, u, v] * X[n, c, y, x]
                    out[n, c, i, j] = acc
    return out


def test_level0_equals_bruteforce_loops():
    p = _params(N=2, C=3, H=6, W=7, k=5, L=0)
    Y = oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], None, None)
    ref = p["s0"][None, :, None, None] * (_direct_dwconv_loops(p["X"], p["W0"]) + p["b0"][None, :, None, None])
    np.testing.assert_allclose(Y, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("k", [1, 3, 5, 7])
def test_level0_equals_torch_conv2d(k):
    p = _params(N=2, C=4, H=9, W=10, k=k, L=0)
    Y = oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], None, None)
    Xt = torch.from_numpy(p["X"])
    ref = F.conv2d(Xt, torch.from_numpy(p["W0"]).unsqueeze(1), torch.from_numpy(p["b0"]), padding=k // 2, groups=4)
    ref = ref * torch.from_numpy(p["s0"]).view(1, -1, 1, 1)
    np.testing.assert_allclose(Y, ref.numpy(), rtol=0, atol=1e-12)


# ----------------------------------------------------------- golden by hand

def _load_golden():
    with open(os.path.join(GOLDEN, "hand_examples.json")) as f:
        return json.load(f)


def test_golden_level1_k1_forward_backward():
    g = _load_golden()["level1_k1"]
    a = {k: np.array(v, dtype=np.float64) for k, v in g.items() if not k.startswith("_") and k != "derivation"}
    Y = oracle.forward(a["X"], a["W0"], a["b0"], a["s0"], a["Wl"], a["sl"])
    np.testing.assert_array_equal(Y, a["Y"])
    gr = oracle.backward(a["X"], a["dY"], a["W0"], a["b0"], a["s0"], a["Wl"], a["sl"])
    for key in ("dX", "dW0", "db0", "ds0", "dWl", "dsl"):
        np.testing.assert_array_equal(gr[key], a[key], err_msg=key)


def test_golden_orientation_k3():
    g = _load_golden()["orientation_k3_L0"]
    a = {k: np.array(v, dtype=np.float64) for k, v in g.items() if k != "derivation"}
    Y = oracle.forward(a["X"], a["W0"], a["b0"], a["s0"], None, None)
    np.testing.assert_array_equal(Y, a["Y"])


# ------------------------------------------------------ delta-kernel closed form

def _block_mean(X, m):
    """U_m(X): mean over the aligned 2^m x 2^m block containing each pixel."""
    if m == 0:
        return X.copy()
    b = 1 << m
    N, C, H, W = X.shape
    means = X.reshape(N, C, H // b, b, W // b, b).mean(axis=(3, 5))
    return np.repeat(np.repeat(means, b, axis=2), b, axis=3)


@pytest.mark.parametrize("L", [1, 2, 3])
def test_delta_kernels_reproduce_scaled_block_means(L):
    """Delta kernels, b0 = 0, scales equal across a channel's 4 bands:
    Y = s0 X + sum_l s_l U_{l-1}(X)   (U_m = aligned 2^m block mean)."""
    N, C, H, W, k = 2, 3, 16, 16, 5
    X = rng.standard_normal((N, C, H, W))
    W0 = np.zeros((C, k, k)); W0[:, 2, 2] = 1.0
    Wl = np.zeros((L, C, 4, k, k)); Wl[:, :, :, 2, 2] = 1.0
    s0 = rng.uniform(0.5, 1.5, C)
    sc = rng.uniform(0.5, 1.5, (L, C))
    sl = np.repeat(sc[:, :, None], 4, axis=2)
    Y = oracle.forward(X, W0, np.zeros(C), s0, Wl, sl)
    ref = s0[None, :, None, None] * X
    for l in range(1, L + 1):
        ref = ref + sc[l - 1][None, :, None, None] * _block_mean(X, l - 1)
    np.testing.assert_allclose(Y, ref, rtol=0, atol=1e-12)


# Signs of the four Haar bands over a 2x2 block, indexed [row bit][col bit]:
# LL (a+b+c+d)/2, LH (a+b-c-d)/2, HL (a-b+c-d)/2, HH (a-b-c+d)/2.
_SIGMA = {0: ((1, 1), (1, 1)), 1: ((1, 1), (-1, -1)), 2: ((1, -1), (1, -1)), 3: ((1, -1), (-1, 1))}


def _single_band_delta_errors(level, band, H=32, W=32):
    """Max |oracle - hand-worked value| of Y, of the band's weight gradient
    and of its scale gradient, for one shifted delta kernel on one band of
    one level, everything else 0.

    Worked by hand from the layer's definition (Haar analysis, depthwise
    conv with scale, inverse cascade): the LL chain gives
    LL_m(p, q) = 2^-m * (sum of the aligned 2^m x 2^m block of X), so band s
    at level l is B(P, Q) = 1/2 sum_{a,b} sigma_s(a, b) LL_{l-1}(2P+a, 2Q+b);
    a delta at tap (r+du, r+dv) reads B(P+du, Q+dv) (zero outside); the level-l
    synthesis spreads c*B/2 with the band's signs over bit l-1 of the output
    coordinates, and every coarser-to-finer step after it halves it again:
        Y(i, j) = 2^-l * c * sigma_s(bit_{l-1} i, bit_{l-1} j) * B(i>>l + du, j>>l + dv).
    Y is linear in each tap, so the gradient of <Y, dY> in tap (u, v) is
        dW(u, v) = c * sum_{i,j} dY(i, j) 2^-l sigma_s(bits) B(i>>l + u-r, j>>l + v-r),
    and in the scale c it is dW(r+du, r+dv) / c; the input gradient is
        dX(i, j) = 2^-l * c * sigma_s(bits) * D(i>>l - du, j>>l - dv),
    D(P, Q) = sum over the level-l block (P, Q) of 2^-l sigma_s(bits) dY.
    Sides that are not
    multiples of 2^l take the zero-padded image in the block sums (the
    layer's reading for such sides) and only outputs inside the image.
    Computed here with plain loops, independent of the oracle's code."""
    N, C, k = 1, 2, 5
    r = k // 2
    du, dv = 1, -2
    L = level
    X = rng.standard_normal((N, C, H, W))
    dY = rng.standard_normal((N, C, H, W))
    c = np.array([0.75, 1.25])
    Wl = np.zeros((L, C, 4, k, k))
    Wl[level - 1, :, band, r + du, r + dv] = 1.0
    sl = rng.uniform(0.5, 1.5, (L, C, 4))
    sl[level - 1, :, band] = c
    W0, b0, s0 = np.zeros((C, k, k)), np.zeros(C), rng.uniform(0.5, 1.5, C)
    Y = oracle.forward(X, W0, b0, s0, Wl, sl)
    g = oracle.backward(X, dY, W0, b0, s0, Wl, sl)

    m = level - 1
    b = 1 << level
    Hp, Wp = -(-H // b) * b, -(-W // b) * b  # sides padded with zeros
    hb, wb = Hp >> level, Wp >> level
    sig = _SIGMA[band]
    ref = np.zeros_like(X)
    dx = np.zeros_like(X)
    dw = np.zeros((C, k, k))
    for ch in range(C):
        x = np.zeros((Hp, Wp))
        x[:H, :W] = X[0, ch]
        llm = np.zeros((Hp >> m, Wp >> m))
        for p in range(Hp >> m):
            for q in range(Wp >> m):
                llm[p, q] = x[p << m:(p + 1) << m, q << m:(q + 1) << m].sum() / 2 ** m
        B = np.zeros((hb, wb))
        for P in range(hb):
            for Q in range(wb):
                B[P, Q] = 0.5 * sum(sig[a][b] * llm[2 * P + a, 2 * Q + b] for a in (0, 1) for b in (0, 1))
        # D(P, Q): dY times the synthesis weight, summed over each level-l block
        D = np.zeros((hb, wb))
        for i in range(H):
            for j in range(W):
                s_ij = sig[(i >> m) & 1][(j >> m) & 1]
                D[i >> level, j >> level] += 2.0 ** -level * s_ij * dY[0, ch, i, j]
                P, Q = (i >> level) + du, (j >> level) + dv
                if 0 <= P < hb and 0 <= Q < wb:
                    ref[0, ch, i, j] = 2.0 ** -level * c[ch] * s_ij * B[P, Q]
        for i in range(H):
            for j in range(W):
                P, Q = (i >> level) - du, (j >> level) - dv
                if 0 <= P < hb and 0 <= Q < wb:
                    dx[0, ch, i, j] = 2.0 ** -level * c[ch] * sig[(i >> m) & 1][(j >> m) & 1] * D[P, Q]
        for u in range(k):
            for v in range(k):
                for P in range(hb):
                    for Q in range(wb):
                        if 0 <= P + u - r < hb and 0 <= Q + v - r < wb:
                            dw[ch, u, v] += c[ch] * D[P, Q] * B[P + u - r, Q + v - r]
    assert np.max(np.abs(ref)) > 0.1 and np.max(np.abs(dx)) > 0.01  # the shifted taps reach the band
    ds = dw[:, r + du, r + dv] / c
    return (float(np.max(np.abs(Y - ref))),
            float(np.max(np.abs(g["dWl"][level - 1, :, band] - dw))),
            float(np.max(np.abs(g["dsl"][level - 1, :, band] - ds))),
            float(np.max(np.abs(g["dX"] - dx))))


@pytest.mark.parametrize("level,band", [(2, 1), (2, 2), (2, 3), (3, 3), (3, 1), (1, 2)])
def test_single_band_shifted_delta_by_hand(level, band):
    ey, ew, es, ex = _single_band_delta_errors(level, band)
    assert ey < 1e-12 and ew < 1e-11 and es < 1e-11 and ex < 1e-12, (ey, ew, es, ex)


@pytest.mark.parametrize("level,band,H,W", [(2, 3, 30, 22), (3, 1, 28, 28), (3, 2, 27, 21), (1, 3, 17, 9)])
def test_single_band_shifted_delta_by_hand_ragged_sides(level, band, H, W):
    ey, ew, es, ex = _single_band_delta_errors(level, band, H, W)
    assert ey < 1e-12 and ew < 1e-11 and es < 1e-11 and ex < 1e-12, (ey, ew, es, ex)


def test_single_band_pin_catches_swapped_bands_and_transposed_kernel(monkeypatch):
    """The pin above fails on an oracle with LH and HL swapped in its
    analysis, with its depthwise kernels transposed, or with its
    weight-gradient correlation transposed."""
    good_analysis = oracle.wtconv_oracle.haar_analysis

    def swapped(A):
        S = good_analysis(A)
        return S[..., [0, 2, 1, 3], :, :]
    monkeypatch.setattr(oracle.wtconv_oracle, "haar_analysis", swapped)
    assert _single_band_delta_errors(2, 1)[0] > 1e-3
    monkeypatch.setattr(oracle.wtconv_oracle, "haar_analysis", good_analysis)
    assert _single_band_delta_errors(2, 1)[0] < 1e-12

    good_conv = oracle.wtconv_oracle.dwconv
    monkeypatch.setattr(oracle.wtconv_oracle, "dwconv", lambda A, Wt: good_conv(A, np.swapaxes(Wt, -1, -2)))
    ey, _, _, ex = _single_band_delta_errors(3, 3)
    assert ey > 1e-3 and ex > 1e-3
    monkeypatch.setattr(oracle.wtconv_oracle, "dwconv", good_conv)

    good_corr = oracle.wtconv_oracle.dwcorr_weight
    monkeypatch.setattr(oracle.wtconv_oracle, "dwcorr_weight",
                        lambda A, G, k: np.swapaxes(good_corr(A, G, k), -1, -2))
    ey, ew, es, _ = _single_band_delta_errors(2, 3)
    # the oracle's scale gradient does not go through the tap correlation
    assert ey < 1e-12 and ew > 1e-3 and es < 1e-11


def test_delta_unit_scales_level1_doubles_input():
    X = rng.standard_normal((1, 2, 8, 8))
    W0 = np.zeros((2, 3, 3)); W0[:, 1, 1] = 1
    Wl = np.zeros((1, 2, 4, 3, 3)); Wl[..., 1, 1] = 1
    Y = oracle.forward(X, W0, np.zeros(2), np.ones(2), Wl, np.ones((1, 2, 4)))
    np.testing.assert_allclose(Y, 2 * X, rtol=0, atol=1e-13)


# ------------------------------------------------ reformulations are algebraic

@pytest.mark.parametrize("L", [1, 2, 3])
def test_closed_form_analysis_equals_cascade(L):
    X = rng.standard_normal((2, 2, 16, 16))
    cur = X
    for l in range(1, L + 1):
        sub = oracle.haar_analysis(cur)
        np.testing.assert_allclose(oracle.analysis_closed_form(X, l), sub, rtol=0, atol=1e-12)
        cur = sub[:, :, 0]


@pytest.mark.parametrize("L", [1, 2, 4])
def test_closed_form_synthesis_equals_cascade(L):
    p = _params(N=1, C=2, H=16, W=16, k=3, L=L)
    Y = oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    base = oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], None, None)
    Zs = oracle.level_outputs(p["X"], p["Wl"], p["sl"])
    np.testing.assert_allclose(base + oracle.synthesis_closed_form(Zs, 16, 16), Y, rtol=0, atol=1e-12)


def test_scale_folding_equals_unfolded():
    """s * dwconv(x, W) == dwconv(x, s * W)   (reformulation (3))."""
    p = _params(N=1, C=3, H=8, W=8, k=5, L=2)
    Y = oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    Wf = p["Wl"] * p["sl"][..., None, None]
    W0f = p["W0"] * p["s0"][:, None, None]
    Y2 = oracle.forward(p["X"], W0f, p["b0"] * p["s0"], np.ones(3), Wf, np.ones_like(p["sl"]))
    np.testing.assert_allclose(Y2, Y, rtol=0, atol=1e-12)


# ----------------------------------- independent composition in torch + autograd

def torch_wtconv(X, W0, b0, s0, Wl, sl):
    """The layer composed from library routines: grouped conv2d for the
    depthwise convs, a stride-2 grouped conv2d for the Haar analysis and
    conv_transpose2d for the synthesis.  Differentiated by autograd."""
    C = X.shape[1]
    k = W0.shape[-1]
    L = 0 if Wl is None else Wl.shape[0]
    h = 0.5
    filt = torch.tensor([[[h, h], [h, h]], [[h, h], [-h, -h]], [[h, -h], [h, -h]], [[h, -h], [-h, h]]],
                        dtype=X.dtype)
    filt = filt.repeat(C, 1, 1).unsqueeze(1)  # [4C, 1, 2, 2], channel 4c+s
    Y = s0.view(1, C, 1, 1) * F.conv2d(X, W0.unsqueeze(1), b0, padding=k // 2, groups=C)
    cur = X
    Zs = []
    for l in range(L):
        sub = F.conv2d(cur, filt, stride=2, groups=C)                        # [N, 4C, h, w]
        Z = F.conv2d(sub, Wl[l].reshape(4 * C, 1, k, k), padding=k // 2, groups=4 * C)
        Zs.append(Z * sl[l].reshape(1, 4 * C, 1, 1))
        cur = sub[:, 0::4]
    t = None
    for l in reversed(range(L)):
        Z = Zs[l]
        if t is not None:
            Z = Z.clone()
            Z[:, 0::4] = Z[:, 0::4] + t
        t = F.conv_transpose2d(Z, filt, stride=2, groups=C)
    return Y if t is None else Y + t


@pytest.mark.parametrize("shape", [(2, 3, 16, 16, 5, 2), (1, 4, 8, 12, 3, 1), (2, 2, 16, 8, 3, 3), (1, 2, 6, 6, 3, 0)])
def test_torch_composition_matches_forward_and_all_gradients(shape):
    N, C, H, W, k, L = shape
    p = _params(N, C, H, W, k, L, seed=3)
    t = {key: (None if v is None else torch.tensor(v, requires_grad=True)) for key, v in p.items()}
    Yt = torch_wtconv(t["X"], t["W0"], t["b0"], t["s0"], t["Wl"], t["sl"])
    Y = oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    np.testing.assert_allclose(Y, Yt.detach().numpy(), rtol=0, atol=1e-10)
    (Yt * torch.from_numpy(p["dY"])).sum().backward()
    g = oracle.backward(p["X"], p["dY"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    names = [("dX", "X"), ("dW0", "W0"), ("db0", "b0"), ("ds0", "s0")]
    if L:
        names += [("dWl", "Wl"), ("dsl", "sl")]
    for gk, tk in names:
        np.testing.assert_allclose(g[gk], t[tk].grad.numpy(), rtol=0, atol=1e-10, err_msg=gk)


# --------------------------------------------------------- finite differences

def test_finite_differences_tiny_workload():
    wl = WORKLOADS["tiny_k5_L2"]
    p = as_float64(make_inputs(wl, 0))
    g = oracle.backward(p["X"], p["dY"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    h = 1e-6
    fd_rng = np.random.default_rng(7)
    pairs = [("X", "dX"), ("W0", "dW0"), ("b0", "db0"), ("s0", "ds0"), ("Wl", "dWl"), ("sl", "dsl")]

    def loss(q):
        return float(np.sum(oracle.forward(q["X"], q["W0"], q["b0"], q["s0"], q["Wl"], q["sl"]) * p["dY"]))

    for name, gname in pairs:
        flat = p[name].reshape(-1)
        for idx in fd_rng.choice(flat.size, size=min(6, flat.size), replace=False):
            q = {key: (None if v is None else v.copy()) for key, v in p.items()}
            q[name].reshape(-1)[idx] += h
            lp = loss(q)
            q[name].reshape(-1)[idx] -= 2 * h
            lm = loss(q)
            fd = (lp - lm) / (2 * h)
            an = g[gname].reshape(-1)[idx]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, idx, fd, an)


# ------------------------------------------------------- exact linearity tests

def test_adjoint_dot_product():
    """<Y(X) - Y(0), dY> == <X, dX(dY)>: Y is affine in X."""
    p = _params(N=2, C=3, H=16, W=16, k=5, L=3, seed=5)
    Y = oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    Y0 = oracle.forward(np.zeros_like(p["X"]), p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    dX = oracle.backward(p["X"], p["dY"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])["dX"]
    lhs = np.sum((Y - Y0) * p["dY"])
    rhs = np.sum(p["X"] * dX)
    assert abs(lhs - rhs) < 1e-10 * max(1.0, abs(lhs))


@pytest.mark.parametrize("which", ["W0", "Wl"])
def test_weight_gradient_linearity(which):
    """Y is affine in each weight tensor: <dW, V> == <Y(W+V) - Y(W), dY>."""
    p = _params(N=2, C=2, H=8, W=8, k=3, L=2, seed=9)
    V = np.random.default_rng(3).standard_normal(p[which].shape)
    g = oracle.backward(p["X"], p["dY"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    q = dict(p)
    q[which] = p[which] + V
    Y1 = oracle.forward(q["X"], q["W0"], q["b0"], q["s0"], q["Wl"], q["sl"])
    Y0 = oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    lhs = np.sum(g["d" + which] * V)
    rhs = np.sum((Y1 - Y0) * p["dY"])
    assert abs(lhs - rhs) < 1e-10 * max(1.0, abs(rhs))


# --------------------------------------------- planted mistakes are caught

def _compose_mismatch(monkeypatch, target, fn):
    monkeypatch.setattr(oracle.wtconv_oracle, target, fn)
    p = _params(2, 3, 16, 16, 3, 2, seed=11)
    t = {key: torch.tensor(v) for key, v in p.items()}
    Yt = torch_wtconv(t["X"], t["W0"], t["b0"], t["s0"], t["Wl"], t["sl"]).numpy()
    Y = oracle.wtconv_oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    return np.max(np.abs(Y - Yt))


def test_planted_sign_error_is_caught(monkeypatch):
    good = oracle.wtconv_oracle.haar_analysis

    def bad(A):
        S = good(A)
        S[..., 2, :, :] *= -1.0  # wrong sign on HL
        return S
    assert _compose_mismatch(monkeypatch, "haar_analysis", bad) > 1e-3


def test_planted_transposed_kernel_is_caught(monkeypatch):
    good = oracle.wtconv_oracle.dwconv

    def bad(A, Wt):
        return good(A, np.swapaxes(Wt, -1, -2))
    assert _compose_mismatch(monkeypatch, "dwconv", bad) > 1e-3


def test_planted_wrong_synthesis_is_caught(monkeypatch):
    good = oracle.wtconv_oracle.haar_synthesis

    def bad(S):
        S = S.copy()
        S[..., [1, 2], :, :] = S[..., [2, 1], :, :]  # LH and HL swapped
        return good(S)
    assert _compose_mismatch(monkeypatch, "haar_synthesis", bad) > 1e-3


# ---------------------------------------------------- regression fixture

def test_regression_fixture_tiny_workload():
    path = os.path.join(GOLDEN, "tiny_k5_L2_seed0.json")
    with open(path) as f:
        ref = json.load(f)
    wl = WORKLOADS["tiny_k5_L2"]
    p = as_float64(make_inputs(wl, 0))
    Y = oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    g = oracle.backward(p["X"], p["dY"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    outs = dict(Y=Y, **g)
    for key, entry in ref["tensors"].items():
        arr = outs[key].reshape(-1)
        np.testing.assert_allclose(arr[entry["index"]], entry["value"], rtol=1e-12, atol=1e-12, err_msg=key)
        assert abs(float(np.sum(arr)) - entry["sum"]) <= 1e-9 * max(1.0, abs(entry["sum"]))


# ------------------------------------------- sides not multiples of 2^L
# The pages are silent on such sides; the oracle pads each level's plane to
# even sides with zeros (bottom, right) and crops each level's synthesis back.

RAGGED = [(2, 3, 13, 11, 5, 2), (1, 2, 7, 9, 3, 3), (2, 2, 5, 6, 3, 1), (1, 3, 9, 14, 1, 2), (1, 2, 3, 3, 3, 3)]


def torch_wtconv_ragged(X, W0, b0, s0, Wl, sl):
    """The layer with per-level padding composed from library routines
    (F.pad, grouped conv2d, conv_transpose2d and slicing), differentiated by
    autograd."""
    C = X.shape[1]
    k = W0.shape[-1]
    L = 0 if Wl is None else Wl.shape[0]
    h = 0.5
    filt = torch.tensor([[[h, h], [h, h]], [[h, h], [-h, -h]], [[h, -h], [h, -h]], [[h, -h], [-h, h]]],
                        dtype=X.dtype).repeat(C, 1, 1).unsqueeze(1)
    Y = s0.view(1, C, 1, 1) * F.conv2d(X, W0.unsqueeze(1), b0, padding=k // 2, groups=C)
    cur, Zs, sizes = X, [], []
    for l in range(L):
        H, W = cur.shape[-2:]
        sizes.append((H, W))
        sub = F.conv2d(F.pad(cur, (0, W % 2, 0, H % 2)), filt, stride=2, groups=C)
        Zs.append(F.conv2d(sub, Wl[l].reshape(4 * C, 1, k, k), padding=k // 2, groups=4 * C)
                  * sl[l].reshape(1, 4 * C, 1, 1))
        cur = sub[:, 0::4]
    t = None
    for l in reversed(range(L)):
        Z = Zs[l]
        if t is not None:
            Z = Z.clone()
            Z[:, 0::4] = Z[:, 0::4] + t
        H, W = sizes[l]
        t = F.conv_transpose2d(Z, filt, stride=2, groups=C)[..., :H, :W]
    return Y if t is None else Y + t


@pytest.mark.parametrize("shape", RAGGED)
def test_ragged_torch_composition_matches_forward_and_all_gradients(shape):
    N, C, H, W, k, L = shape
    p = _params(N, C, H, W, k, L, seed=11)
    t = {key: (None if v is None else torch.tensor(v, requires_grad=True)) for key, v in p.items()}
    Yt = torch_wtconv_ragged(t["X"], t["W0"], t["b0"], t["s0"], t["Wl"], t["sl"])
    Y = oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    assert Y.shape == (N, C, H, W)
    np.testing.assert_allclose(Y, Yt.detach().numpy(), rtol=0, atol=1e-10)
    (Yt * torch.from_numpy(p["dY"])).sum().backward()
    g = oracle.backward(p["X"], p["dY"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    for gk, tk in [("dX", "X"), ("dW0", "W0"), ("db0", "b0"), ("ds0", "s0"), ("dWl", "Wl"), ("dsl", "sl")]:
        np.testing.assert_allclose(g[gk], t[tk].grad.numpy(), rtol=0, atol=1e-10, err_msg=gk)


@pytest.mark.parametrize("shape", [(2, 3, 13, 11), (1, 2, 7, 5), (1, 1, 3, 9)])
def test_ragged_delta_kernels_reproduce_zero_padded_block_means(shape):
    """Delta kernels, b0 = 0, equal band scales: Y = s0 X + sum_l s_l U_{l-1}(X)
    with U_m the mean over the aligned 2^m x 2^m block, pixels outside the
    image counting as zeros (brute force over each block)."""
    N, C, H, W = shape
    L, k = 3, 3
    X = rng.standard_normal((N, C, H, W))
    W0 = np.zeros((C, k, k)); W0[:, 1, 1] = 1.0
    Wl = np.zeros((L, C, 4, k, k)); Wl[:, :, :, 1, 1] = 1.0
    s0 = rng.uniform(0.5, 1.5, C)
    sc = rng.uniform(0.5, 1.5, (L, C))
    Y = oracle.forward(X, W0, np.zeros(C), s0, Wl, np.repeat(sc[:, :, None], 4, axis=2))
    ref = s0[None, :, None, None] * X
    for l in range(1, L + 1):
        b = 1 << (l - 1)
        U = np.zeros_like(X)
        for i in range(H):
            for j in range(W):
                i0, j0 = i // b * b, j // b * b
                U[:, :, i, j] = X[:, :, i0:i0 + b, j0:j0 + b].sum(axis=(2, 3)) / (b * b)
        ref = ref + sc[l - 1][None, :, None, None] * U
    np.testing.assert_allclose(Y, ref, rtol=0, atol=1e-12)


def test_ragged_adjoint_dot_product_and_finite_differences():
    p = _params(N=2, C=2, H=11, W=7, k=3, L=2, seed=13)
    Y = oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    Y0 = oracle.forward(np.zeros_like(p["X"]), p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    g = oracle.backward(p["X"], p["dY"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    lhs, rhs = np.sum((Y - Y0) * p["dY"]), np.sum(p["X"] * g["dX"])
    assert abs(lhs - rhs) < 1e-10 * max(1.0, abs(lhs))

    def loss(q):
        return float(np.sum(oracle.forward(q["X"], q["W0"], q["b0"], q["s0"], q["Wl"], q["sl"]) * p["dY"]))

    h = 1e-6
    fd_rng = np.random.default_rng(17)
    for name, gname in [("X", "dX"), ("W0", "dW0"), ("s0", "ds0"), ("Wl", "dWl"), ("sl", "dsl")]:
        flat = p[name].reshape(-1)
        for idx in fd_rng.choice(flat.size, size=min(4, flat.size), replace=False):
            q = {key: (None if v is None else v.copy()) for key, v in p.items()}
            q[name].reshape(-1)[idx] += h
            lp = loss(q)
            q[name].reshape(-1)[idx] -= 2 * h
            fd = (lp - loss(q)) / (2 * h)
            an = g[gname].reshape(-1)[idx]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, idx, fd, an)


@pytest.mark.parametrize("shape", RAGGED)
def test_ragged_equals_one_padding_to_multiples_of_2L(shape):
    """Zero-padding X once to multiples of 2^L (bottom, right), running the
    layer on the padded planes and cropping gives the per-level reading's
    output; dY zero-padded the same way gives its gradients (dX cropped).
    This is how the CUDA library computes such sides."""
    N, C, H, W, k, L = shape
    p = _params(N, C, H, W, k, L, seed=19)
    m = 1 << L
    Hp, Wp = -(-H // m) * m, -(-W // m) * m
    pad = lambda A: np.pad(A, [(0, 0), (0, 0), (0, Hp - H), (0, Wp - W)])
    Y = oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    Yp = oracle.forward(pad(p["X"]), p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    np.testing.assert_allclose(Yp[:, :, :H, :W], Y, rtol=0, atol=1e-12)
    g = oracle.backward(p["X"], p["dY"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    gp = oracle.backward(pad(p["X"]), pad(p["dY"]), p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    np.testing.assert_allclose(gp["dX"][:, :, :H, :W], g["dX"], rtol=0, atol=1e-12)
    for key in ("dW0", "db0", "ds0", "dWl", "dsl"):
        np.testing.assert_allclose(gp[key], g[key], rtol=0, atol=1e-11, err_msg=key)
