"""Plain float64 CPU oracle for the WTConv layer (test infrastructure only).

This module is the yardstick the CUDA library is checked against.  Only the
tests, the smoke check and the benchmark's CPU-baseline leg may import it; the
library itself never does, and this module imports nothing from the library.

What it computes (the plain, unfused definition of the layer):

  Source: "I/O-aware reformulation of wavelet convolution (WTConv)",
  arXiv:2608.10805, abstract -- the layer is a multi-level Haar wavelet
  decomposition with a per-channel depthwise convolution and a learned
  per-channel scale on every subband, followed by the multi-level synthesis
  cascade, added to a scaled base depthwise convolution.

  * Haar analysis of one 2x2 block (a, b / c, d) with taps +-1/2:
        LL = (a+b+c+d)/2   LH = (a+b-c-d)/2   HL = (a-b+c-d)/2   HH = (a-b-c+d)/2
    (a = (2i,2j), b = (2i,2j+1), c = (2i+1,2j), d = (2i+1,2j+1)).
  * dwconv(A, W)[c,i,j] = sum_{u,v<k} W[c,u,v] * A[c, i+u-r, j+v-r]
    (cross-correlation, zero 'same' padding, r = (k-1)/2).
  * Ybase = s0 * (dwconv(X, W0) + b0)
  * cur = X; for l = 1..L: sub_l = Haar(cur) (4 bands per input channel,
    channel order 4c+s); Z_l = s_l * dwconv(sub_l, W_l); cur = raw LL band.
  * t = 0; for l = L..1: t = IWT(Z_l with t added to its LL band)
  * Y = Ybase + t

Planes whose sides are not divisible by 2^L: the pages are silent.  Reading
taken here: at every level the plane entering the analysis (X, then the raw
LL band) gets one zero row at the bottom and / or one zero column at the
right when that side is odd, and the synthesis output of that level is
cropped back to the size the plane had before the padding.  With even sides
throughout this is the plain definition above.

The backward pass is the hand-derived adjoint of those steps in reverse order
(IWT^T = Haar and Haar^T = IWT because the +-1/2 Haar is orthonormal;
dwconv^T is the correlation with the spatially flipped kernel).

Closed forms used as cross-checks of the reformulations on the same page:
analysis_closed_form (reformulation (1): every subband is a fixed linear map
of X) and synthesis_closed_form (reformulation (2): one pass over output
pixels indexed by the bits of the output coordinates).

All arrays are numpy float64.  Shapes:
  X, Y, dY, dX : [N, C, H, W]
  W0 : [C, k, k]   b0, s0 : [C]
  Wl : [L, C, 4, k, k]   sl : [L, C, 4]     (band order LL, LH, HL, HH)
"""
import numpy as np

BANDS = ("LL", "LH", "HL", "HH")

# sign of band s at block position (py, px): SIGN[s, py, px]
SIGN = np.array(
    [
        [[1, 1], [1, 1]],      # LL
        [[1, 1], [-1, -1]],    # LH: (-1)^py
        [[1, -1], [1, -1]],    # HL: (-1)^px
        [[1, -1], [-1, 1]],    # HH: (-1)^(py+px)
    ],
    dtype=np.float64,
)


def haar_analysis(A):
    """One level of the 2-D Haar analysis with +-1/2 taps.

    A [..., 2h, 2w] -> [..., 4, h, w] with bands (LL, LH, HL, HH).
    Source: arXiv:2608.10805 abstract, "Haar analysis butterfly".
    """
    a = A[..., 0::2, 0::2]
    b = A[..., 0::2, 1::2]
    c = A[..., 1::2, 0::2]
    d = A[..., 1::2, 1::2]
    LL = (a + b + c + d) / 2.0
    LH = (a + b - c - d) / 2.0
    HL = (a - b + c - d) / 2.0
    HH = (a - b - c + d) / 2.0
    return np.stack([LL, LH, HL, HH], axis=-3)


def haar_synthesis(S):
    """Inverse of haar_analysis: [..., 4, h, w] -> [..., 2h, 2w]."""
    LL, LH, HL, HH = S[..., 0, :, :], S[..., 1, :, :], S[..., 2, :, :], S[..., 3, :, :]
    h, w = LL.shape[-2:]
    out = np.zeros(LL.shape[:-2] + (2 * h, 2 * w), dtype=np.float64)
    out[..., 0::2, 0::2] = (LL + LH + HL + HH) / 2.0
    out[..., 0::2, 1::2] = (LL + LH - HL - HH) / 2.0
    out[..., 1::2, 0::2] = (LL - LH + HL - HH) / 2.0
    out[..., 1::2, 1::2] = (LL - LH - HL + HH) / 2.0
    return out


def dwconv(A, Wt):
    """Depthwise k x k cross-correlation with zero 'same' padding.

    A [..., h, w]; Wt [..., k, k] whose leading dims broadcast against A's
    leading dims (one kernel per channel).  Loops over the k*k taps.
    """
    k = Wt.shape[-1]
    r = k // 2
    h, w = A.shape[-2:]
    pad = [(0, 0)] * (A.ndim - 2) + [(r, r), (r, r)]
    P = np.pad(A, pad)
    out = np.zeros(np.broadcast_shapes(A.shape[:-2], Wt.shape[:-2]) + (h, w), dtype=np.float64)
    for u in range(k):
        for v in range(k):
            out += Wt[..., u, v][..., None, None] * P[..., u:u + h, v:v + w]
    return out


def dwcorr_weight(A, G, k):
    """Per-tap correlation sum_{n,i,j} G[n,...,i,j] * A[n,...,i+u-r,j+v-r].

    The gradient of sum(G * dwconv(A, Wt)) with respect to Wt; the sum runs
    over the batch axis (axis 0) and the two spatial axes.
    Returns [..., k, k] with the batch axis removed.
    """
    r = k // 2
    h, w = A.shape[-2:]
    pad = [(0, 0)] * (A.ndim - 2) + [(r, r), (r, r)]
    P = np.pad(A, pad)
    out = np.zeros(A.shape[1:-2] + (k, k), dtype=np.float64)
    for u in range(k):
        for v in range(k):
            out[..., u, v] = np.sum(G * P[..., u:u + h, v:v + w], axis=(0, -2, -1))
    return out


def _check(X, W0, Wl, L):
    N, C, H, W = X.shape
    k = W0.shape[-1]
    assert k % 2 == 1 and W0.shape == (C, k, k)
    if L:
        assert Wl.shape == (L, C, 4, k, k)


def pad_even(A):
    """Zero row at the bottom / zero column at the right of the last two
    axes where that side is odd (the plane entering one analysis level)."""
    h, w = A.shape[-2:]
    pad = [(0, 0)] * (A.ndim - 2) + [(0, h % 2), (0, w % 2)]
    return np.pad(A, pad)


def crop(A, shape):
    """The top-left shape[0] x shape[1] corner of the last two axes."""
    return A[..., :shape[0], :shape[1]]


def forward(X, W0, b0, s0, Wl, sl, return_intermediates=False):
    """Forward pass of the layer, as the unfused cascade.

    Source: arXiv:2608.10805 abstract (multi-level decomposition, per-channel
    scales, multi-level synthesis cascade); base branch is the scaled
    depthwise convolution with bias, s0 * (dwconv(X, W0) + b0).
    """
    L = 0 if Wl is None else Wl.shape[0]
    _check(X, W0, Wl, L)
    base_pre = dwconv(X, W0[None]) + b0[None, :, None, None]
    Y = s0[None, :, None, None] * base_pre
    subs, convs, shapes = [], [], []
    cur = X
    for l in range(L):
        shapes.append(cur.shape[-2:])            # size before this level's padding
        sub = haar_analysis(pad_even(cur))       # [N, C, 4, h, w]
        conv = dwconv(sub, Wl[l][None])          # unscaled level conv
        subs.append(sub)
        convs.append(conv)
        cur = sub[:, :, 0]                       # raw LL goes one level deeper
    t = None
    for l in reversed(range(L)):
        Z = sl[l][None, :, :, None, None] * convs[l]
        if t is not None:
            Z = Z.copy()
            Z[:, :, 0] += t
        t = crop(haar_synthesis(Z), shapes[l])
    if t is not None:
        Y = Y + t
    if return_intermediates:
        return Y, dict(base_pre=base_pre, subs=subs, convs=convs, shapes=shapes)
    return Y


def backward(X, dY, W0, b0, s0, Wl, sl):
    """Adjoint of `forward`: returns dict dX, dW0, db0, ds0, dWl, dsl.

    Each step reverses one forward step: IWT^T = Haar, Haar^T = IWT (the
    +-1/2 Haar is orthonormal), dwconv^T = correlation with the flipped
    kernel, and the weight/scale/bias gradients are the per-tap sums.
    """
    L = 0 if Wl is None else Wl.shape[0]
    _, inter = forward(X, W0, b0, s0, Wl, sl, return_intermediates=True)
    base_pre, subs, convs, shapes = inter["base_pre"], inter["subs"], inter["convs"], inter["shapes"]
    k = W0.shape[-1]

    # base branch: Y += s0 * base_pre
    ds0 = np.sum(dY * base_pre, axis=(0, 2, 3))
    dbase = s0[None, :, None, None] * dY
    db0 = np.sum(dbase, axis=(0, 2, 3))
    dW0 = dwcorr_weight(X, dbase, k)
    dX = dwconv(dbase, W0[None, :, ::-1, ::-1])

    # synthesis cascade, reversed: t_{l-1} = crop(IWT(Z_l + t_l on LL));
    # crop^T pads with zeros, IWT^T = Haar
    dZ = []
    dt = dY
    for l in range(L):
        g = haar_analysis(pad_even(dt))
        dZ.append(g)
        dt = g[:, :, 0]
    dWl = np.zeros_like(Wl) if L else None
    dsl = np.zeros_like(sl) if L else None
    dsub = []
    for l in range(L):
        dsl[l] = np.sum(dZ[l] * convs[l], axis=(0, 3, 4))
        dconv = sl[l][None, :, :, None, None] * dZ[l]
        dWl[l] = dwcorr_weight(subs[l], dconv, k)
        dsub.append(dwconv(dconv, Wl[l][None, :, :, ::-1, ::-1]))
    # analysis chain, reversed: sub_l = Haar(pad(cur_{l-1})), cur_l = sub_l[LL];
    # Haar^T = IWT, pad^T crops
    dcur = None
    for l in reversed(range(L)):
        g = dsub[l]
        if dcur is not None:
            g = g.copy()
            g[:, :, 0] += dcur
        dcur = crop(haar_synthesis(g), shapes[l])
    if dcur is not None:
        dX = dX + dcur
    return dict(dX=dX, dW0=dW0, db0=db0, ds0=ds0, dWl=dWl, dsl=dsl)


def analysis_closed_form(X, l):
    """Level-l subbands straight from X (reformulation (1) of arXiv:2608.10805).

    sub_l^s(i, j) = 2^-l * sum over the 2^l x 2^l block (i, j) of
    sigma_s(bit_{l-1}(y), bit_{l-1}(x)) * X(y, x).
    """
    N, C, H, W = X.shape
    b = 1 << l
    ys = np.arange(H)
    xs = np.arange(W)
    py = (ys >> (l - 1)) & 1
    px = (xs >> (l - 1)) & 1
    out = np.zeros((N, C, 4, H // b, W // b))
    for s in range(4):
        sig = SIGN[s][py[:, None], px[None, :]]          # [H, W]
        weighted = X * sig
        out[:, :, s] = weighted.reshape(N, C, H // b, b, W // b, b).sum(axis=(3, 5)) / b
    return out


def synthesis_closed_form(Zs, H, W):
    """Sum over levels of the synthesised contributions, one pass per pixel.

    Zs[l-1] is Z_l [N, C, 4, H/2^l, W/2^l].  Output pixel (y, x) receives
    2^-l * sum_s sigma_s(bit_{l-1}(y), bit_{l-1}(x)) * Z_l^s(y >> l, x >> l)
    from every level l (reformulation (2) of arXiv:2608.10805).
    """
    N, C = Zs[0].shape[:2]
    ys = np.arange(H)
    xs = np.arange(W)
    out = np.zeros((N, C, H, W))
    for li, Z in enumerate(Zs):
        l = li + 1
        py = (ys >> (l - 1)) & 1
        px = (xs >> (l - 1)) & 1
        for s in range(4):
            sig = SIGN[s][py[:, None], px[None, :]]
            up = Z[:, :, s][:, :, ys >> l][:, :, :, xs >> l]
            out += sig * up / (1 << l)
    return out


def level_outputs(X, Wl, sl):
    """Z_l for every level (scaled level-conv outputs), for closed-form checks.

    Taken from `forward`'s own intermediates (the level-conv outputs before
    their scale), so the closed form is checked against exactly what the
    cascade computed, on any plane size.
    """
    C, k = X.shape[1], Wl.shape[-1]
    zero = np.zeros(C)
    _, inter = forward(X, np.zeros((C, k, k)), zero, zero, Wl, sl, return_intermediates=True)
    return [sl[l][None, :, :, None, None] * conv for l, conv in enumerate(inter["convs"])]
