"""Parity of the CUDA library (through its C ABI) with the float64 oracle.

Tolerances (per tensor, normwise): fp32 I/O max|gpu - oracle| / max|oracle|
<= 1e-4; bf16 I/O <= 2e-2 of the oracle's max-abs.  The oracle sees the
exact bf16 values of bf16 inputs.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import depthwise_convolution_wtconv_b200 as wt
from depthwise_convolution_wtconv_b200.configs import WORKLOADS, Workload
from depthwise_convolution_wtconv_b200.inputs import make_inputs, as_float64

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def _dev(inp, io):
    dt = torch.float32 if io == "f32" else torch.bfloat16
    d = {}
    for k, v in inp.items():
        if k in ("X", "dY"):
            d[k] = v.to(dt).cuda().contiguous()
        else:
            d[k] = v.cuda().contiguous()
    if d["Wl"].numel() == 0:
        d["Wl"] = None
        d["sl"] = None
    return d


def _rel(gpu, ref):
    gpu = np.asarray(gpu, dtype=np.float64)
    scale = max(np.max(np.abs(ref)), 1e-30)
    return float(np.max(np.abs(gpu - ref)) / scale)


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def run_gpu(d):
    y = wt.forward(d["X"], d["W0"], d["b0"], d["s0"], d["Wl"], d["sl"])
    dx = wt.backward_data(d["dY"], d["W0"], d["s0"], d["Wl"], d["sl"])
    g = wt.backward_weight(d["X"], d["dY"], d["W0"], d["b0"], d["s0"], d["Wl"], d["sl"])
    torch.cuda.synchronize()
    out = dict(Y=y, dX=dx, dW0=g["dw0"], db0=g["db0"], ds0=g["ds0"])
    if d["Wl"] is not None:
        out.update(dWl=g["dwl"], dsl=g["dsl"])
    return out


def run_oracle(p):
    Y = oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    g = oracle.backward(p["X"], p["dY"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    out = dict(Y=Y, dX=g["dX"], dW0=g["dW0"], db0=g["db0"], ds0=g["ds0"])
    if p["Wl"] is not None:
        out.update(dWl=g["dWl"], dsl=g["dsl"])
    return out


def check_all(wl, seed=0):
    inp = make_inputs(wl, seed)
    gpu = run_gpu(_dev(inp, wl.io))
    ref = run_oracle(as_float64(inp))
    errs = {k: _rel(_np(gpu[k]), ref[k]) for k in ref}
    bad = {k: e for k, e in errs.items() if not e <= TOL[wl.io]}
    assert not bad, (wl, errs)
    return errs


EDGE = [
    Workload("tiny", 1, 8, 16, 16, 5, 2, "f32"),
    Workload("ragged_L3", 3, 5, 24, 40, 3, 3, "f32"),
    Workload("deepest_1x1", 2, 3, 8, 8, 5, 3, "f32"),
    Workload("k7_L1", 2, 3, 16, 12, 7, 1, "f32"),
    Workload("k1_L2", 2, 4, 16, 16, 1, 2, "f32"),
    Workload("odd_L0", 2, 3, 7, 13, 5, 0, "f32"),
    Workload("odd_L0_bf16", 2, 3, 9, 11, 3, 0, "bf16"),
    Workload("bf16_w12", 2, 3, 12, 12, 5, 2, "bf16"),
    Workload("min_2x2", 1, 1, 2, 2, 3, 1, "f32"),
    Workload("w20", 2, 2, 20, 20, 5, 2, "f32"),
    Workload("tall", 1, 2, 64, 8, 5, 3, "f32"),
    Workload("multi_tile_L4", 2, 3, 64, 64, 5, 4, "f32"),
    Workload("L4_bf16", 3, 2, 48, 32, 5, 4, "bf16"),
    Workload("batchy_small", 37, 3, 14, 14, 5, 1, "f32"),
    # more work units than resident CTAs: every slot of the ring is reused
    Workload("reuse_L1_k5", 1, 1024, 8, 8, 5, 1, "f32"),
    Workload("reuse_L3_k3", 2, 600, 16, 16, 3, 3, "f32"),
    Workload("reuse_bf16_L2", 3, 500, 12, 12, 5, 2, "bf16"),
    Workload("reuse_L0_k5", 2, 900, 14, 14, 5, 0, "f32"),
    # planes too large for one SM's shared memory: row-band weight gradients
    Workload("band_L0_k3", 2, 3, 224, 224, 3, 0, "f32"),
    Workload("band_L1_bf16", 1, 2, 192, 160, 5, 1, "bf16"),
    Workload("band_L3_k7", 2, 2, 256, 128, 7, 3, "f32"),
    Workload("band_ragged_L2", 1, 2, 200, 180, 3, 2, "f32"),
    # level-0 weight gradients in row bands: rows not 16-byte multiples (no
    # bulk copies), and bf16
    Workload("band_L0_nobulk", 1, 2, 150, 146, 5, 0, "f32"),
    Workload("band_L0_bf16", 2, 2, 160, 132, 3, 0, "bf16"),
    # level-0 fp32 rows of 64 or more floats: input rows copied straight
    # into the padded row buffers (row bands with k = 7; batched whole planes
    # with a partial last batch; many units per CTA alternating the two
    # buffers; k = 1)
    Workload("rows_L0_k7_bands", 2, 2, 256, 96, 7, 0, "f32"),
    Workload("rows_L0_k5_batched", 5, 4, 8, 64, 5, 0, "f32"),
    Workload("rows_L0_k3_reuse", 6, 1000, 8, 64, 3, 0, "f32"),
    Workload("rows_L0_k1", 2, 3, 12, 64, 1, 0, "f32"),
    # level-0 fp32 planes by tensor copies (zero-padded boxes): the output
    # kernel and, where two buffer sets fit, the weight-gradient kernel with
    # no staging pass; heights not multiples of 4, the widest box (W + 8 =
    # 256), batched small planes with a partial last unit, k = 1 and 7
    Workload("tma_L0_k3_20x12", 3, 5, 20, 12, 3, 0, "f32"),
    Workload("tma_L0_k5_h7", 2, 4, 7, 16, 5, 0, "f32"),
    Workload("tma_L0_k7_8x8_batched", 7, 3, 8, 8, 7, 0, "f32"),
    Workload("tma_L0_k3_w248", 1, 2, 40, 248, 3, 0, "f32"),
    Workload("tma_L0_k1_30x40", 2, 2, 30, 40, 1, 0, "f32"),
    Workload("tma_L0_k5_reuse", 3, 700, 12, 20, 5, 0, "f32"),
    Workload("tma_L0_k5_bands_300", 1, 2, 300, 64, 5, 0, "f32"),
    Workload("tma_L0_k7_36x36_batched", 7, 3, 36, 36, 7, 0, "f32"),
    Workload("tma_L0_k5_reuse_40x36", 3, 300, 40, 36, 5, 0, "f32"),
    # level 0 on planes of at most 32x32: a warp takes up to 8 planes at a
    # time, a 4x4 tile per lane (two for 64-tile planes), the next planes
    # prefetched into registers (planes past 512 elements per warp load the
    # rest directly)
    Workload("small_L0_k1_14", 5, 7, 14, 14, 1, 0, "f32"),
    Workload("small_L0_k3_7x5_bf16", 3, 4, 7, 5, 3, 0, "bf16"),
    Workload("small_L0_k7_16x16", 9, 2, 16, 16, 7, 0, "f32"),
    Workload("small_L0_k5_32x16_bf16", 2, 3, 32, 16, 5, 0, "bf16"),
    Workload("small_L0_k3_1x1", 4, 3, 1, 1, 3, 0, "f32"),
    Workload("small_L0_k5_3x30", 6, 5, 3, 30, 5, 0, "f32"),
    Workload("small_L0_k5_many", 37, 129, 14, 14, 5, 0, "f32"),
    # sides not multiples of 2^L (zero-padded copies, cropped results)
    Workload("ragged_13x11_L2", 2, 3, 13, 11, 5, 2, "f32"),
    Workload("ragged_7x9_L3_bf16", 1, 2, 7, 9, 3, 3, "bf16"),
    Workload("ragged_55x54_L3", 2, 3, 55, 54, 5, 3, "f32"),
    Workload("ragged_bands_250_L2", 1, 2, 250, 246, 5, 2, "bf16"),
    Workload("ragged_3x3_L3_k1", 2, 2, 3, 3, 1, 3, "f32"),
    # planes too large for the deep kernel: levels >= 2 as a smaller layer on
    # the level-1 LL planes (twice for 1024x1024)
    Workload("recursive_512_L2", 1, 2, 512, 512, 5, 2, "f32"),
    Workload("recursive_640x384_L3_bf16", 1, 2, 640, 384, 3, 3, "bf16"),
]


@pytest.mark.parametrize("wl", EDGE, ids=[w.name for w in EDGE])
def test_parity_edge_cases(cuda_ok, wl):
    check_all(wl)


SMALL = {name: dataclasses.replace(w, N=min(w.N, 2)) for name, w in WORKLOADS.items()}


@pytest.mark.parametrize("name", list(SMALL))
def test_parity_workload_shapes_small_batch(cuda_ok, name):
    """Every workload's plane shape, k, L and dtype at batch 2: all outputs."""
    check_all(SMALL[name])


FULL = ["stage1_f32_k5_L3", "stage2_bf16_k5_L2", "dw_k3_112_f32", "dw_k5_14_f32"]


@pytest.mark.slow
@pytest.mark.parametrize("name", FULL)
def test_parity_full_size(cuda_ok, name):
    """Full workload size, every output element against the oracle."""
    check_all(WORKLOADS[name])


@pytest.mark.slow
def test_parity_deep_full_size_sampled(cuda_ok):
    """256x256 planes with 5 levels at full batch: y and dx on sampled batch
    entries (the layer is independent across n); parameter gradients on a
    sub-batch of the same planes."""
    wl = WORKLOADS["deep_bf16_k5_L5"]
    inp = make_inputs(wl, 0)
    d = _dev(inp, wl.io)
    y = wt.forward(d["X"], d["W0"], d["b0"], d["s0"], d["Wl"], d["sl"])
    dx = wt.backward_data(d["dY"], d["W0"], d["s0"], d["Wl"], d["sl"])
    torch.cuda.synchronize()
    for n in (0, wl.N - 1):
        p = as_float64({k: (v[n:n + 1] if k in ("X", "dY") else v) for k, v in inp.items()})
        ref = run_oracle(p)
        assert _rel(_np(y[n:n + 1]), ref["Y"]) <= TOL["bf16"]
        assert _rel(_np(dx[n:n + 1]), ref["dX"]) <= TOL["bf16"]
    sub = dataclasses.replace(wl, N=2)
    check_all(sub)


def test_data_passes_recurse_twice_for_1024x1024(cuda_ok):
    """1024x1024 planes with L = 3: the levels >= 2 run as a 512x512 layer
    with L = 2, whose own levels >= 2 run as a 256x256 layer with L = 1.
    Forward and backward-data against the oracle (the row-band weight
    gradients do not reach planes this wide with k = 7)."""
    wl = Workload("recursive_twice", 1, 1, 1024, 1024, 7, 3, "f32")
    inp = make_inputs(wl, 4)
    d = _dev(inp, wl.io)
    y = wt.forward(d["X"], d["W0"], d["b0"], d["s0"], d["Wl"], d["sl"])
    dx = wt.backward_data(d["dY"], d["W0"], d["s0"], d["Wl"], d["sl"])
    torch.cuda.synchronize()
    p = as_float64(inp)
    Y = oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    dX = oracle.backward(p["X"], p["dY"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])["dX"]
    assert _rel(_np(y), Y) <= TOL["f32"]
    assert _rel(_np(dx), dX) <= TOL["f32"]


def test_weight_gradients_deterministic(cuda_ok):
    wl = Workload("det", 4, 6, 32, 32, 5, 3, "f32")
    d = _dev(make_inputs(wl, 1), wl.io)
    a = run_gpu(d)
    b = run_gpu(d)
    for k in a:
        assert torch.equal(a[k], b[k]), k


@pytest.mark.parametrize("wl", [Workload("fused", 3, 4, 32, 32, 5, 2, "f32"),
                                Workload("fused_ragged", 2, 3, 29, 27, 5, 2, "f32")], ids=["even", "ragged"])
def test_fused_backward_matches_separate_calls(cuda_ok, wl):
    d = _dev(make_inputs(wl, 2), wl.io)
    sep = run_gpu(d)
    dx, g = wt.backward(d["X"], d["dY"], d["W0"], d["b0"], d["s0"], d["Wl"], d["sl"])
    torch.cuda.synchronize()
    assert torch.equal(dx, sep["dX"])
    for k, kk in (("dw0", "dW0"), ("db0", "db0"), ("ds0", "ds0"), ("dwl", "dWl"), ("dsl", "dsl")):
        assert torch.allclose(g[k], sep[kk], rtol=1e-6, atol=1e-6), k


FUSED_BWD = [
    Workload("fbwd_stage1_n3", 3, 5, 56, 56, 5, 3, "f32"),
    Workload("fbwd_bf16_L2", 4, 3, 28, 28, 5, 2, "bf16"),
    Workload("fbwd_L1_k3", 5, 2, 24, 20, 3, 1, "f32"),
    Workload("fbwd_L0_k5_small", 9, 3, 14, 14, 5, 0, "f32"),
    Workload("fbwd_L0_k3_bf16", 3, 2, 24, 24, 3, 0, "bf16"),
    # k = 7 runs the two passes apart (too many registers for the fused pass)
    Workload("bwd_L1_k7_apart", 3, 2, 24, 24, 7, 1, "bf16"),
    Workload("fbwd_L4_k1", 2, 3, 32, 48, 1, 4, "f32"),
    Workload("fbwd_L3_k3", 2, 2, 40, 40, 3, 3, "f32"),
    Workload("fbwd_ragged_L3", 3, 2, 53, 45, 3, 3, "f32"),
    Workload("fbwd_many_units", 13, 300, 16, 16, 5, 2, "f32"),
    # several units per CTA: the Z planes written over x's buffers must not
    # leak into the next unit's zero borders
    Workload("fbwd_units_L1", 40, 3, 16, 16, 3, 1, "f32"),
    Workload("fbwd_units_L3", 6, 3, 32, 32, 5, 3, "f32"),
    Workload("fbwd_units_L2_bf16", 9, 2, 24, 24, 5, 2, "bf16"),
]


@pytest.mark.parametrize("wl", FUSED_BWD, ids=[w.name for w in FUSED_BWD])
def test_fused_backward_against_oracle(cuda_ok, wl):
    """wtconv_backward (one staging of x and dy per unit on whole planes: the
    correlations, then the adjoint data pass from the same dy pyramid)
    against the oracle: dx and every parameter gradient."""
    inp = make_inputs(wl, 7)
    d = _dev(inp, wl.io)
    desc = wt.make_desc(wl.N, wl.C, wl.H, wl.W, wl.k, wl.L, wl.io)
    dx, g = wt.backward(d["X"], d["dY"], d["W0"], d["b0"], d["s0"], d["Wl"], d["sl"])
    torch.cuda.synchronize()
    p = as_float64(inp)
    ref = oracle.backward(p["X"], p["dY"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    pairs = [(dx, "dX"), (g["dw0"], "dW0"), (g["db0"], "db0"), (g["ds0"], "ds0")]
    if wl.L:
        pairs += [(g["dwl"], "dWl"), (g["dsl"], "dsl")]
    for got, key in pairs:
        err = _rel(_np(got), ref[key])
        assert err <= TOL[wl.io], (wl.name, key, err)
    # k <= 5 takes the fused pass: fold, fused kernel, finalize (plus one pad
    # per input for sides not multiples of 2^L)
    pads = 2 if (wl.H % (1 << wl.L) or wl.W % (1 << wl.L)) else 0
    apart = wt.kernel_launches(desc, 1) + wt.kernel_launches(desc, 2)
    assert wt.kernel_launches(desc, 3) == (3 + pads if wl.k <= 5 else apart)


BANDED = [
    Workload("band_k3_L1", 8, 64, 192, 192, 3, 1, "f32"),
    Workload("band_k5_L2_bf16", 4, 64, 192, 192, 5, 2, "bf16"),
    Workload("band_k7_L1_bf16", 8, 64, 160, 160, 7, 1, "bf16"),
    Workload("band_k3_L3", 4, 64, 256, 256, 3, 3, "f32"),
]


@pytest.mark.parametrize("wl", BANDED, ids=[w.name for w in BANDED])
def test_row_bands_on_sampled_planes(cuda_ok, wl):
    """Row-band shapes with thousands of bands (more than the resident CTAs
    take in one round) and every odd kernel size.  The layer is independent
    across (n, c) planes, so the forward and backward-data outputs of
    sampled planes are checked against the oracle run on those planes
    alone."""
    inp = make_inputs(wl, 11)
    d = _dev(inp, wl.io)
    y = wt.forward(d["X"], d["W0"], d["b0"], d["s0"], d["Wl"], d["sl"])
    dx = wt.backward_data(d["dY"], d["W0"], d["s0"], d["Wl"], d["sl"])
    torch.cuda.synchronize()
    p = as_float64(inp)
    for n, c in ((0, 0), (wl.N - 1, wl.C - 1), (wl.N // 2, wl.C // 3)):
        one = {key: p[key][n:n + 1, c:c + 1] for key in ("X", "dY")}
        one.update(W0=p["W0"][c:c + 1], b0=p["b0"][c:c + 1], s0=p["s0"][c:c + 1],
                   Wl=p["Wl"][:, c:c + 1], sl=p["sl"][:, c:c + 1])
        Y = oracle.forward(one["X"], one["W0"], one["b0"], one["s0"], one["Wl"], one["sl"])
        dX = oracle.backward(one["X"], one["dY"], one["W0"], one["b0"], one["s0"], one["Wl"], one["sl"])["dX"]
        assert _rel(_np(y[n:n + 1, c:c + 1]), Y) <= TOL[wl.io], (wl.name, n, c, "Y")
        assert _rel(_np(dx[n:n + 1, c:c + 1]), dX) <= TOL[wl.io], (wl.name, n, c, "dX")


def test_delta_kernels_on_gpu(cuda_ok):
    """Closed form Y = s0 X + sum_l s_l U_{l-1}(X) through the CUDA path."""
    N, C, H, W, k, L = 2, 3, 32, 32, 5, 3
    g = torch.Generator().manual_seed(5)
    X = torch.randn(N, C, H, W, generator=g)
    W0 = torch.zeros(C, k, k); W0[:, 2, 2] = 1
    Wl = torch.zeros(L, C, 4, k, k); Wl[..., 2, 2] = 1
    s0 = torch.rand(C, generator=g) + 0.5
    sc = torch.rand(L, C, generator=g) + 0.5
    sl = sc[:, :, None].repeat(1, 1, 4).contiguous()
    y = wt.forward(X.cuda(), W0.cuda(), torch.zeros(C).cuda(), s0.cuda(), Wl.cuda(), sl.cuda()).cpu()
    ref = s0.view(1, C, 1, 1) * X
    for l in range(1, L + 1):
        b = 1 << (l - 1)
        m = torch.nn.functional.avg_pool2d(X, b) if b > 1 else X
        m = m.repeat_interleave(b, 2).repeat_interleave(b, 3)
        ref = ref + sc[l - 1].view(1, C, 1, 1) * m
    assert (y - ref).abs().max().item() <= 1e-5 * ref.abs().max().item()


def test_stream_argument_and_preallocated_outputs(cuda_ok):
    wl = Workload("stream", 2, 3, 16, 16, 3, 2, "f32")
    d = _dev(make_inputs(wl, 3), wl.io)
    s = torch.cuda.Stream()
    y = torch.empty_like(d["X"])
    with torch.cuda.stream(s):
        wt.forward(d["X"], d["W0"], d["b0"], d["s0"], d["Wl"], d["sl"], y=y, stream=s)
    s.synchronize()
    ref = wt.forward(d["X"], d["W0"], d["b0"], d["s0"], d["Wl"], d["sl"])
    torch.cuda.synchronize()
    assert torch.equal(y, ref)


@pytest.mark.parametrize("wl", [Workload("status_whole", 2, 3, 32, 32, 5, 3, "f32"),
                                Workload("status_bands", 1, 2, 256, 128, 5, 3, "bf16"),
                                Workload("status_ragged", 2, 3, 30, 27, 3, 2, "f32")],
                         ids=["whole_planes", "row_bands", "ragged"])
def test_status_word_stays_clear(cuda_ok, wl):
    """The workspace header's status word is set only when a bounded wait for
    an asynchronous copy runs out; after ordinary calls of every entry point
    (whole-plane and row-band paths) it must still read 0."""
    d = _dev(make_inputs(wl, 6), wl.io)
    desc = wt.make_desc(wl.N, wl.C, wl.H, wl.W, wl.k, wl.L, wl.io)
    ws = torch.zeros(wt.workspace_size(desc, 3), dtype=torch.uint8, device="cuda")
    wt.forward(d["X"], d["W0"], d["b0"], d["s0"], d["Wl"], d["sl"], ws=ws)
    wt.backward_data(d["dY"], d["W0"], d["s0"], d["Wl"], d["sl"], ws=ws)
    wt.backward_weight(d["X"], d["dY"], d["W0"], d["b0"], d["s0"], d["Wl"], d["sl"], ws=ws)
    wt.backward(d["X"], d["dY"], d["W0"], d["b0"], d["s0"], d["Wl"], d["sl"], ws=ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
