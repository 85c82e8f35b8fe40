"""C-ABI checks that need no GPU: the library loads, exports every declared
entry point, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest
import torch

import depthwise_convolution_wtconv_b200 as wt
from depthwise_convolution_wtconv_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wtconv.h")

OK, ARG, SHAPE, ALIGN, WS = 0, 1, 2, 3, 4
FAKE = 0x10000          # 16-byte aligned address that is never dereferenced
FAKE_MIS = 0x10004      # misaligned


@pytest.fixture(scope="module")
def lib():
    return wt.load()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const char\*|size_t|int|wtconv_status)\s+(wtconv_\w+)\s*\(", text, re.M)))


def test_header_declares_the_binding_exports():
    assert declared_functions() == sorted(_lib.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for s in range(7):
        assert lib.wtconv_status_string(s)
    assert lib.wtconv_status_string(99) == b"unknown status"


def _desc(N=2, C=3, H=16, W=16, k=5, L=2, io=0):
    return _lib.WTConvDesc(N, C, H, W, k, L, io)


def test_workspace_sizes(lib):
    d = _desc()
    V = 25 * (1 + 4 * 2) + 1
    t1 = 2 * 3 * 8 * 8 * 4  # level-1 resolution synthesis of levels >= 2
    folded = 3 * ((1 + 4 * 2) * 28 + 4) * 4  # per channel: base + 4 kernels per level (k*k padded to 28) + bias
    assert lib.wtconv_workspace_size(ctypes.byref(d), 0) == 16 + t1 + folded
    assert lib.wtconv_workspace_size(ctypes.byref(d), 1) == 16 + t1 + folded
    assert lib.wtconv_workspace_size(ctypes.byref(d), 2) == 16 + 2 * 3 * V * 4
    # both backward passes: whole 16x16 planes take the fused pass, whose
    # workspace holds the partial sums and the adjoint folded block at once
    assert lib.wtconv_workspace_size(ctypes.byref(d), 3) == 16 + max(2 * 3 * V * 4, t1 + folded,
                                                                     2 * 3 * V * 4 + folded)
    assert lib.wtconv_workspace_size(ctypes.byref(_desc(L=1)), 0) == 16 + 3 * (5 * 28 + 4) * 4
    assert lib.wtconv_workspace_size(ctypes.byref(_desc(L=0)), 0) == 16 + 3 * (28 + 4) * 4
    assert lib.wtconv_workspace_size(ctypes.byref(_desc(k=4)), 2) == 0
    assert lib.wtconv_workspace_size(None, 2) == 0


def test_workspace_of_the_row_band_weight_gradient_path(lib):
    """256x256 planes with 5 levels do not fit one SM: the weight-gradient
    workspace then holds fewer partial-sum groups than N plus the raw LL
    planes of x and dy that each level hands to the next."""
    N, C, H, W, k, L = 16, 64, 256, 256, 5, 5
    d = _lib.WTConvDesc(N, C, H, W, k, L, 1)
    V = k * k * (1 + 4 * L) + 1
    ll = sum(2 * N * C * (H >> l) * (W >> l) for l in range(1, L)) * 4
    ws = lib.wtconv_workspace_size(ctypes.byref(d), 2)
    part = ws - 16 - ll  # C * V * 4 = 134656 bytes, a multiple of 16: no rounding
    assert part % (C * V * 4) == 0
    assert 1 <= part // (C * V * 4) < N
    assert lib.wtconv_workspace_size(ctypes.byref(d), 3) == max(ws, lib.wtconv_workspace_size(ctypes.byref(d), 0))


def test_kernel_launch_counts(lib):
    """Whole 56x56 planes with L = 3: fold + output kernel per data pass, the
    weight-gradient kernel + finalize, and both backward passes fused (fold,
    fused pass, finalize); 256x256 planes with L = 5 run as row bands: fold +
    deep + output kernel, and one launch per level + finalize (the backward
    passes one after the other)."""
    n = lambda d, op: lib.wtconv_kernel_launches(ctypes.byref(d), op)
    whole = _lib.WTConvDesc(32, 96, 56, 56, 5, 3, 0)
    assert [n(whole, op) for op in range(4)] == [2, 2, 2, 3]
    bands = _lib.WTConvDesc(16, 64, 256, 256, 5, 5, 1)
    assert [n(bands, op) for op in range(4)] == [3, 3, 6, 9]
    assert n(_lib.WTConvDesc(2, 3, 16, 16, 4, 2, 0), 0) == 0
    assert n(whole, 7) == 0


def test_level0_data_passes_take_one_kernel(lib):
    """Level-0 planes of at most 32x32 (on warps of their own) and fp32
    level-0 planes on the tensor-copy path run one launch per data pass (the
    scale is applied as the kernel loads the weights, no fold launch), then
    the weight-gradient kernel + finalize, and the backward as the two passes
    in turn; other level-0 planes (bf16 rows too wide for one tensor copy
    per unit here) keep fold + output kernel."""
    n = lambda d, op: lib.wtconv_kernel_launches(ctypes.byref(d), op)
    small = _lib.WTConvDesc(64, 384, 14, 14, 5, 0, 0)
    assert [n(small, op) for op in range(6)] == [1, 1, 2, 3, 1, 1]
    edge = _lib.WTConvDesc(2, 3, 32, 32, 7, 0, 1)     # 64 tiles: two per lane
    assert [n(edge, op) for op in range(4)] == [1, 1, 2, 3]
    tall = _lib.WTConvDesc(2, 3, 40, 16, 7, 0, 1)     # bf16, taller than 32: fold + output kernel
    assert [n(tall, op) for op in range(4)] == [2, 2, 2, 4]
    large = _lib.WTConvDesc(64, 32, 112, 112, 3, 0, 0)  # fp32, 112-float rows: one tensor copy per unit
    assert [n(large, op) for op in range(4)] == [1, 1, 2, 3]


def test_workspace_of_ragged_sides(lib):
    """Sides not multiples of 2^L: the workspace of the padded shape (H and W
    rounded up to multiples of 2^L), then the padded input planes (x or dy;
    both for the weight-gradient passes), each rounded to 16 bytes; outputs
    go straight to the caller's tensors."""
    d = _desc(H=18, W=13, L=2)                       # padded to 20 x 16
    t1 = 2 * 3 * 10 * 8 * 4
    folded = 3 * ((1 + 4 * 2) * 28 + 4) * 4
    act = 2 * 3 * 20 * 16 * 4
    V = 25 * (1 + 4 * 2) + 1
    fwd = 16 + t1 + folded                           # 5008, a multiple of 16
    bw = 16 + 2 * 3 * V * 4
    fused = bw + folded                              # partial sums and the adjoint block together
    assert lib.wtconv_workspace_size(ctypes.byref(d), 0) == fwd + act
    assert lib.wtconv_workspace_size(ctypes.byref(d), 1) == fwd + act
    assert lib.wtconv_workspace_size(ctypes.byref(d), 2) == bw + 2 * act
    assert lib.wtconv_workspace_size(ctypes.byref(d), 3) == (max(bw, fwd, fused) + 15) // 16 * 16 + 2 * act
    assert lib.wtconv_workspace_size(ctypes.byref(d), 4) == 16 + t1 + act
    bf = _desc(H=7, W=5, L=1, io=1)                  # 8 x 6 bf16: 2*3*8*6*2 = 576 bytes
    assert lib.wtconv_workspace_size(ctypes.byref(bf), 0) == 16 + 3 * (5 * 28 + 4) * 4 + 576


def test_ragged_launch_counts_and_noalloc(lib):
    """Ragged sides add one pad launch per input; the no-allocation weight
    gradients refuse them (no room for the copies)."""
    n = lambda d, op: lib.wtconv_kernel_launches(ctypes.byref(d), op)
    d = _lib.WTConvDesc(32, 96, 55, 54, 5, 3, 0)      # padded to 56 x 56; backward fused
    assert [n(d, op) for op in range(6)] == [3, 3, 4, 5, 2, 1]
    args = [FAKE] * 12
    assert lib.wtconv_backward_weight_noalloc(ctypes.byref(d), *args, None) == SHAPE


def test_large_planes_take_their_deep_levels_from_a_smaller_layer(lib):
    """512x512 planes with L = 2 do not fit the deep kernel: the levels >= 2
    run as a layer of L - 1 levels on the 256x256 LL planes.  Workspace:
    header, t1, the LL planes (as large as t1), the smaller layer's folded
    block and its own data-pass workspace (header only at L = 1), then this
    layer's folded block; launches: fold, LL planes, shifted block, the
    smaller layer's output kernel, this layer's output kernel."""
    d = _lib.WTConvDesc(2, 3, 512, 512, 5, 2, 0)
    t1 = 2 * 3 * 256 * 256 * 4
    fold_half = 3 * (5 * 28 + 4) * 4                 # L = 1 block of the smaller layer
    fold = 3 * (9 * 28 + 4) * 4
    assert lib.wtconv_workspace_size(ctypes.byref(d), 0) == 16 + t1 + t1 + fold_half + 16 + fold
    assert lib.wtconv_workspace_size(ctypes.byref(d), 4) == 16 + t1 + t1 + fold_half + 16
    n = lambda d, op: lib.wtconv_kernel_launches(ctypes.byref(d), op)
    assert n(d, 0) == 5 and n(d, 4) == 4
    # 1024x1024 with L = 3 recurses twice (512x512 L = 2, then 256x256 L = 1)
    big = _lib.WTConvDesc(1, 1, 1024, 1024, 3, 3, 0)
    assert n(big, 0) == 8
    fold = lambda L: (((1 + 4 * L) * 12 + 4 + 3) // 4 * 4) * 4    # k = 3: k*k padded to 12
    t1_512, t1_1024 = 256 * 256 * 4, 512 * 512 * 4
    inner = 16 + t1_512 + t1_512 + fold(1) + 16                     # the 512x512 L = 2 layer's pass
    outer = 16 + t1_1024 + t1_1024 + fold(2) + inner
    assert lib.wtconv_workspace_size(ctypes.byref(big), 4) == outer
    assert lib.wtconv_workspace_size(ctypes.byref(big), 0) == outer + fold(3)


def test_planes_wider_than_the_row_bands_hold_are_not_planned(lib):
    """Row bands keep whole rows on chip: with L >= 1 and k = 5 the data
    passes plan widths up to 1280 and no wider (0 launches = refused)."""
    n = lambda d, op: lib.wtconv_kernel_launches(ctypes.byref(d), op)
    assert n(_lib.WTConvDesc(1, 1, 64, 1280, 5, 2, 0), 0) > 0
    assert n(_lib.WTConvDesc(1, 1, 64, 1536, 5, 2, 0), 0) == 0
    assert n(_lib.WTConvDesc(1, 1, 4096, 64, 5, 2, 0), 0) > 0   # tall planes are fine


def test_folded_block_size_and_launches(lib):
    """The folded block: per channel k*k padded to 4, then the bias slot (4
    floats), then 4 padded kernels per level.  forward_folded launches the
    data pass alone (output kernel; deep kernel first for row-band planes
    with L >= 2); folding is one launch; its workspace is the status header
    plus the level >= 2 synthesis."""
    d = _desc()
    assert lib.wtconv_folded_size(ctypes.byref(d)) == 3 * ((1 + 4 * 2) * 28 + 4) * 4
    assert lib.wtconv_folded_size(ctypes.byref(_desc(L=0, k=3))) == 3 * (12 + 4) * 4
    assert lib.wtconv_folded_size(ctypes.byref(_desc(k=4))) == 0
    assert lib.wtconv_workspace_size(ctypes.byref(d), 4) == 16 + 2 * 3 * 8 * 8 * 4
    assert lib.wtconv_workspace_size(ctypes.byref(_desc(L=1)), 4) == 16
    n = lambda d, op: lib.wtconv_kernel_launches(ctypes.byref(d), op)
    assert n(_lib.WTConvDesc(32, 96, 56, 56, 5, 3, 0), 4) == 1
    assert n(_lib.WTConvDesc(16, 64, 256, 256, 5, 5, 1), 4) == 2
    assert n(_lib.WTConvDesc(16, 64, 256, 256, 5, 5, 1), 5) == 1


def test_fold_and_forward_folded_checks(lib):
    d = _desc()
    need = lib.wtconv_folded_size(ctypes.byref(d))
    f = lib.wtconv_fold_weights
    assert f(ctypes.byref(_desc(k=4)), FAKE, FAKE, FAKE, FAKE, FAKE, 0, FAKE, need, None) == ARG
    assert f(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 2, FAKE, need, None) == ARG
    assert f(ctypes.byref(d), FAKE, None, FAKE, FAKE, FAKE, 0, FAKE, need, None) == ARG  # forward needs b0
    assert f(ctypes.byref(d), FAKE, FAKE, FAKE, None, FAKE, 0, FAKE, need, None) == ARG
    assert f(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 0, None, need, None) == ARG
    assert f(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 0, FAKE + 4, need, None) == ALIGN
    assert f(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, 0, FAKE, need - 4, None) == WS
    g = lib.wtconv_forward_folded
    ws = lib.wtconv_workspace_size(ctypes.byref(d), 4)
    assert g(ctypes.byref(_desc(H=18, L=2)), FAKE, FAKE, FAKE, FAKE, ws, None) == WS  # padded copies need more
    assert g(ctypes.byref(d), None, FAKE, FAKE, FAKE, ws, None) == ARG
    assert g(ctypes.byref(d), FAKE, None, FAKE, FAKE, ws, None) == ARG
    assert g(ctypes.byref(d), FAKE, FAKE + 8, FAKE, FAKE, ws, None) == ALIGN
    assert g(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, ws - 4, None) == WS
    assert g(ctypes.byref(d), FAKE, FAKE, FAKE, None, ws, None) == WS


def _fwd(lib, d, x=FAKE, y=FAKE, w0=FAKE, b0=FAKE, s0=FAKE, wl=FAKE, sl=FAKE, ws=FAKE, nws=1 << 30):
    return lib.wtconv_forward(ctypes.byref(d) if d is not None else None, x, w0, b0, s0, wl, sl, y, ws, nws, None)


@pytest.mark.parametrize("kw,status", [
    (dict(k=4), ARG), (dict(k=9), ARG), (dict(k=0), ARG), (dict(L=-1), ARG), (dict(L=9), ARG),
    (dict(N=0), ARG), (dict(C=-1), ARG), (dict(H=0), ARG), (dict(io=7), ARG),
    (dict(H=1 << 16, W=(1 << 14) + 1, L=1), ARG),  # padded plane beyond 32-bit indexing
])
def test_forward_rejects_bad_descriptors(lib, kw, status):
    assert _fwd(lib, _desc(**kw)) == status


def test_forward_rejects_null_and_misaligned(lib):
    assert _fwd(lib, None) == ARG
    assert _fwd(lib, _desc(), x=None) == ARG
    assert _fwd(lib, _desc(), w0=None) == ARG
    assert _fwd(lib, _desc(), b0=None) == ARG
    assert _fwd(lib, _desc(), wl=None) == ARG
    assert _fwd(lib, _desc(), x=FAKE_MIS) == ALIGN
    assert _fwd(lib, _desc(), y=FAKE + 8) == ALIGN
    assert _fwd(lib, _desc(), w0=FAKE + 2) == ALIGN
    assert _fwd(lib, _desc(), ws=None) == WS
    assert _fwd(lib, _desc(), nws=16) == WS
    assert _fwd(lib, _desc(), ws=FAKE + 4) == ALIGN


def test_level0_allows_null_level_params(lib):
    # L = 0 with NULL wl/sl passes every host check; with the fake pointers a
    # compute call would follow, so only a bad descriptor is tried here.
    assert _fwd(lib, _desc(L=0, k=2), wl=None, sl=None) == ARG


def test_backward_data_checks(lib):
    d = _desc()
    f = lib.wtconv_backward_data
    assert f(ctypes.byref(d), None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == ARG
    assert f(ctypes.byref(d), FAKE_MIS, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None) == ALIGN
    ragged = _desc(W=10, L=2)
    need = lib.wtconv_workspace_size(ctypes.byref(ragged), 1)
    assert f(ctypes.byref(ragged), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need - 16, None) == WS
    assert f(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 0, None) == WS


def test_backward_weight_checks_workspace(lib):
    d = _desc()
    need = lib.wtconv_workspace_size(ctypes.byref(d), 2)
    f = lib.wtconv_backward_weight
    args = [FAKE] * 12
    assert f(ctypes.byref(d), *args, None, need, None) == WS
    assert f(ctypes.byref(d), *args, FAKE, need - 4, None) == WS
    assert f(ctypes.byref(d), *args, FAKE + 4, need, None) == ALIGN
    bad = list(args)
    bad[7] = None  # dw0
    assert f(ctypes.byref(d), *bad, FAKE, need, None) == ARG


def test_backward_checks(lib):
    d = _desc()
    need = lib.wtconv_workspace_size(ctypes.byref(d), 3)
    f = lib.wtconv_backward
    args = [FAKE] * 13
    assert f(ctypes.byref(d), *args, None, need, None) == WS
    bad = list(args)
    bad[7] = None  # dx
    assert f(ctypes.byref(d), *bad, FAKE, need, None) == ARG


def test_python_binding_refuses_cpu_tensors():
    x = torch.zeros(1, 1, 4, 4)
    w = torch.zeros(1, 3, 3)
    with pytest.raises(TypeError):
        wt.forward(x, w, torch.zeros(1), torch.ones(1))


_CPU = dict(x=torch.zeros(1, 2, 8, 8), w0=torch.zeros(2, 3, 3), b0=torch.zeros(2), s0=torch.ones(2),
            wl=torch.zeros(1, 2, 4, 3, 3), sl=torch.ones(1, 2, 4))
_CALLS = {
    "forward": lambda t: wt.forward(t["x"], t["w0"], t["b0"], t["s0"], t["wl"], t["sl"]),
    "backward_data": lambda t: wt.backward_data(t["x"], t["w0"], t["s0"], t["wl"], t["sl"]),
    "backward_weight": lambda t: wt.backward_weight(t["x"], t["x"], t["w0"], t["b0"], t["s0"], t["wl"], t["sl"]),
    "backward_weight_noalloc": lambda t: wt.backward_weight_noalloc(t["x"], t["x"], t["w0"], t["b0"], t["s0"],
                                                                    t["wl"], t["sl"]),
    "backward": lambda t: wt.backward(t["x"], t["x"], t["w0"], t["b0"], t["s0"], t["wl"], t["sl"]),
    "fold_weights": lambda t: wt.fold_weights(t["w0"], t["b0"], t["s0"], t["wl"], t["sl"]),
    "forward_folded": lambda t: wt.forward_folded(t["x"], torch.zeros(4096, dtype=torch.uint8), 3, 1),
}


@pytest.mark.parametrize("name", sorted(_CALLS))
def test_every_binding_refuses_cpu_tensors(name):
    """No entry point has a CPU path: host tensors are refused before any
    library call, on a machine with or without a GPU."""
    with pytest.raises(TypeError, match="CUDA tensor"):
        _CALLS[name](_CPU)
