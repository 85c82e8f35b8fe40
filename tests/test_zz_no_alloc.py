"""The no-allocation weight-gradient entry point.

wtconv_backward_weight_noalloc serves callers that cannot allocate device
memory where they call the library (no allocator at the call site, or one
that must not run during steady-state steps): it keeps its partial sums in
the library's own fixed device array instead of a caller workspace.  These
tests check it against wtconv_backward_weight, the entry point that takes a
workspace, on two calls in a row, and that oversized shapes are refused
before anything reaches the GPU.  The file is named so that pytest collects
it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import depthwise_convolution_wtconv_b200 as wt
from depthwise_convolution_wtconv_b200 import _lib
from depthwise_convolution_wtconv_b200.configs import Workload
from depthwise_convolution_wtconv_b200.inputs import make_inputs

TOL = {"f32": 1e-4, "bf16": 2e-2}
SCRATCH_LIMIT = 7
FAKE = 0x10000


def _dev(inp, io):
    dt = torch.float32 if io == "f32" else torch.bfloat16
    d = {k: (v.to(dt) if k in ("X", "dY") else v).cuda().contiguous() for k, v in inp.items()}
    if d["Wl"].numel() == 0:
        d["Wl"] = None
        d["sl"] = None
    return d


def _rel(a, b):
    a = a.double().cpu().numpy()
    b = b.double().cpu().numpy()
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


CASES = [
    Workload("stage1_shape_n4", 4, 96, 56, 56, 5, 3, "f32"),
    # 2048 channels: one group of partial sums is 1.85 MB, so the library
    # must use fewer CTAs per channel than it would with a workspace
    Workload("many_channels", 8, 2048, 16, 16, 5, 2, "f32"),
    Workload("bf16_L0", 6, 64, 28, 28, 3, 0, "bf16"),
    # planes too large for one SM: the row-band path, LL planes in the array too
    Workload("band_path_L2", 1, 2, 192, 192, 5, 2, "f32"),
    # row-band path whose LL planes (7.9 MB) leave room for 10 groups of
    # partial sums where the workspace entry point would use 20: the array
    # forces fewer CTAs per channel on the row-band path
    Workload("band_fewer_groups", 2, 14, 384, 384, 5, 2, "f32"),
]


@pytest.mark.gpu
@pytest.mark.parametrize("wl", CASES, ids=[w.name for w in CASES])
def test_noalloc_matches_workspace_entry_point_on_two_calls(cuda_ok, wl):
    d = _dev(make_inputs(wl, 4), wl.io)
    args = (d["X"], d["dY"], d["W0"], d["b0"], d["s0"], d["Wl"], d["sl"])
    ref = wt.backward_weight(*args)
    torch.cuda.synchronize()
    for call in range(2):
        got = wt.backward_weight_noalloc(*args)
        torch.cuda.synchronize()
        for key in ("dw0", "db0", "ds0", "dwl", "dsl"):
            if ref[key] is None:
                assert got[key] is None
                continue
            err = _rel(got[key], ref[key])
            assert err <= TOL[wl.io], (wl.name, call, key, err)


def test_noalloc_refuses_shapes_beyond_its_array():
    """C * (k*k*(1+4L)+1) floats + 16 bytes over 8 MiB is refused on the host
    (no GPU is touched, so this runs anywhere)."""
    lib = wt.load()
    V = 25 * (1 + 4 * 2) + 1
    C = (_lib.noalloc_scratch_bytes() // (V * 4)) + 1
    d = _lib.WTConvDesc(1, C, 16, 16, 5, 2, 0)
    st = lib.wtconv_backward_weight_noalloc(ctypes.byref(d), *([FAKE] * 12), None)
    assert st == SCRATCH_LIMIT
    assert b"no-allocation" in lib.wtconv_status_string(st)
    d_ok = _lib.WTConvDesc(1, C, 16, 16, 4, 2, 0)  # even k: argument error comes first
    assert lib.wtconv_backward_weight_noalloc(ctypes.byref(d_ok), *([FAKE] * 12), None) == 1
