"""ctypes binding of libwtconv.so (argument marshalling only).

Every computation runs in the library's CUDA kernels; this module passes
tensor data pointers, the shape descriptor and the current CUDA stream.
It raises when the library is missing or a tensor is not on a CUDA device:
there is no CPU fallback.
"""
import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libwtconv.so")

F32, BF16 = 0, 1
OP_FORWARD, OP_BACKWARD_DATA, OP_BACKWARD_WEIGHT, OP_BACKWARD = 0, 1, 2, 3
OP_FORWARD_FOLDED, OP_FOLD = 4, 5
STATUS_NAMES = {0: "WTCONV_OK", 1: "WTCONV_ERR_ARG", 2: "WTCONV_ERR_SHAPE", 3: "WTCONV_ERR_ALIGN",
                4: "WTCONV_ERR_WORKSPACE", 5: "WTCONV_ERR_CUDA", 6: "WTCONV_ERR_UNSUPPORTED",
                7: "WTCONV_ERR_SCRATCH_LIMIT"}

# every symbol include/wtconv.h declares
EXPORTS = ("wtconv_workspace_size", "wtconv_forward", "wtconv_backward_data", "wtconv_backward_weight",
           "wtconv_backward", "wtconv_backward_weight_noalloc", "wtconv_folded_size", "wtconv_fold_weights",
           "wtconv_forward_folded", "wtconv_kernel_launches", "wtconv_status_string",
           "wtconv_noalloc_scratch_bytes")


class WTConvDesc(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int), ("C", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("k", ctypes.c_int), ("L", ctypes.c_int), ("io", ctypes.c_int)]


class WTConvError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


_lib = None


def load(path=LIB_PATH):
    """Loads the shared library (raises OSError when it is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise OSError(f"libwtconv.so not built at {path}; run python -m depthwise_convolution_wtconv_b200.build")
    lib = ctypes.CDLL(path)
    vp, fp, sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t
    dp = ctypes.POINTER(WTConvDesc)
    lib.wtconv_workspace_size.argtypes = [dp, ctypes.c_int]
    lib.wtconv_workspace_size.restype = sz
    lib.wtconv_forward.argtypes = [dp, vp, fp, fp, fp, fp, fp, vp, vp, sz, vp]
    lib.wtconv_forward.restype = ctypes.c_int
    lib.wtconv_backward_data.argtypes = [dp, vp, fp, fp, fp, fp, vp, vp, sz, vp]
    lib.wtconv_backward_data.restype = ctypes.c_int
    lib.wtconv_backward_weight.argtypes = [dp, vp, vp, fp, fp, fp, fp, fp, fp, fp, fp, fp, fp, vp, sz, vp]
    lib.wtconv_backward_weight.restype = ctypes.c_int
    lib.wtconv_backward.argtypes = [dp, vp, vp, fp, fp, fp, fp, fp, vp, fp, fp, fp, fp, fp, vp, sz, vp]
    lib.wtconv_backward.restype = ctypes.c_int
    lib.wtconv_backward_weight_noalloc.argtypes = [dp, vp, vp, fp, fp, fp, fp, fp, fp, fp, fp, fp, fp, vp]
    lib.wtconv_backward_weight_noalloc.restype = ctypes.c_int
    lib.wtconv_status_string.argtypes = [ctypes.c_int]
    lib.wtconv_status_string.restype = ctypes.c_char_p
    lib.wtconv_folded_size.argtypes = [dp]
    lib.wtconv_folded_size.restype = sz
    lib.wtconv_fold_weights.argtypes = [dp, fp, fp, fp, fp, fp, ctypes.c_int, vp, sz, vp]
    lib.wtconv_fold_weights.restype = ctypes.c_int
    lib.wtconv_forward_folded.argtypes = [dp, vp, vp, vp, vp, sz, vp]
    lib.wtconv_forward_folded.restype = ctypes.c_int
    lib.wtconv_kernel_launches.argtypes = [dp, ctypes.c_int]
    lib.wtconv_kernel_launches.restype = ctypes.c_int
    lib.wtconv_noalloc_scratch_bytes.argtypes = []
    lib.wtconv_noalloc_scratch_bytes.restype = sz
    _lib = lib
    return lib


def noalloc_scratch_bytes():
    """Size of the device array the no-allocation weight-gradient call uses,
    as the loaded library was built with."""
    return int(load().wtconv_noalloc_scratch_bytes())


def make_desc(N, C, H, W, k, L, io):
    return WTConvDesc(N, C, H, W, k, L, BF16 if io in ("bf16", torch.bfloat16, BF16) else F32)


def workspace_size(desc, op):
    return int(load().wtconv_workspace_size(ctypes.byref(desc), op))


def kernel_launches(desc, op):
    """Kernel launches one call of `op` makes for the shape `desc`."""
    return int(load().wtconv_kernel_launches(ctypes.byref(desc), op))


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status, what):
    if status != 0:
        raise WTConvError(status, what)


def _cuda(t, name, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}")
    return t


def _levels(wl):
    return 0 if (wl is None or wl.numel() == 0) else int(wl.shape[0])


def _desc_from(x, w0, wl):
    N, C, H, W = x.shape
    return make_desc(N, C, H, W, int(w0.shape[-1]), _levels(wl), x.dtype)


def _params(w0, b0, s0, wl, sl):
    for t, n in ((w0, "w0"), (s0, "s0")):
        _cuda(t, n, torch.float32)
    if b0 is not None:
        _cuda(b0, "b0", torch.float32)
    if _levels(wl):
        _cuda(wl, "wl", torch.float32)
        _cuda(sl, "sl", torch.float32)
        return wl, sl
    return None, None


def _workspace(desc, op, ws):
    need = workspace_size(desc, op)
    if need == 0:
        return None, 0
    if ws is None:
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    return ws, ws.numel() * ws.element_size()


def forward(x, w0, b0, s0, wl=None, sl=None, y=None, ws=None, stream=None):
    """y = WTConv(x); x [N,C,H,W] fp32/bf16 CUDA, parameters fp32 CUDA."""
    lib = load()
    _cuda(x, "x")
    wl, sl = _params(w0, b0, s0, wl, sl)
    desc = _desc_from(x, w0, wl)
    y = torch.empty_like(x) if y is None else _cuda(y, "y", x.dtype)
    ws, nws = _workspace(desc, OP_FORWARD, ws)
    _check(lib.wtconv_forward(ctypes.byref(desc), _ptr(x), _ptr(w0), _ptr(b0), _ptr(s0), _ptr(wl), _ptr(sl),
                              _ptr(y), _ptr(ws), nws, _stream(stream)), "wtconv_forward")
    return y


def backward_data(dy, w0, s0, wl=None, sl=None, dx=None, ws=None, stream=None):
    """dx = J^T dy (adjoint of the forward map in x)."""
    lib = load()
    _cuda(dy, "dy")
    wl, sl = _params(w0, None, s0, wl, sl)
    desc = _desc_from(dy, w0, wl)
    dx = torch.empty_like(dy) if dx is None else _cuda(dx, "dx", dy.dtype)
    ws, nws = _workspace(desc, OP_BACKWARD_DATA, ws)
    _check(lib.wtconv_backward_data(ctypes.byref(desc), _ptr(dy), _ptr(w0), _ptr(s0), _ptr(wl), _ptr(sl),
                                    _ptr(dx), _ptr(ws), nws, _stream(stream)), "wtconv_backward_data")
    return dx


def _grad_outputs(w0, b0, s0, wl, sl, grads):
    if grads is not None:
        return grads
    return dict(dw0=torch.empty_like(w0), db0=torch.empty_like(s0), ds0=torch.empty_like(s0),
                dwl=None if wl is None else torch.empty_like(wl), dsl=None if sl is None else torch.empty_like(sl))


def backward_weight(x, dy, w0, b0, s0, wl=None, sl=None, grads=None, ws=None, stream=None):
    """Parameter gradients of <y, dy>: dict dw0, db0, ds0, dwl, dsl."""
    lib = load()
    _cuda(x, "x")
    _cuda(dy, "dy", x.dtype)
    wl, sl = _params(w0, b0, s0, wl, sl)
    desc = _desc_from(x, w0, wl)
    g = _grad_outputs(w0, b0, s0, wl, sl, grads)
    ws, nws = _workspace(desc, OP_BACKWARD_WEIGHT, ws)
    _check(lib.wtconv_backward_weight(ctypes.byref(desc), _ptr(x), _ptr(dy), _ptr(w0), _ptr(b0), _ptr(s0),
                                      _ptr(wl), _ptr(sl), _ptr(g["dw0"]), _ptr(g["db0"]), _ptr(g["ds0"]),
                                      _ptr(g["dwl"]), _ptr(g["dsl"]), _ptr(ws), nws, _stream(stream)),
           "wtconv_backward_weight")
    return g


def backward_weight_noalloc(x, dy, w0, b0, s0, wl=None, sl=None, grads=None, stream=None):
    """Parameter gradients without a workspace: the library keeps its partial
    sums in its own fixed device array (for callers that cannot allocate
    device memory where they call it).  Same outputs as backward_weight.
    The C call allocates nothing; this wrapper allocates the gradient tensors
    only when `grads` is not given, so pass `grads` to keep the call
    allocation-free."""
    lib = load()
    _cuda(x, "x")
    _cuda(dy, "dy", x.dtype)
    wl, sl = _params(w0, b0, s0, wl, sl)
    desc = _desc_from(x, w0, wl)
    g = _grad_outputs(w0, b0, s0, wl, sl, grads)
    _check(lib.wtconv_backward_weight_noalloc(ctypes.byref(desc), _ptr(x), _ptr(dy), _ptr(w0), _ptr(b0), _ptr(s0),
                                              _ptr(wl), _ptr(sl), _ptr(g["dw0"]), _ptr(g["db0"]), _ptr(g["ds0"]),
                                              _ptr(g["dwl"]), _ptr(g["dsl"]), _stream(stream)),
           "wtconv_backward_weight_noalloc")
    return g


def backward(x, dy, w0, b0, s0, wl=None, sl=None, dx=None, grads=None, ws=None, stream=None):
    """dx and all parameter gradients in one call: (dx, grads dict)."""
    lib = load()
    _cuda(x, "x")
    _cuda(dy, "dy", x.dtype)
    wl, sl = _params(w0, b0, s0, wl, sl)
    desc = _desc_from(x, w0, wl)
    dx = torch.empty_like(dy) if dx is None else _cuda(dx, "dx", dy.dtype)
    g = _grad_outputs(w0, b0, s0, wl, sl, grads)
    ws, nws = _workspace(desc, OP_BACKWARD, ws)
    _check(lib.wtconv_backward(ctypes.byref(desc), _ptr(x), _ptr(dy), _ptr(w0), _ptr(b0), _ptr(s0), _ptr(wl),
                               _ptr(sl), _ptr(dx), _ptr(g["dw0"]), _ptr(g["db0"]), _ptr(g["ds0"]), _ptr(g["dwl"]),
                               _ptr(g["dsl"]), _ptr(ws), nws, _stream(stream)), "wtconv_backward")
    return dx, g


def fold_weights(w0, b0, s0, wl=None, sl=None, adjoint=False, folded=None, stream=None):
    """The scales folded into the weights once (for fixed parameters, e.g.
    inference): a uint8 CUDA tensor holding the library's folded block; with
    adjoint=True the backward-data block (flipped kernels, no bias)."""
    lib = load()
    wl, sl = _params(w0, None if adjoint else b0, s0, wl, sl)
    C, k = w0.shape[0], w0.shape[-1]
    desc = make_desc(1, C, 1 << _levels(wl), 1 << _levels(wl), k, _levels(wl), "f32")
    need = lib.wtconv_folded_size(ctypes.byref(desc))
    if folded is None:
        folded = torch.empty(max(need, 16), dtype=torch.uint8, device="cuda")
    _check(lib.wtconv_fold_weights(ctypes.byref(desc), _ptr(w0), _ptr(None if adjoint else b0), _ptr(s0),
                                   _ptr(wl), _ptr(sl), int(bool(adjoint)), _ptr(folded),
                                   folded.numel() * folded.element_size(), _stream(stream)), "wtconv_fold_weights")
    return folded


def forward_folded(x, folded, k, L, y=None, ws=None, stream=None):
    """y = WTConv(x) over a block from fold_weights (kernel size k, L levels);
    with an adjoint block and dy for x, the backward-data pass."""
    lib = load()
    _cuda(x, "x")
    _cuda(folded, "folded")
    N, C, H, W = x.shape
    desc = make_desc(N, C, H, W, k, L, "bf16" if x.dtype == torch.bfloat16 else "f32")
    if folded.numel() * folded.element_size() < lib.wtconv_folded_size(ctypes.byref(desc)):
        raise ValueError("folded block too small for this shape")
    y = torch.empty_like(x) if y is None else _cuda(y, "y", x.dtype)
    ws, nws = _workspace(desc, OP_FORWARD_FOLDED, ws)
    _check(lib.wtconv_forward_folded(ctypes.byref(desc), _ptr(x), _ptr(folded), _ptr(y), _ptr(ws), nws,
                                     _stream(stream)), "wtconv_forward_folded")
    return y
