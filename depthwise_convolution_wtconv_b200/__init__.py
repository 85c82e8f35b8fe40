"""WTConv (multi-level Haar wavelet depthwise convolution) for B200.

The compute path is libwtconv.so (hand-written sm_100a CUDA kernels behind a
C ABI, see include/wtconv.h); `forward`, `backward_data`, `backward_weight`,
`backward`, `fold_weights` and `forward_folded` are thin ctypes wrappers over
it that take CUDA tensors.
"""
from ._lib import (  # noqa: F401
    forward, backward_data, backward_weight, backward, backward_weight_noalloc, fold_weights, forward_folded,
    workspace_size, kernel_launches, make_desc, load,
    WTConvError, EXPORTS, LIB_PATH,
)
