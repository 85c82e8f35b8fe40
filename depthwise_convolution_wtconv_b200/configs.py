"""The synthetic WTConv workloads (shapes and dtypes) used by tests and bench.

Each entry names a layer shape: batch N, channels C, spatial H x W, kernel
size k, wavelet levels L and the I/O dtype ("f32" or "bf16"; arithmetic is
always fp32).  The shapes follow ConvNeXt-T-like stage shapes for the
WTConvNeXt evaluation mentioned in arXiv:2608.10805 (abstract).
"""
from dataclasses import dataclass


@dataclass(frozen=True)
class Workload:
    name: str
    N: int
    C: int
    H: int
    W: int
    k: int
    L: int
    io: str  # "f32" or "bf16"

    @property
    def P(self):
        return self.N * self.C * self.H * self.W

    @property
    def io_bytes(self):
        return 4 if self.io == "f32" else 2

    def as_dict(self):
        return dict(name=self.name, N=self.N, C=self.C, H=self.H, W=self.W,
                    k=self.k, L=self.L, io=self.io)


WORKLOADS = {
    # tiny case the oracle finishes in milliseconds
    "tiny_k5_L2": Workload("tiny_k5_L2", 1, 8, 16, 16, 5, 2, "f32"),
    # ConvNeXt-T stage-1 shape, 56 -> 28 -> 14 -> 7
    "stage1_f32_k5_L3": Workload("stage1_f32_k5_L3", 32, 96, 56, 56, 5, 3, "f32"),
    # stage-2 shape with bf16 I/O
    "stage2_bf16_k5_L2": Workload("stage2_bf16_k5_L2", 64, 192, 28, 28, 5, 2, "bf16"),
    # level-0 (plain depthwise conv) comparators
    "dw_k3_112_f32": Workload("dw_k3_112_f32", 64, 32, 112, 112, 3, 0, "f32"),
    "dw_k5_14_f32": Workload("dw_k5_14_f32", 64, 384, 14, 14, 5, 0, "f32"),
    # deep pyramid 256 -> 8 with bf16 I/O
    "deep_bf16_k5_L5": Workload("deep_bf16_k5_L5", 16, 64, 256, 256, 5, 5, "bf16"),
}

# the headline workload (the largest single-GPU shape) and the other
# full-size workloads the benchmark reports beside it
BENCH_WORKLOAD = "deep_bf16_k5_L5"
OTHER_WORKLOADS = ("stage1_f32_k5_L3", "stage2_bf16_k5_L2", "dw_k3_112_f32", "dw_k5_14_f32")
