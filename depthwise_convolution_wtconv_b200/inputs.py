"""Seeded synthetic inputs shared by the tests, the benchmark and smoke check.

Holds no layer arithmetic: it only draws random tensors.  Recipe (one CPU
generator seeded once, draws in this fixed order, all fp32):
  X ~ N(0,1) [N,C,H,W]; dY ~ N(0,1) [N,C,H,W];
  W0 ~ N(0, 1/k^2) [C,k,k]; b0 ~ N(0, 0.1^2) [C]; s0 ~ U(0.5,1.5) [C];
  then for l = 1..L: W_l ~ N(0, 1/k^2) [C,4,k,k] and s_l ~ U(0.5,1.5) [C,4].
For bf16 I/O the activations X and dY are rounded to bf16 (round to nearest
even); the parameters stay fp32.
"""
import torch


def make_inputs(wl, seed=0):
    """Return a dict of CPU fp32 tensors: X, dY, W0, b0, s0, Wl, sl.

    X and dY carry bf16-representable values when wl.io == "bf16".
    Wl is [L,C,4,k,k] and sl is [L,C,4] (empty tensors when L == 0).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    N, C, H, W, k, L = wl.N, wl.C, wl.H, wl.W, wl.k, wl.L
    X = torch.randn(N, C, H, W, generator=g, dtype=torch.float32)
    dY = torch.randn(N, C, H, W, generator=g, dtype=torch.float32)
    W0 = torch.randn(C, k, k, generator=g, dtype=torch.float32) / k
    b0 = torch.randn(C, generator=g, dtype=torch.float32) * 0.1
    s0 = torch.rand(C, generator=g, dtype=torch.float32) + 0.5
    Wl = torch.empty(L, C, 4, k, k, dtype=torch.float32)
    sl = torch.empty(L, C, 4, dtype=torch.float32)
    for l in range(L):
        Wl[l] = torch.randn(C, 4, k, k, generator=g, dtype=torch.float32) / k
        sl[l] = torch.rand(C, 4, generator=g, dtype=torch.float32) + 0.5
    if wl.io == "bf16":
        X = X.to(torch.bfloat16).to(torch.float32)
        dY = dY.to(torch.bfloat16).to(torch.float32)
    return dict(X=X, dY=dY, W0=W0, b0=b0, s0=s0, Wl=Wl, sl=sl)


def as_float64(inp):
    """numpy float64 copies of every tensor in `inp` (None for empty L)."""
    out = {}
    for key, t in inp.items():
        out[key] = t.double().numpy()
    if out["Wl"].shape[0] == 0:
        out["Wl"] = None
        out["sl"] = None
    return out
