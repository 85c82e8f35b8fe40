"""Host-side pieces of the benchmark that need no GPU: the algorithmic counts
behind the roofline, the launch count it reports, and the source hash that
decides whether the committed DRAM traffic still describes the kernels."""
import json
import os

import pytest

import bench
import depthwise_convolution_wtconv_b200 as wt
from depthwise_convolution_wtconv_b200.configs import WORKLOADS


def test_algorithmic_counts_of_the_stage1_workload():
    """32x96x56x56, k = 5, L = 3, fp32: per pixel and pass
    k^2 (1 + (4/3)(1 - 4^-3)) = 25 * 1 + 25 * (4/3) * (63/64) = 57.8125 FMAs;
    forward bytes = read x + write y = 8 per pixel (plus the parameters)."""
    wl = WORKLOADS["stage1_f32_k5_L3"]
    c = bench.algorithmic_counts(wl)
    P = 32 * 96 * 56 * 56
    assert c["passes"]["fwd"]["fma"] == pytest.approx(P * 57.8125, rel=1e-12)
    params = 4 * (96 * 25 + 2 * 96 + 3 * 96 * 4 * 26)
    assert bench.param_bytes(wl) == params
    assert c["passes"]["fwd"]["bytes"] == 8 * P + params
    assert c["passes"]["bwd_weight"]["bytes"] == 8 * P + 2 * params
    # a step must read x, write y, read x and dy, write dx: 5 activations
    assert c["step"]["bytes"] == 5 * 4 * P + 2 * params
    assert c["step"]["design_bytes"] == 6 * 4 * P + 4 * params
    assert c["step"]["fma"] == pytest.approx(3 * P * 57.8125, rel=1e-12)
    # level 0: the plain depthwise conv, k^2 FMAs per pixel
    c0 = bench.algorithmic_counts(WORKLOADS["dw_k3_112_f32"])
    assert c0["passes"]["fwd"]["fma"] == 64 * 32 * 112 * 112 * 9


def test_algorithmic_bytes_of_the_deep_bf16_workload():
    """16x64x256x256 bf16: S = 134.2 MB; 5S + 2 params = 671.4 MB a step."""
    wl = WORKLOADS["deep_bf16_k5_L5"]
    c = bench.algorithmic_counts(wl)
    S = 16 * 64 * 256 * 256 * 2
    assert S == 134217728
    assert c["step"]["bytes"] == 5 * S + 2 * bench.param_bytes(wl)
    assert c["step"]["bytes"] == pytest.approx(671.4e6, rel=1e-3)


def test_step_and_pass_rooflines_pick_the_slower_bound():
    wl = WORKLOADS["dw_k3_112_f32"]
    c = bench.algorithmic_counts(wl)
    peaks = {"hbm_gbs": 6528.7, "hbm_source": "m", "fp32_tflops": 74.45, "fp32_source": "n"}
    kernels = {"fwd": 0.05, "bwd_data": 0.05, "bwd_weight": 0.1}
    r = bench.pass_roofline(c, kernels, peaks)
    assert r["pass_name"] == "bwd_weight" and r["bound"] == "hbm"
    assert r["frac"] == pytest.approx(c["passes"]["bwd_weight"]["bytes"] / 0.1e-3 / 1e9 / 6528.7)
    s = bench.step_bound(c, 0.2, peaks)
    assert s["bound"] == "hbm"
    assert s["frac"] == pytest.approx(c["step"]["bytes"] / 6528.7e9 / 0.2e-3)
    wl3 = WORKLOADS["stage1_f32_k5_L3"]
    assert bench.step_bound(bench.algorithmic_counts(wl3), 0.2, peaks)["bound"] == "alu"


def test_launches_per_step_of_the_stage1_workload():
    """fold + output kernel for the forward, then the fused backward (fold,
    fused pass, finalize): five library kernels per step."""
    wl = WORKLOADS["stage1_f32_k5_L3"]
    desc = wt.make_desc(wl.N, wl.C, wl.H, wl.W, wl.k, wl.L, wl.io)
    assert bench.fused_backward(wt, desc)
    assert bench.launches_per_step(wt, desc) == 5


def test_launches_per_step_of_the_deep_workload():
    """Row-band planes: the backward passes run apart (forward: fold, deep
    kernel, output kernel; backward-data the same; weight gradients: one
    launch per level and the finalize)."""
    wl = WORKLOADS["deep_bf16_k5_L5"]
    desc = wt.make_desc(wl.N, wl.C, wl.H, wl.W, wl.k, wl.L, wl.io)
    assert not bench.fused_backward(wt, desc)
    assert bench.launches_per_step(wt, desc) == 3 + 3 + 6


def test_source_hash_ignores_comments_and_layout_only():
    a = "int f(int x) {  // doubles\n  return 2 * x;  /* no overflow check */\n}\n"
    b = "int f(int x) {\n    return 2 * x;\n}\n"
    c = "int f(int x) {\n  return 3 * x;\n}\n"
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)


def test_committed_traffic_is_used_only_while_the_sources_match(monkeypatch):
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    wl = "stage1_f32_k5_L3"
    monkeypatch.setattr(bench, "sources_sha256", lambda: rec["sources_sha256"])
    assert bench.load_traffic("fwd", wl) == rec[wl]["fwd"]
    monkeypatch.setattr(bench, "sources_sha256", lambda: "0" * 64)
    assert bench.load_traffic("fwd", wl) is None
