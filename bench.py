"""WTConv layer fwd+bwd benchmark on B200 (prints one JSON line on rank 0).

A step is one pass of the whole layer hot path over one batch: forward,
backward-data and backward-weight (the kernels of libwtconv).  The headline
workload is the largest single-GPU shape, the deep pyramid (N=16, C=64,
256x256, k=5, L=5, bf16 I/O); the same run times every other full-size
workload (stage-1 and stage-2 shapes, the two level-0 convs) and reports
them under `per_config`.

  python bench.py --gpus N --steps K --warmup W [--impl reference]

Timing: W untimed warm-up steps; then a barrier + synchronize, K timed steps
with CUDA events on the launching stream (each step preceded by an L2 flush
that writes a buffer larger than L2, outside the events), a synchronize +
barrier, and the max over ranks.  Per-pass times flush L2 before every pass
as well, so no pass reads what the previous one left in L2.  Multi-GPU runs
are data parallel with weak scaling: every rank runs the full per-GPU batch
and the parameter gradients are summed over ranks with one NCCL all-reduce
inside the step.
"""
import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import time

import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from depthwise_convolution_wtconv_b200.configs import WORKLOADS, BENCH_WORKLOAD, OTHER_WORKLOADS  # noqa: E402
from depthwise_convolution_wtconv_b200.inputs import make_inputs  # noqa: E402

METRIC = "WTConv layer fwd+bwd steps/s and achieved HBM GB/s (% of B200 peak)"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FP32_LANES_PER_SM = 128
L2_FLUSH_BYTES = 256 << 20
PASSES = ("fwd", "bwd_data", "bwd_weight")


def param_bytes(wl):
    """fp32 bytes of the layer's parameters (w0, b0, s0, wl, sl)."""
    k2 = wl.k * wl.k
    return 4 * (wl.C * k2 + 2 * wl.C + wl.L * wl.C * 4 * (k2 + 1))


def algorithmic_counts(wl):
    """Algorithmic FMAs and bytes of each pass and of the whole step.

    FMAs per pass: P*k^2*(1 + (4/3)(1 - 4^-L)) (the base conv plus the
    level-l convs on 4C channels at 4^-l of the pixels); the step is three
    times that.  Bytes: the minimal traffic of the layer.  A step must read
    x and write y (forward) and read x and dy and write dx (the backward
    passes together): 5S + 2 * params (S = bytes of one activation tensor;
    parameters read, gradients written).  Each pass on its own must move
    2S (forward: x, y; backward-data: dy, dx; weight gradients: x, dy) plus
    its parameters, so the three separate passes move 6S + 4 * params, the
    design traffic of running them as three passes.
    """
    P = wl.P
    fma = P * wl.k * wl.k * (1.0 + (4.0 / 3.0) * (1.0 - 4.0 ** (-wl.L)))
    S = P * wl.io_bytes
    prm = param_bytes(wl)
    passes = dict(fwd=dict(fma=fma, bytes=2 * S + prm),
                  bwd_data=dict(fma=fma, bytes=2 * S + prm),
                  bwd_weight=dict(fma=fma, bytes=2 * S + 2 * prm),
                  bwd=dict(fma=2 * fma, bytes=3 * S + 2 * prm))  # both backward passes in one
    step = dict(fma=3 * fma, bytes=5 * S + 2 * prm, design_bytes=6 * S + 4 * prm)
    return dict(passes=passes, step=step)


def fused_backward(wt, desc):
    """True when the library runs both backward passes of the shape as one
    fused pass (fewer launches for op 3 than for ops 1 and 2)."""
    return wt.kernel_launches(desc, 3) < wt.kernel_launches(desc, 1) + wt.kernel_launches(desc, 2)


def launches_per_step(wt, desc):
    """Kernels of this library launched per step (forward, then the fused
    backward or backward-data and backward-weight), as the library reports
    them for the shape."""
    if fused_backward(wt, desc):
        return wt.kernel_launches(desc, 0) + wt.kernel_launches(desc, 3)
    return sum(wt.kernel_launches(desc, op) for op in (0, 1, 2))


PASS_KERNELS = {
    "fwd": "wtconv_fold_kernel + wtconv_main_kernel (+ wtconv_deep_kernel for row-band planes)",
    "bwd_data": "wtconv_fold_kernel + wtconv_main_kernel, flipped (+ wtconv_deep_kernel for row-band planes)",
    "bwd_weight": "wtconv_bwdw_kernel + wtconv_bwdw_finalize (row-band planes: wtconv_bwband_kernel per level)",
    "bwd": "wtconv_fold_kernel + wtconv_bwd_fused_kernel + wtconv_bwdw_finalize (both backward passes)",
}


def load_peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "sm_max_mhz": 1965.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 20 ms from the
    first warm-up step to the end of the last timed region (a timed region
    of a few milliseconds alone would fall between two samples), plus one
    query right after the headline's timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.extra = []

    def _cmd(self, loop):
        cmd = ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits"]
        return cmd + (["-lms", "20"] if loop else [])

    def start(self):
        try:
            self.proc = subprocess.Popen(self._cmd(True), stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None

    def query_now(self):
        """One extra sample taken while the GPU is still warm."""
        try:
            out = subprocess.run(self._cmd(False), capture_output=True, text=True, timeout=10).stdout
            self.extra.extend(out.strip().splitlines())
        except (OSError, subprocess.SubprocessError):
            pass

    def stop(self):
        out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=10)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() + self.extra if r.strip()]
        sm, smax, reasons = [], [], set()
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
                for name, v in zip(self.NAMES, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(name)
            except (IndexError, ValueError):
                continue
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "window": "every 20 ms from the first warm-up step to the last timed step"}


def setup_dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        from datetime import timedelta
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(value, world, device):
    if world == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_inputs(wl, rank):
    """Inputs of one data-parallel rank: the parameters are the same on every
    rank (seed 0), the activations X and dY are this rank's own batch
    (seed = rank; rank 0 sees exactly the seed-0 workload)."""
    inp = make_inputs(wl, seed=0)
    if rank:
        mine = make_inputs(wl, seed=rank)
        inp["X"], inp["dY"] = mine["X"], mine["dY"]
    return inp


def allreduce_grads(flat, world):
    """Sums the parameter gradients over the ranks (the layer is a sum over
    the batch, so the sum of per-rank gradients is the global-batch one)."""
    if world > 1:
        dist.all_reduce(flat)


def grads_flat_views(wl, device):
    """One flat fp32 buffer with views for every parameter gradient (so the
    data-parallel all-reduce is a single collective)."""
    k2 = wl.k * wl.k
    sizes = [wl.C * k2, wl.C, wl.C, wl.L * wl.C * 4 * k2, wl.L * wl.C * 4]
    flat = torch.empty(sum(sizes), dtype=torch.float32, device=device)
    views, o = [], 0
    for s in sizes:
        views.append(flat[o:o + s])
        o += s
    g = dict(dw0=views[0].view(wl.C, wl.k, wl.k), db0=views[1], ds0=views[2],
             dwl=views[3].view(wl.L, wl.C, 4, wl.k, wl.k) if wl.L else None,
             dsl=views[4].view(wl.L, wl.C, 4) if wl.L else None)
    return flat, g


class Layer:
    """Device tensors, workspaces and captured graphs of one workload."""

    def __init__(self, wt, wl, device, rank):
        self.wt, self.wl, self.device = wt, wl, device
        dt = torch.float32 if wl.io == "f32" else torch.bfloat16
        self.dt = dt
        self.inp = rank_inputs(wl, rank)
        self.X = self.inp["X"].to(dt).to(device)
        self.dY = self.inp["dY"].to(dt).to(device)
        self.p = {k: self.inp[k].to(device) for k in ("W0", "b0", "s0")}
        self.Wl = self.inp["Wl"].to(device) if wl.L else None
        self.sl = self.inp["sl"].to(device) if wl.L else None
        self.Y = torch.empty_like(self.X)
        self.dX = torch.empty_like(self.X)
        self.gflat, self.grads = grads_flat_views(wl, device)
        self.desc = wt.make_desc(wl.N, wl.C, wl.H, wl.W, wl.k, wl.L, wl.io)
        self.ws = torch.empty(max(16, wt.workspace_size(self.desc, 3)), dtype=torch.uint8, device=device)
        self.ws2 = torch.empty(max(16, wt.workspace_size(self.desc, 2)), dtype=torch.uint8, device=device)
        self.graphs = {}
        self.step_graph = None
        self.fused = fused_backward(wt, self.desc)
        self.passes = PASSES + (("bwd",) if self.fused else ())
        self.step_backward = "two streams"

    def fwd(self, st, x=None, y=None):
        p = self.p
        self.wt.forward(self.X if x is None else x, p["W0"], p["b0"], p["s0"], self.Wl, self.sl,
                        y=self.Y if y is None else y, ws=self.ws, stream=st)

    def bwd_data(self, st, dy=None, dx=None):
        p = self.p
        self.wt.backward_data(self.dY if dy is None else dy, p["W0"], p["s0"], self.Wl, self.sl,
                              dx=self.dX if dx is None else dx, ws=self.ws, stream=st)

    def bwd_weight(self, st, x=None, dy=None, ws=None):
        p = self.p
        self.wt.backward_weight(self.X if x is None else x, self.dY if dy is None else dy, p["W0"], p["b0"],
                                p["s0"], self.Wl, self.sl, grads=self.grads, ws=self.ws if ws is None else ws,
                                stream=st)

    def bwd(self, st, x=None, dy=None, dx=None):
        p = self.p
        self.wt.backward(self.X if x is None else x, self.dY if dy is None else dy, p["W0"], p["b0"], p["s0"],
                         self.Wl, self.sl, dx=self.dX if dx is None else dx, grads=self.grads, ws=self.ws,
                         stream=st)

    def eager_step(self, st, x=None, dy=None, y=None, dx=None):
        self.fwd(st, x, y)
        if self.step_backward == "fused":
            self.bwd(st, x, dy, dx)
        else:
            self.bwd_data(st, dy, dx)
            self.bwd_weight(st, x, dy)

    def capture(self, stream, warmup, flush):
        """Each pass as a CUDA graph of its own, and the whole step as one
        graph: the forward, then the fused backward where the library fuses
        the shape's backward passes, else backward-data and the weight
        gradients, which are independent, on two streams (a workspace
        each)."""
        cap = torch.cuda.Stream(self.device)
        cap2 = torch.cuda.Stream(self.device)
        cap.wait_stream(stream)
        for name in self.passes:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                getattr(self, name)(cap)
            self.graphs[name] = g
        steps = {}
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            self.fwd(cap)
            cap2.wait_stream(cap)
            self.bwd_weight(cap2, ws=self.ws2)
            self.bwd_data(cap)
            cap.wait_stream(cap2)
        steps["two streams"] = g
        if self.fused:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                self.fwd(cap)
                self.bwd(cap)
            steps["fused"] = g
        stream.wait_stream(cap)
        for _ in range(warmup):
            flush.fill_(0.0)
            for name in self.passes:
                self.graphs[name].replay()
            for g in steps.values():
                flush.fill_(0.0)
                g.replay()
        torch.cuda.synchronize(self.device)
        # the step runs the faster of the two backward forms, timed here on
        # warm-up replays (L2 flushed before each)
        best = None
        for name, g in steps.items():
            t = 0.0
            for _ in range(max(3, warmup)):
                flush.fill_(0.0)
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g.replay()
                e1.record(stream)
                torch.cuda.synchronize(self.device)
                t += e0.elapsed_time(e1)
            if best is None or t < best[1]:
                best = (name, t)
        self.step_backward = best[0]
        self.step_graph = steps[best[0]]


def timed_steps(steps, run, flush, device, world, nev):
    """K steps, each after an L2 flush outside the events; returns the
    per-step event lists."""
    torch.cuda.synchronize(device)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(device)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(steps)]
    for i in range(steps):
        flush.fill_(0.0)
        run(evs[i])
    torch.cuda.synchronize(device)
    if world > 1:
        dist.barrier()
    return evs


def pass_roofline(counts, kernels, peaks):
    """The roofline of the slowest pass: its bound (FP32 ALUs or HBM, whichever
    needs more time for the pass's algorithmic work), the achieved rate and the
    fraction of the peak."""
    dom = max(kernels, key=kernels.get)
    dom_ms = kernels[dom]
    c = counts["passes"][dom]
    t_alu = 2 * c["fma"] / (peaks["fp32_tflops"] * 1e12)
    t_hbm = c["bytes"] / (peaks["hbm_gbs"] * 1e9)
    if t_hbm > t_alu:
        achieved = c["bytes"] / (dom_ms * 1e-3) / 1e9
        return dict(pass_name=dom, bound="hbm", achieved=achieved, peak=peaks["hbm_gbs"], unit="GB/s",
                    frac=achieved / peaks["hbm_gbs"], peak_source=peaks["hbm_source"])
    achieved = 2 * c["fma"] / (dom_ms * 1e-3) / 1e12
    return dict(pass_name=dom, bound="alu", achieved=achieved, peak=peaks["fp32_tflops"], unit="TFLOP/s",
                frac=achieved / peaks["fp32_tflops"], peak_source=peaks["fp32_source"])


def step_bound(counts, ms_per_step, peaks):
    """Roofline of the whole step: t_ALU and t_HBM of its algorithmic FMAs and
    bytes, and max(t_ALU, t_HBM) / measured time."""
    t_alu = 2 * counts["step"]["fma"] / (peaks["fp32_tflops"] * 1e12) * 1e6
    t_hbm = counts["step"]["bytes"] / (peaks["hbm_gbs"] * 1e9) * 1e6
    return dict(t_alu_us=t_alu, t_hbm_us=t_hbm, bound="alu" if t_alu > t_hbm else "hbm",
                frac=max(t_alu, t_hbm) / (ms_per_step * 1e3))


def measure(layer, args, world, flush, stream, peaks):
    """Times one workload: the whole-step graph (the metric), each pass's
    graph with L2 flushed before it and back to back, and eager calls."""
    wl, device = layer.wl, layer.device
    for _ in range(args.warmup):
        flush.fill_(0.0)
        layer.eager_step(stream)
    torch.cuda.synchronize(device)
    layer.capture(stream, args.warmup, flush)

    names = layer.passes

    def per_pass_flushed(ev):
        for i, name in enumerate(names):
            if i:
                flush.fill_(0.0)
            ev[2 * i].record(stream)
            layer.graphs[name].replay()
            ev[2 * i + 1].record(stream)

    def per_pass_warm(ev):
        ev[0].record(stream)
        for i, name in enumerate(names):
            layer.graphs[name].replay()
            ev[i + 1].record(stream)

    def whole(ev):
        ev[0].record(stream)
        layer.step_graph.replay()
        allreduce_grads(layer.gflat, world)
        ev[1].record(stream)

    def eager(ev):
        ev[0].record(stream)
        layer.eager_step(stream)
        allreduce_grads(layer.gflat, world)
        ev[1].record(stream)

    K = args.steps
    evs = timed_steps(K, per_pass_flushed, flush, device, world, 2 * len(names))
    kernels = {n: max_over_ranks(sum(e[2 * i].elapsed_time(e[2 * i + 1]) for e in evs) / K, world, device)
               for i, n in enumerate(names)}
    evs = timed_steps(K, per_pass_warm, flush, device, world, len(names) + 1)
    warm = {n: max_over_ranks(sum(e[i].elapsed_time(e[i + 1]) for e in evs) / K, world, device)
            for i, n in enumerate(names)}
    evs = timed_steps(K, eager, flush, device, world, 2)
    eager_ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in evs), world, device) / K
    t_wall = time.perf_counter()
    evs = timed_steps(K, whole, flush, device, world, 2)
    t_wall = time.perf_counter() - t_wall
    ms_per_step = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in evs), world, device) / K

    counts = algorithmic_counts(wl)
    # the roofline of the slowest pass the step runs
    step_passes = ("fwd", "bwd") if layer.step_backward == "fused" else PASSES
    roof = pass_roofline(counts, {n: kernels[n] for n in step_passes}, peaks)
    hbm_gbs = counts["step"]["bytes"] / (ms_per_step * 1e-3) / 1e9
    return dict(
        workload=wl.name, ms_per_step=ms_per_step, value=world * 1000.0 / ms_per_step, unit="steps/s",
        kernels_ms=kernels, kernels_ms_warm=warm, fused_backward=layer.fused,
        step_backward=layer.step_backward,
        roofline=roof,
        step_roofline=step_bound(counts, ms_per_step, peaks),
        hbm={"achieved_gbs": hbm_gbs, "peak_gbs": peaks["hbm_gbs"], "frac": hbm_gbs / peaks["hbm_gbs"],
             "algorithmic_bytes_per_step": counts["step"]["bytes"],
             "design_bytes_per_step": counts["step"]["design_bytes"], "peak_source": peaks["hbm_source"]},
        eager={"ms_per_step": eager_ms, "value": world * 1000.0 / eager_ms, "unit": "steps/s"},
        gpu_launches_per_step=(launches_per_step(layer.wt, layer.desc) if layer.step_backward == "fused" else
                               sum(layer.wt.kernel_launches(layer.desc, op) for op in (0, 1, 2))),
        wall_s_timed_region=t_wall,
    )


def end_to_end(layer, args, world, stream):
    """The same step end to end through the public API: pinned host inputs
    copied in and the results (y, dx, the gradients) copied out every step.
    Steps are pipelined as a data loader would run them: copies in on one
    stream, the passes on the compute stream, copies out on a third, with
    device buffers alternating between steps, so that step i+1's copies in
    and step i-1's copies out (opposite PCIe directions) overlap step i's
    passes."""
    device, dt = layer.device, layer.dt
    hX = layer.inp["X"].to(dt).pin_memory()
    hdY = layer.inp["dY"].to(dt).pin_memory()
    hY = torch.empty_like(hX).pin_memory()
    hdX = torch.empty_like(hX).pin_memory()
    hg = torch.empty_like(layer.gflat, device="cpu").pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    cin, cout = torch.cuda.Stream(device), torch.cuda.Stream(device)
    X = layer.X
    bufs = [dict(x=torch.empty_like(X), dy=torch.empty_like(X), y=torch.empty_like(X), dx=torch.empty_like(X),
                 g=torch.empty_like(layer.gflat)) for _ in range(2)]
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for b in range(2):  # every event recorded once before its first wait
        ev_comp[b].record(stream)
        ev_out[b].record(stream)

    def e2e_step(i):
        b = bufs[i % 2]
        cin.wait_event(ev_comp[i % 2])       # the passes two steps back are done with these inputs
        with torch.cuda.stream(cin):
            b["x"].copy_(hX, non_blocking=True)
            b["dy"].copy_(hdY, non_blocking=True)
        ev_in[i % 2].record(cin)
        stream.wait_event(ev_in[i % 2])
        stream.wait_event(ev_out[i % 2])     # the copies out two steps back are done with these outputs
        layer.eager_step(stream, b["x"], b["dy"], b["y"], b["dx"])
        allreduce_grads(layer.gflat, world)
        b["g"].copy_(layer.gflat)
        ev_comp[i % 2].record(stream)
        cout.wait_event(ev_comp[i % 2])
        with torch.cuda.stream(cout):
            hY.copy_(b["y"], non_blocking=True)
            hdX.copy_(b["dx"], non_blocking=True)
            hg.copy_(b["g"], non_blocking=True)
        ev_out[i % 2].record(cout)

    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize(device)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    cin.wait_stream(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_stream(cout)
    e1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, device) / e2e_steps
    h2d = 2 * X.numel() * X.element_size()
    d2h = 2 * X.numel() * X.element_size() + layer.gflat.numel() * 4
    return {"value": world * 1000.0 / e2e_ms, "unit": "steps/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": e2e_steps,
            "overlap": "copies in and out on their own streams, device buffers alternating between steps"}


def device_peaks(device):
    peaks, src = load_peaks()
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    sm_max = float(peaks.get("sm_max_mhz", 1965.0))
    return {"hbm_gbs": float(peaks["hbm_gbs"]), "hbm_source": f"{src} copy bandwidth",
            "fp32_tflops": sms * FP32_LANES_PER_SM * 2 * sm_max * 1e6 / 1e12,
            "fp32_source": f"{sms} SMs x {FP32_LANES_PER_SM} FP32 lanes x 2 x {sm_max:.0f} MHz "
                           f"(an FFMA probe reached 97% of it: profiles/ffma_peak_probe.md)"}


def run_ours(args, wl, world, rank, local):
    import depthwise_convolution_wtconv_b200 as wt
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    peaks = device_peaks(device)
    sampler = ClockSampler(local)
    sampler.start()

    layer = Layer(wt, wl, device, rank)
    m = measure(layer, args, world, flush, stream, peaks)
    sampler.query_now()
    e2e = end_to_end(layer, args, world, stream)
    counts = algorithmic_counts(wl)
    roof = dict(m["roofline"])
    dom = roof.pop("pass_name")
    traffic = load_traffic(dom, wl.name)
    line = {
        "metric": METRIC,
        "value": m["value"],
        "unit": "steps/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": m["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32" if wl.io == "f32" else "bf16-io/f32",
        "data": "synthetic (seeded N(0,1) activations, N(0,1/k^2) weights, U(0.5,1.5) scales)",
        "config": {"workload": wl.name, **{k: v for k, v in wl.as_dict().items() if k != "name"},
                   "global_batch": wl.N * world, "parallelism": f"dp{world}",
                   "l2": "flushed before every timed step (256 MiB write); per-pass times flushed before "
                         "every pass"},
        "roofline": {"bound": roof["bound"], "kernel": f"{dom} pass: {PASS_KERNELS[dom]}",
                     "achieved": roof["achieved"], "peak": roof["peak"], "unit": roof["unit"],
                     "frac": roof["frac"], "traffic": traffic,
                     "traffic_source": ("profiles/traffic.json (ncu dram__bytes_read.sum + dram__bytes_write.sum "
                                        "of the pass's kernels, per launch, same sources)" if traffic is not None
                                        else "none: no ncu capture of the current sources"),
                     "peak_source": roof["peak_source"]},
        "step_roofline": m["step_roofline"],
        "hbm": m["hbm"],
        "fma_per_step": counts["step"]["fma"],
        "kernels_ms": m["kernels_ms"],
        "kernels_ms_warm": m["kernels_ms_warm"],
        "fused_backward": m["fused_backward"],
        "step_backward": m["step_backward"],
        "timing": ("the whole step one CUDA graph replay: the forward, then the backward as step_backward "
                   "says (\"fused\": one wtconv_backward call; \"two streams\": backward-data and weight "
                   "gradients on two streams with a workspace each; where the library fuses the shape's "
                   "backward, the faster of the two on warm-up replays); kernels_ms: one graph per pass (bwd: "
                   "wtconv_backward), L2 flushed before each pass; kernels_ms_warm: the pass graphs back to "
                   "back; CUDA events on the launching stream"),
        "eager": m["eager"],
        "e2e": e2e,
        "gpu_launches": m["gpu_launches_per_step"] * args.steps,
        "wall_s_timed_region": m["wall_s_timed_region"],
    }
    if rank == 0 and not args.no_comparators:
        extra = (layer.Y.numel() + layer.dX.numel()) * layer.Y.element_size() + layer.gflat.numel() * 4 + \
            layer.ws.numel()
        line["comparators"] = comparators(wl, device, layer.inp, lambda: layer.eager_step(stream), extra)
    del layer
    torch.cuda.empty_cache()
    if not args.no_per_config:
        per = {}
        for name in OTHER_WORKLOADS:
            if name == wl.name:
                continue
            other = Layer(wt, WORKLOADS[name], device, rank)
            e = measure(other, args, world, flush, stream, peaks)
            r = dict(e["roofline"])
            e["roofline"] = {**r, "traffic": load_traffic(r["pass_name"], name)}
            if rank == 0 and not args.no_comparators:
                e["comparators"] = comparators(other.wl, device, other.inp, lambda: other.eager_step(stream),
                                               None, steps=10)
            del e["wall_s_timed_region"]
            per[name] = e
            del other
            torch.cuda.empty_cache()
        line["per_config"] = per
    line["clocks"] = sampler.stop()
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_seconds)
    return line


def _code_only(text):
    """C/C++ source without comments and whitespace (a comment edit does not
    change a kernel)."""
    import re
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "".join(text.split())


def sources_sha256():
    """Hash of the CUDA sources' code, to tell whether committed counters
    still apply."""
    import glob
    import hashlib
    paths = sorted(glob.glob(os.path.join(ROOT, "depthwise_convolution_wtconv_b200", "csrc", "*")))
    return hashlib.sha256("".join(_code_only(open(p).read()) for p in paths).encode()).hexdigest()


def torch_cascade(X, W0, b0, s0, Wl, sl):
    """The layer composed from plain PyTorch GPU ops, written here as a
    comparator (the unfused cascade, as a framework user would write it):
    grouped conv2d for the depthwise convs, a stride-2 grouped conv2d with
    the +-1/2 Haar taps for the analysis, conv_transpose2d for the synthesis;
    autograd for the backward.  Every subband, Z and LL tensor goes through
    HBM and is kept for the backward."""
    import torch.nn.functional as F
    C, k = X.shape[1], W0.shape[-1]
    L = 0 if Wl is None else Wl.shape[0]
    h = 0.5
    filt = torch.tensor([[[h, h], [h, h]], [[h, h], [-h, -h]], [[h, -h], [h, -h]], [[h, -h], [-h, h]]],
                        dtype=X.dtype, device=X.device).repeat(C, 1, 1).unsqueeze(1)
    Y = s0.view(1, C, 1, 1) * F.conv2d(X, W0.unsqueeze(1), b0, padding=k // 2, groups=C)
    cur, Zs = X, []
    for lv in range(L):
        sub = F.conv2d(cur, filt, stride=2, groups=C)
        Zs.append(F.conv2d(sub, Wl[lv].reshape(4 * C, 1, k, k), padding=k // 2, groups=4 * C)
                  * sl[lv].reshape(1, 4 * C, 1, 1))
        cur = sub[:, 0::4]
    t = None
    for lv in reversed(range(L)):
        Z = Zs[lv]
        if t is not None:
            Z = torch.cat([(Z[:, 0::4] + t).unsqueeze(2), Z.view(Z.shape[0], C, 4, *Z.shape[2:])[:, :, 1:]],
                          dim=2).view_as(Z)
        t = F.conv_transpose2d(Z, filt, stride=2, groups=C)
    return Y if t is None else Y + t


def diagonalwise_conv(X, W0, b0, s0, block=32):
    """The level-0 layer (a depthwise conv with bias and per-channel scale) by
    diagonalwise refactorization ("Diagonalwise Refactorization: An Efficient
    Training Method for Depthwise Convolutions", abstract): the channels are
    taken in blocks of `block`, and each block's depthwise kernels are placed
    on the diagonal of one dense block x block weight, so that the depthwise
    conv becomes a grouped dense conv with C / block groups.  Channels are
    zero-padded to a multiple of the block (the padded outputs are dropped).
    s0 * (dwconv(X, W0) + b0), differentiable by autograd."""
    import torch.nn.functional as F
    N, C, H, W = X.shape
    k = W0.shape[-1]
    G = min(block, C)
    Cp = (C + G - 1) // G * G
    if Cp != C:
        X = F.pad(X, (0, 0, 0, 0, 0, Cp - C))
        W0 = F.pad(W0, (0, 0, 0, 0, 0, Cp - C))
        b0 = F.pad(b0, (0, Cp - C))
    groups = Cp // G
    eye = torch.eye(G, dtype=X.dtype, device=X.device).view(1, G, G, 1, 1)
    w = (W0.view(groups, G, 1, k, k) * eye).reshape(Cp, G, k, k)
    Y = F.conv2d(X, w, b0, padding=k // 2, groups=groups)[:, :C]
    return s0.view(1, -1, 1, 1) * Y


def comparators(wl, device, inp, ours_step, ours_extra_bytes, steps=20):
    """Same-GPU comparators of one fwd+bwd step (not part of the timed
    metric): the plain PyTorch cascade (time and peak memory beyond the
    inputs), and for L = 0 the diagonalwise-refactorized conv
    (`diagonalwise_conv`).  fp32 arithmetic on fp32 copies of the inputs."""
    X = inp["X"].float().to(device).requires_grad_(True)
    dY = inp["dY"].float().to(device)
    P = {kk: inp[kk].to(device).requires_grad_(True) for kk in ("W0", "b0", "s0")}
    Wl = inp["Wl"].to(device).requires_grad_(True) if wl.L else None
    sl = inp["sl"].to(device).requires_grad_(True) if wl.L else None
    leaves = [X, P["W0"], P["b0"], P["s0"]] + ([Wl, sl] if wl.L else [])

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize(device)
        base = torch.cuda.memory_allocated(device)
        torch.cuda.reset_peak_memory_stats(device)
        fn()
        torch.cuda.synchronize(device)
        peak = torch.cuda.max_memory_allocated(device) - base
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(steps):
            fn()
        e1.record()
        torch.cuda.synchronize(device)
        return e0.elapsed_time(e1) / steps, peak

    def cascade_step():
        for t in leaves:
            t.grad = None
        Y = torch_cascade(X, P["W0"], P["b0"], P["s0"], Wl, sl)
        Y.backward(dY)

    out = {}
    ms, peak = timed(cascade_step)
    ours_ms, _ = timed(ours_step)
    out["torch_cascade"] = {"ms_per_step": ms, "peak_extra_bytes": peak,
                            "what": "plain PyTorch ops (grouped conv2d, Haar as stride-2 conv, conv_transpose2d) "
                                    "+ autograd, fp32"}
    out["ours_eager_ms_per_step"] = ours_ms
    out["speedup_vs_torch_cascade"] = ms / ours_ms
    if ours_extra_bytes is not None:
        out["ours_extra_bytes"] = ours_extra_bytes
        out["memory_ratio_vs_torch_cascade"] = peak / max(1, ours_extra_bytes)
    if wl.L == 0:
        def diag_step():
            for t in leaves:
                t.grad = None
            diagonalwise_conv(X, P["W0"], P["b0"], P["s0"]).backward(dY)

        dms, dpeak = timed(diag_step)
        out["diagonalwise_refactorization"] = {"ms_per_step": dms, "peak_extra_bytes": dpeak,
                                               "block": min(32, wl.C), "speedup_of_ours": dms / ours_ms}
    return out


def load_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, or None when it
    is missing or the kernels changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    if d.get("sources_sha256") != sources_sha256():
        return None
    return d.get(workload, {}).get(kernel)


def oracle_step(p):
    import oracle
    oracle.forward(p["X"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    oracle.backward(p["X"], p["dY"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])


def _plane_sample(wl, planes):
    """Sub-workload of `planes` (n, c) planes: the first channels of the
    first batch entries, with every other dimension unchanged."""
    planes = max(1, min(planes, wl.N * wl.C))
    if planes >= wl.C:
        return dataclasses.replace(wl, N=planes // wl.C), (planes // wl.C) * wl.C
    return dataclasses.replace(wl, N=1, C=planes), planes


def _oracle_seconds_per_plane(wl):
    """Oracle seconds per (n, c) plane, from one step on a few planes."""
    from depthwise_convolution_wtconv_b200.inputs import as_float64
    from threadpoolctl import threadpool_limits
    cal, cal_planes = _plane_sample(wl, min(8, wl.N * wl.C))
    pc = as_float64(make_inputs(cal, 0))
    with threadpool_limits(limits=1):
        t = time.perf_counter()
        oracle_step(pc)
        return (time.perf_counter() - t) / cal_planes


def cpu_baseline(wl, seconds):
    """The float64 oracle, as it stands, timed on one host core on a bounded
    sample of the same workload: as many (n, c) planes as take about
    `seconds`, the rate scaled to the whole workload."""
    from depthwise_convolution_wtconv_b200.inputs import as_float64
    from threadpoolctl import threadpool_limits
    tau = _oracle_seconds_per_plane(wl)
    sub, planes = _plane_sample(wl, int(seconds / max(1e-9, tau)))
    p = as_float64(make_inputs(sub, 0))
    with threadpool_limits(limits=1):
        t = time.perf_counter()
        oracle_step(p)
        dt = time.perf_counter() - t
    frac = planes / (wl.N * wl.C)
    return {"value": frac / dt, "unit": "steps/s", "cores": 1, "kind": "oracle",
            "sample": f"{planes} of {wl.N * wl.C} (n, c) planes ({sub.N}x{sub.C}x{wl.H}x{wl.W}, k={wl.k}, "
                      f"L={wl.L}), one fwd+bwd in numpy float64, single-threaded; host has {os.cpu_count()} "
                      f"cores; rate scaled by {planes}/{wl.N * wl.C}",
            "seconds": dt}


def run_reference(args, wl, world, rank):
    """The oracle as the reference arm: rank 0 only, on the host cores.
    Each step runs the oracle on a bounded plane sample sized so that the
    whole run stays near two minutes; the rate is scaled to the workload."""
    if rank != 0:
        return None
    from depthwise_convolution_wtconv_b200.inputs import as_float64
    from threadpoolctl import threadpool_limits
    tau = _oracle_seconds_per_plane(wl)
    planes = int(120.0 / max(1e-9, (args.steps + args.warmup) * tau))
    sub, planes = _plane_sample(wl, planes)
    p = as_float64(make_inputs(sub, 0))
    with threadpool_limits(limits=1):
        for _ in range(args.warmup):
            oracle_step(p)
        t = time.perf_counter()
        for _ in range(args.steps):
            oracle_step(p)
        dt = (time.perf_counter() - t) / args.steps
    frac = planes / (wl.N * wl.C)
    value = frac / dt
    sample = (f"{planes} of {wl.N * wl.C} (n, c) planes per step ({sub.N}x{sub.C}x{wl.H}x{wl.W}), numpy float64, "
              f"single-threaded, rate scaled by {planes}/{wl.N * wl.C}")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 / value, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, **{k: v for k, v in wl.as_dict().items() if k != "name"},
                   "global_batch": wl.N, "parallelism": "host (rank 0 only, one core)"},
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": 1, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


FFMA_PROBE_SRC = r"""
// FP32 FMA throughput probe: every thread runs 8 independent FMA chains
// (scalar) or 8 independent chains of packed pairs (fma.rn.f32x2, two FMAs
// per instruction); the results are summed and stored so nothing is dropped.
#include <cuda_runtime.h>
__global__ void __launch_bounds__(512) ffma_scalar(float* out, int iters, float a, float b) {
  float x[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) x[j] = threadIdx.x * 1e-3f + j;
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int u = 0; u < 16; ++u)
#pragma unroll
      for (int j = 0; j < 8; ++j) x[j] = fmaf(x[j], a, b);
  }
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) s += x[j];
  out[blockIdx.x * blockDim.x + threadIdx.x] = s;
}
__global__ void __launch_bounds__(512) ffma_packed(float* out, int iters, float a, float b) {
  unsigned long long x[8];
  float2 av = make_float2(a, a), bv = make_float2(b, b);
  const unsigned long long A = *reinterpret_cast<unsigned long long*>(&av);
  const unsigned long long B = *reinterpret_cast<unsigned long long*>(&bv);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float2 t = make_float2(threadIdx.x * 1e-3f + j, j + 0.5f);
    x[j] = *reinterpret_cast<unsigned long long*>(&t);
  }
  for (int i = 0; i < iters; ++i) {
#pragma unroll
    for (int u = 0; u < 8; ++u)
#pragma unroll
      for (int j = 0; j < 8; ++j) asm volatile("fma.rn.f32x2 %0, %0, %1, %2;" : "+l"(x[j]) : "l"(A), "l"(B));
  }
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float2 t = *reinterpret_cast<float2*>(&x[j]);
    s += t.x + t.y;
  }
  out[blockIdx.x * blockDim.x + threadIdx.x] = s;
}
extern "C" int ffma_probe_launch(int packed, float* out, int blocks, int threads, int iters, void* stream) {
  if (packed) ffma_packed<<<blocks, threads, 0, (cudaStream_t)stream>>>(out, iters, 0.999f, 1e-3f);
  else ffma_scalar<<<blocks, threads, 0, (cudaStream_t)stream>>>(out, iters, 0.999f, 1e-3f);
  return (int)cudaGetLastError();
}
"""


def ffma_probe():
    """Measures the FP32 FMA rate the ALU roofline rests on: a throughput
    kernel (compiled here for sm_100a with nvcc) of independent FMA chains,
    scalar and packed, timed with CUDA events; 128 FMAs per thread and loop
    iteration in both forms."""
    import ctypes
    import tempfile
    device = torch.device("cuda", 0)
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    with tempfile.TemporaryDirectory() as d:
        src, lib = os.path.join(d, "probe.cu"), os.path.join(d, "probe.so")
        open(src, "w").write(FFMA_PROBE_SRC)
        subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-shared", "-Xcompiler",
                        "-fPIC", "-o", lib, src], check=True)
        so = ctypes.CDLL(lib)
        blocks, threads, iters = sms * 4, 512, 4096
        out = torch.empty(blocks * threads, dtype=torch.float32, device=device)
        st = torch.cuda.current_stream(device)
        res = {}
        sampler = ClockSampler(0)
        sampler.start()
        for name, packed in (("scalar", 0), ("packed_f32x2", 1)):
            for _ in range(3):
                so.ffma_probe_launch(packed, ctypes.c_void_p(out.data_ptr()), blocks, threads, iters,
                                     ctypes.c_void_p(st.cuda_stream))
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
            reps = 20
            for _ in range(reps):
                rc = so.ffma_probe_launch(packed, ctypes.c_void_p(out.data_ptr()), blocks, threads, iters,
                                          ctypes.c_void_p(st.cuda_stream))
                if rc:
                    raise RuntimeError(f"probe launch failed: {rc}")
            e1.record(st)
            torch.cuda.synchronize(device)
            ms = e0.elapsed_time(e1) / reps
            fma = blocks * threads * iters * 128
            res[name] = {"tfma_per_s": fma / (ms * 1e-3) / 1e12, "ms": ms}
        clocks = sampler.stop()
    peak = sms * FP32_LANES_PER_SM * 1965e6 / 1e12
    return {"probe": "ffma", "sms": sms, "nominal_tfma_per_s_at_1965_mhz": peak,
            **{k: {**v, "frac_of_nominal": v["tfma_per_s"] / peak} for k, v in res.items()}, "clocks": clocks}


def passes_once(wl_name, reps, batch=0):
    """Runs every pass of a workload `reps` times, eagerly and untimed (for
    profiler captures: each pass's kernels appear in order forward,
    backward-data, weight gradients, and the fused backward where the
    library fuses the shape's backward passes); `batch` > 0 replaces N
    (a smaller case of the same kernels)."""
    import depthwise_convolution_wtconv_b200 as wt
    device = torch.device("cuda", 0)
    wl = WORKLOADS[wl_name]
    if batch:
        wl = dataclasses.replace(wl, N=batch)
    layer = Layer(wt, wl, device, 0)
    st = torch.cuda.current_stream(device)
    for _ in range(reps):
        for name in layer.passes:
            getattr(layer, name)(st)
    torch.cuda.synchronize(device)
    return {"workload": wl_name, "N": wl.N, "passes": list(layer.passes), "reps": reps,
            "launches": {name: wt.kernel_launches(layer.desc, op) for name, op in
                         (("fwd", 0), ("bwd_data", 1), ("bwd_weight", 2), ("bwd", 3))}}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=BENCH_WORKLOAD, choices=list(WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="about how long the oracle's CPU-baseline sample runs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="time the headline workload only")
    ap.add_argument("--no-comparators", action="store_true", help="skip the same-GPU PyTorch comparators")
    ap.add_argument("--ffma-probe", action="store_true", help="measure the FP32 FMA rate and exit")
    ap.add_argument("--passes-once", type=int, default=0, metavar="R",
                    help="run every pass of --workload R times, untimed (for profiler captures), and exit")
    ap.add_argument("--batch", type=int, default=0, help="with --passes-once: batch size N in place of the workload's")
    args = ap.parse_args(argv)
    if args.ffma_probe:
        print(json.dumps(ffma_probe()), flush=True)
        return
    if args.passes_once:
        print(json.dumps(passes_once(args.workload, args.passes_once, args.batch)), flush=True)
        return
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = WORKLOADS[args.workload]
    world, rank, local = setup_dist()
    try:
        if args.impl == "reference":
            line = run_reference(args, wl, world, rank)
        else:
            line = run_ours(args, wl, world, rank, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
