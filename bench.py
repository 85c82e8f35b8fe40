"""WTConv layer fwd+bwd benchmark on B200 (prints one JSON line on rank 0).

A step is one pass of the whole layer hot path over one batch: forward,
backward-data and backward-weight (the kernels of libwtconv) on the
ConvNeXt-T stage-1 shape (N=32, C=96, 56x56, k=5, L=3, fp32) by default.

  python bench.py --gpus N --steps K --warmup W [--impl reference]

Timing: W untimed warm-up steps; then a barrier + synchronize, K timed steps
with CUDA events on the launching stream (each step preceded by an L2 flush
that writes a buffer larger than L2, outside the events), a synchronize +
barrier, and the max over ranks.  Multi-GPU runs are data parallel with
weak scaling: every rank runs the full per-GPU batch and the parameter
gradients are summed over ranks with one NCCL all-reduce inside the step.
"""
import argparse
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

from depthwise_convolution_wtconv_b200.configs import WORKLOADS, BENCH_WORKLOAD  # noqa: E402
from depthwise_convolution_wtconv_b200.inputs import make_inputs  # noqa: E402

METRIC = "WTConv layer fwd+bwd steps/s and achieved HBM GB/s (% of B200 peak)"
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
SM_COUNT_NOMINAL = 148
FP32_LANES_PER_SM = 128
L2_FLUSH_BYTES = 256 << 20


def algorithmic_counts(wl):
    """Per-launch algorithmic FMAs and bytes of each pass (fp32 arithmetic).

    FMAs: P*k^2*(1 + (4/3)(1 - 4^-L)) per pass (base conv plus the level-l
    convs on 4C channels at 4^-l of the pixels).  Bytes: forward reads x and
    writes y; backward-data reads dy, writes dx; backward-weight reads x and
    dy; parameters (and gradients) are counted once per pass they touch.
    """
    P = wl.P
    k2 = wl.k * wl.k
    fma = P * k2 * (1.0 + (4.0 / 3.0) * (1.0 - 4.0 ** (-wl.L)))
    S = P * wl.io_bytes
    params = 4 * (wl.C * k2 + 2 * wl.C + wl.L * wl.C * 4 * (k2 + 1))
    return dict(
        fwd=dict(fma=fma, bytes=2 * S + params),
        bwd_data=dict(fma=fma, bytes=2 * S + params),
        bwd_weight=dict(fma=fma, bytes=2 * S + 2 * params),
    )


def launches_per_step(wt, desc):
    """Kernels of this library launched per step (forward, backward-data,
    backward-weight), as the library reports them for the shape."""
    return sum(wt.kernel_launches(desc, op) for op in (0, 1, 2))


PASS_KERNELS = {
    "fwd": "wtconv_fold_kernel + wtconv_main_kernel (+ wtconv_deep_kernel for row-band planes)",
    "bwd_data": "wtconv_fold_kernel + wtconv_main_kernel, flipped (+ wtconv_deep_kernel for row-band planes)",
    "bwd_weight": "wtconv_bwdw_kernel + wtconv_bwdw_finalize (row-band planes: wtconv_bwband_kernel per level)",
}


def load_peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "sm_max_mhz": 1965.0}, "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = [r.split(",") for r in out.strip().splitlines() if r.strip()]
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax.append(float(r[2]))
                for name, v in zip(names, r[5:9]):
                    if v.strip().lower() == "active":
                        reasons.add(name)
            except (IndexError, ValueError):
                continue
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


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


def run_ours(args, wl, world, rank, local):
    import depthwise_convolution_wtconv_b200 as wt
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dt = torch.float32 if wl.io == "f32" else torch.bfloat16
    inp = rank_inputs(wl, rank)
    X = inp["X"].to(dt).to(device)
    dY = inp["dY"].to(dt).to(device)
    p = {k: inp[k].to(device) for k in ("W0", "b0", "s0")}
    Wl = inp["Wl"].to(device) if wl.L else None
    sl = inp["sl"].to(device) if wl.L else None
    Y = torch.empty_like(X)
    dX = torch.empty_like(X)
    gflat, grads = grads_flat_views(wl, device)
    desc = wt.make_desc(wl.N, wl.C, wl.H, wl.W, wl.k, wl.L, wl.io)
    ws = torch.empty(max(16, wt.workspace_size(desc, 3)), dtype=torch.uint8, device=device)
    ws2 = torch.empty(max(16, wt.workspace_size(desc, 2)), dtype=torch.uint8, device=device)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def step(ev=None, x=X, dy=dY, y=Y, dx=dX, st=stream):
        if ev is not None:
            ev[0].record(stream)
        wt.forward(x, p["W0"], p["b0"], p["s0"], Wl, sl, y=y, ws=ws, stream=st)
        if ev is not None:
            ev[1].record(stream)
        wt.backward_data(dy, p["W0"], p["s0"], Wl, sl, dx=dx, ws=ws, stream=st)
        if ev is not None:
            ev[2].record(stream)
        wt.backward_weight(x, dy, p["W0"], p["b0"], p["s0"], Wl, sl, grads=grads, ws=ws, stream=st)
        if ev is not None:
            ev[3].record(stream)
        allreduce_grads(gflat, world)
        if ev is not None:
            ev[4].record(stream)

    for _ in range(args.warmup):
        flush.fill_(0.0)
        step()
    torch.cuda.synchronize(device)

    # each pass captured once as a CUDA graph (the same kernels, launched
    # without per-call host work); the gradient all-reduce stays eager
    graphs = []
    step_graph = None
    if not args.eager:
        cap = torch.cuda.Stream(device)
        cap.wait_stream(stream)
        for fn in (lambda: wt.forward(X, p["W0"], p["b0"], p["s0"], Wl, sl, y=Y, ws=ws, stream=cap),
                   lambda: wt.backward_data(dY, p["W0"], p["s0"], Wl, sl, dx=dX, ws=ws, stream=cap),
                   lambda: wt.backward_weight(X, dY, p["W0"], p["b0"], p["s0"], Wl, sl, grads=grads, ws=ws,
                                              stream=cap)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                fn()
            graphs.append(g)
        stream.wait_stream(cap)
        for _ in range(args.warmup):
            flush.fill_(0.0)
            for g in graphs:
                g.replay()
        torch.cuda.synchronize(device)
        # the whole step as one graph: the forward, then backward-data and the
        # weight gradients, which are independent, on two streams (each with
        # its own workspace), joined before the all-reduce
        cap2 = torch.cuda.Stream(device)
        step_graph = torch.cuda.CUDAGraph()
        cap.wait_stream(stream)
        with torch.cuda.graph(step_graph, stream=cap):
            wt.forward(X, p["W0"], p["b0"], p["s0"], Wl, sl, y=Y, ws=ws, stream=cap)
            cap2.wait_stream(cap)
            wt.backward_weight(X, dY, p["W0"], p["b0"], p["s0"], Wl, sl, grads=grads, ws=ws2, stream=cap2)
            wt.backward_data(dY, p["W0"], p["s0"], Wl, sl, dx=dX, ws=ws, stream=cap)
            cap.wait_stream(cap2)
        stream.wait_stream(cap)
        for _ in range(args.warmup):
            flush.fill_(0.0)
            step_graph.replay()
        torch.cuda.synchronize(device)

    def graph_step(ev):
        ev[0].record(stream)
        for i, g in enumerate(graphs):
            g.replay()
            ev[i + 1].record(stream)
        allreduce_grads(gflat, world)
        ev[4].record(stream)

    def whole_step(ev):
        ev[0].record(stream)
        step_graph.replay()
        allreduce_grads(gflat, world)
        ev[4].record(stream)

    def timed(run):
        torch.cuda.synchronize(device)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(device)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(args.steps)]
        sampler = ClockSampler(local)
        sampler.start()
        t_wall = time.perf_counter()
        for i in range(args.steps):
            flush.fill_(0.0)
            run(evs[i])
        torch.cuda.synchronize(device)
        t_wall = time.perf_counter() - t_wall
        clocks = sampler.stop()
        if world > 1:
            dist.barrier()
        return evs, clocks, t_wall

    eager_evs, _, _ = timed(step) if graphs else (None, None, None)
    evs, clocks, t_wall = timed(graph_step if graphs else step)
    t_fwd = sum(e[0].elapsed_time(e[1]) for e in evs) / args.steps
    t_bd = sum(e[1].elapsed_time(e[2]) for e in evs) / args.steps
    t_bw = sum(e[2].elapsed_time(e[3]) for e in evs) / args.steps
    passes_ms = max_over_ranks(sum(e[0].elapsed_time(e[4]) for e in evs), world, device) / args.steps
    if graphs:  # the step metric: the whole-step graph
        evs, clocks, t_wall = timed(whole_step)
    per_step = [e[0].elapsed_time(e[4]) for e in evs]
    total_ms = max_over_ranks(sum(per_step), world, device)
    ms_per_step = total_ms / args.steps
    eager_ms = None
    if eager_evs is not None:
        eager_ms = max_over_ranks(sum(e[0].elapsed_time(e[4]) for e in eager_evs), world, device) / args.steps

    # end to end through the public API: pinned host inputs copied in and
    # the results (y, dx, the gradients) copied out every step.  Steps are
    # pipelined as a data loader would run them: copies in on one stream,
    # the passes on the compute stream, copies out on a third, with device
    # buffers alternating between steps, so that step i+1's copies in and
    # step i-1's copies out (opposite PCIe directions) overlap step i's passes.
    hX = inp["X"].to(dt).pin_memory()
    hdY = inp["dY"].to(dt).pin_memory()
    hY = torch.empty_like(hX).pin_memory()
    hdX = torch.empty_like(hX).pin_memory()
    hg = torch.empty_like(gflat, device="cpu").pin_memory()
    e2e_steps = max(3, min(args.steps, 20))
    cin, cout = torch.cuda.Stream(device), torch.cuda.Stream(device)
    bufs = [dict(x=torch.empty_like(X), dy=torch.empty_like(dY), y=torch.empty_like(Y), dx=torch.empty_like(dX),
                 g=torch.empty_like(gflat)) for _ in range(2)]
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
        step(None, b["x"], b["dy"], b["y"], b["dx"])
        b["g"].copy_(gflat)
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
    d2h = 2 * X.numel() * X.element_size() + gflat.numel() * 4

    counts = algorithmic_counts(wl)
    peaks, peak_src = load_peaks()
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    sm_max = float(peaks.get("sm_max_mhz", 1965.0))
    fp32_peak_tflops = sms * FP32_LANES_PER_SM * 2 * sm_max * 1e6 / 1e12
    hbm_peak = float(peaks["hbm_gbs"])
    kernels = {"fwd": t_fwd, "bwd_data": t_bd, "bwd_weight": t_bw}
    dom = max(kernels, key=kernels.get)
    dom_ms = kernels[dom]
    # the bound of the pass: FP32 ALUs or HBM, whichever needs more time
    t_alu = 2 * counts[dom]["fma"] / (fp32_peak_tflops * 1e12)
    t_hbm = counts[dom]["bytes"] / (hbm_peak * 1e9)
    if t_hbm > t_alu:
        bound, unit, peak = "hbm", "GB/s", hbm_peak
        achieved = counts[dom]["bytes"] / (dom_ms * 1e-3) / 1e9
        peak_source = f"{peak_src} copy bandwidth"
    else:
        bound, unit, peak = "alu", "TFLOP/s", fp32_peak_tflops
        achieved = 2 * counts[dom]["fma"] / (dom_ms * 1e-3) / 1e12
        peak_source = f"{sms} SMs x {FP32_LANES_PER_SM} FP32 lanes x 2 x {sm_max:.0f} MHz"
    step_bytes = sum(c["bytes"] for c in counts.values())
    hbm_gbs = step_bytes / (ms_per_step * 1e-3) / 1e9
    traffic = load_traffic(dom, wl.name)
    line = {
        "metric": METRIC,
        "value": world * 1000.0 / ms_per_step,
        "unit": "steps/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32" if wl.io == "f32" else "bf16-io/f32",
        "data": "synthetic (seeded N(0,1) activations, N(0,1/k^2) weights, U(0.5,1.5) scales)",
        "config": {"workload": wl.name, **{k: v for k, v in wl.as_dict().items() if k != "name"},
                   "global_batch": wl.N * world, "parallelism": f"dp{world}",
                   "l2": "flushed before every timed step (256 MiB write)"},
        "roofline": {"bound": bound, "kernel": f"{dom} pass: {PASS_KERNELS[dom]}", "achieved": achieved,
                     "peak": peak, "unit": unit, "frac": achieved / peak, "traffic": traffic,
                     "traffic_source": ("profiles/traffic.json (ncu dram__bytes_read.sum + dram__bytes_write.sum "
                                        "per launch, same sources)" if traffic is not None else
                                        "none: no ncu capture of the current sources"),
                     "peak_source": peak_source},
        "hbm": {"achieved_gbs": hbm_gbs, "peak_gbs": hbm_peak, "frac": hbm_gbs / hbm_peak,
                "algorithmic_bytes_per_step": step_bytes, "peak_source": peak_src},
        "kernels_ms": kernels,
        "timing": ("the whole step one CUDA graph replay (forward, then backward-data and weight gradients on "
                   "two streams with a workspace each); kernels_ms from one graph per pass replayed in turn"
                   if graphs else "eager library calls") + ", CUDA events on the launching stream",
        "passes_ms_per_step": passes_ms,
        "eager": None if eager_ms is None else {"ms_per_step": eager_ms, "value": world * 1000.0 / eager_ms,
                                                "unit": "steps/s"},
        "e2e": {"value": world * 1000.0 / e2e_ms, "unit": "steps/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "overlap": "copies in and out on their own streams, device buffers alternating between steps"},
        "gpu_launches": launches_per_step(wt, desc) * args.steps,
        "clocks": clocks,
        "wall_s_timed_region": t_wall,
    }
    if rank == 0 and not args.no_comparators:
        extra = (Y.numel() + dX.numel()) * Y.element_size() + gflat.numel() * 4 + ws.numel()
        line["comparators"] = comparators(wl, device, inp, lambda: step(), extra)
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, args.cpu_sample_n)
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


def comparators(wl, device, inp, ours_step, ours_extra_bytes, steps=20):
    """Same-GPU comparators of one fwd+bwd step (not part of the timed
    metric): the plain PyTorch cascade (time and peak memory beyond the
    inputs), and for L = 0 a diagonalwise-refactorized conv (channels in
    blocks of 32, each block one dense conv with a block-diagonal weight, as
    in "Diagonalwise Refactorization: An Efficient Training Method for
    Depthwise Convolutions").  fp32 arithmetic on fp32 copies of the inputs."""
    import torch.nn.functional as F
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
    out["ours_extra_bytes"] = ours_extra_bytes
    out["speedup_vs_torch_cascade"] = ms / ours_ms
    out["memory_ratio_vs_torch_cascade"] = peak / max(1, ours_extra_bytes)
    if wl.L == 0:
        G = min(32, wl.C)
        groups = wl.C // G
        k = wl.k
        eye = torch.eye(G, device=device).view(1, G, G, 1, 1)

        def diag_step():
            for t in leaves:
                t.grad = None
            w = (P["W0"].view(groups, G, 1, k, k) * eye).reshape(wl.C, G, k, k)
            Y = P["s0"].view(1, -1, 1, 1) * F.conv2d(X, w, P["b0"], padding=k // 2, groups=groups)
            Y.backward(dY)

        dms, dpeak = timed(diag_step)
        out["diagonalwise_refactorization"] = {"ms_per_step": dms, "peak_extra_bytes": dpeak, "block": G}
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


def cpu_baseline(wl, sample_n):
    """The float64 oracle, as it stands, timed on the host on a bounded
    sample (the first `sample_n` batch entries of the same workload)."""
    import dataclasses
    from depthwise_convolution_wtconv_b200.inputs import as_float64
    n = max(1, min(sample_n, wl.N))
    sub = dataclasses.replace(wl, N=n)
    p = as_float64(make_inputs(sub, 0))
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        t = time.perf_counter()
        oracle_step(p)
        dt = time.perf_counter() - t
    return {"value": (n / wl.N) / dt, "unit": "steps/s", "cores": 1, "kind": "oracle",
            "sample": f"N={n} of {wl.N} (same C, H, W, k, L), one fwd+bwd in numpy float64, "
                      f"single-threaded; host has {os.cpu_count()} cores; scaled by {n}/{wl.N}",
            "seconds": dt}


def _plane_sample(wl, planes):
    """Sub-workload of `planes` (n, c) planes: the first channels of the
    first batch entries, with every other dimension unchanged."""
    import dataclasses
    planes = max(1, min(planes, wl.N * wl.C))
    if planes >= wl.C:
        return dataclasses.replace(wl, N=planes // wl.C), (planes // wl.C) * wl.C
    return dataclasses.replace(wl, N=1, C=planes), planes


def run_reference(args, wl, world, rank):
    """The oracle as the reference arm: rank 0 only, on the host cores.
    Each step runs the oracle on a bounded plane sample sized so that the
    whole run stays near two minutes; the rate is scaled to the workload."""
    if rank != 0:
        return None
    from depthwise_convolution_wtconv_b200.inputs import as_float64
    cal, cal_planes = _plane_sample(wl, min(8, wl.N * wl.C))
    pc = as_float64(make_inputs(cal, 0))
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        t = time.perf_counter()
        oracle_step(pc)
        tau = (time.perf_counter() - t) / cal_planes
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


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=BENCH_WORKLOAD, choices=list(WORKLOADS))
    ap.add_argument("--cpu-sample-n", type=int, default=32)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--eager", action="store_true", help="time eager library calls instead of CUDA graph replays")
    ap.add_argument("--no-comparators", action="store_true", help="skip the same-GPU PyTorch comparators")
    args = ap.parse_args(argv)
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
