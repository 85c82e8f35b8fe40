"""Host logic of the data-parallel bench path on two gloo ranks (CPU).

The layer is a sum over the batch, so data parallelism needs exactly one
exchange: the parameter gradients of every rank summed with one all-reduce.
These tests run bench.py's own rendezvous, per-rank inputs, gradient
all-reduce and max-over-ranks timing on two CPU processes, with the float64
oracle standing in for the GPU kernels, and check that the summed
gradients equal the oracle's gradients of the concatenated global batch.
"""
import dataclasses
import os
import socket
import sys

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(WORLD), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist

    import bench
    import oracle
    from depthwise_convolution_wtconv_b200.configs import Workload
    from depthwise_convolution_wtconv_b200.inputs import as_float64

    world, r, _ = bench.setup_dist()
    assert (world, r) == (WORLD, rank)
    wl = Workload("dp", 2, 3, 16, 16, 3, 2, "f32")
    inp = bench.rank_inputs(wl, rank)
    p = as_float64(inp)
    g = oracle.backward(p["X"], p["dY"], p["W0"], p["b0"], p["s0"], p["Wl"], p["sl"])
    flat, views = bench.grads_flat_views(wl, "cpu")
    for key, ok in (("dw0", "dW0"), ("db0", "db0"), ("ds0", "ds0"), ("dwl", "dWl"), ("dsl", "dsl")):
        views[key].copy_(torch.from_numpy(np.ascontiguousarray(g[ok])).float())
    bench.allreduce_grads(flat, world)
    slowest = bench.max_over_ranks(1.5 + rank, world, "cpu")
    ref_line = bench.run_reference(type("A", (), {"steps": 1, "warmup": 0})(), wl, world, rank)
    torch.save({"flat": flat, "slowest": slowest, "ref_line_is_none": ref_line is None,
                "X": inp["X"], "dY": inp["dY"], "W0": inp["W0"]}, os.path.join(out_dir, f"rank{rank}.pt"))
    dist.barrier()
    dist.destroy_process_group()


def test_data_parallel_gradients_equal_global_batch_gradients(tmp_path):
    import oracle
    import bench
    from depthwise_convolution_wtconv_b200.configs import Workload
    from depthwise_convolution_wtconv_b200.inputs import as_float64, make_inputs

    mp.start_processes(_rank_main, args=(_free_port(), str(tmp_path)), nprocs=WORLD, join=True,
                       start_method="spawn")
    res = [torch.load(tmp_path / f"rank{r}.pt") for r in range(WORLD)]
    # the ranks agree on the summed gradients and on the slowest time
    assert torch.equal(res[0]["flat"], res[1]["flat"])
    assert res[0]["slowest"] == res[1]["slowest"] == 1.5 + (WORLD - 1)
    # parameters are shared, activations are each rank's own
    assert torch.equal(res[0]["W0"], res[1]["W0"])
    assert not torch.equal(res[0]["X"], res[1]["X"])
    # the reference arm runs on rank 0 only
    assert not res[0]["ref_line_is_none"] and res[1]["ref_line_is_none"]

    wl = Workload("dp", 2, 3, 16, 16, 3, 2, "f32")
    glob = as_float64(make_inputs(wl, 0))
    glob["X"] = np.concatenate([res[r]["X"].double().numpy() for r in range(WORLD)])
    glob["dY"] = np.concatenate([res[r]["dY"].double().numpy() for r in range(WORLD)])
    g = oracle.backward(glob["X"], glob["dY"], glob["W0"], glob["b0"], glob["s0"], glob["Wl"], glob["sl"])
    flat, views = bench.grads_flat_views(dataclasses.replace(wl, N=WORLD * wl.N), "cpu")
    flat.copy_(res[0]["flat"])
    for key, ok in (("dw0", "dW0"), ("db0", "db0"), ("ds0", "ds0"), ("dwl", "dWl"), ("dsl", "dsl")):
        ref = g[ok]
        err = np.max(np.abs(views[key].double().numpy() - ref)) / max(np.max(np.abs(ref)), 1e-30)
        assert err < 1e-6, (key, err)


def test_rank_inputs_rank0_is_the_single_gpu_workload():
    import bench
    from depthwise_convolution_wtconv_b200.configs import Workload
    from depthwise_convolution_wtconv_b200.inputs import make_inputs

    wl = Workload("dp", 2, 3, 16, 16, 3, 2, "f32")
    a, b = bench.rank_inputs(wl, 0), make_inputs(wl, 0)
    assert all(torch.equal(a[k], b[k]) for k in b)
