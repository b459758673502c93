"""The N > 1 host path of bench.py, as two gloo ranks on the CPU.

bench.py under torchrun runs one process per GPU, each quantising its own
layer's MLP weights (weak scaling, no data-path collective); the process group
only carries the barrier and the max over ranks of the timed region, and rank
0 alone prints.  Here the same functions run with the gloo backend and world
size 2: rank setup from the environment, different inputs per rank, the max
over ranks, the whole-job throughput, and the reference arm doing no work on
rank 1.
"""
import io
import os
import socket
import sys
import contextlib

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    import bench
    w, r, local = bench.dist_setup(backend="gloo")
    assert (w, r, local) == (world, rank, rank)
    # each rank's own layer: different weights, same shapes
    ins = bench.make_inputs(r)
    sig = torch.tensor([float(ins["gate"][:4, :4].float().sum())], dtype=torch.float64)
    sigs = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
    torch.distributed.all_gather(sigs, sig)
    bench.barrier(w)
    # max over ranks of a per-rank time
    t = bench.max_over_ranks(10.0 + rank, w)
    # the reference arm: only rank 0 works and prints
    buf = io.StringIO()
    if rank != 0:
        class A:
            gpus, steps, warmup, ref_budget, ref_step = world, 1, 0, 0.1, 0.1
        with contextlib.redirect_stdout(buf):
            bench.run_reference(A, w, r)
    cfg = bench.config_dict(w)
    torch.distributed.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.txt"), "w") as f:
        f.write(repr(dict(sigs=[float(x) for x in sigs], t=t, ref_out=buf.getvalue(),
                          parallelism=cfg["parallelism"], shapes=[tuple(v.shape) for v in ins.values()])))


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    res = [eval(open(tmp_path / f"rank{r}.txt").read()) for r in range(world)]
    for r in res:
        assert r["t"] == 11.0                      # max over ranks
        assert r["parallelism"] == "replicas2"
        assert r["shapes"] == [(11008, 4096), (11008, 4096), (4096, 11008)]
    assert res[0]["sigs"] == res[1]["sigs"]        # all-gather agrees
    assert res[0]["sigs"][0] != res[0]["sigs"][1]  # per-rank layer seeds differ
    assert res[1]["ref_out"] == ""                 # rank 1 runs no reference work


def test_stream_layers_split_across_ranks():
    sys.path.insert(0, ROOT)
    import bench
    for layers, world in ((80, 1), (80, 8), (80, 3), (5, 8)):
        parts = [bench.rank_layers(layers, world, r) for r in range(world)]
        flat = sorted(x for p in parts for x in p)
        assert flat == list(range(layers))  # every layer once
        assert max(map(len, parts)) - min(map(len, parts)) <= 1  # balanced


def test_throughput_is_whole_job():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.throughput(1, 1_000_000_000, 10, 100.0)
    assert one == pytest.approx(100.0)
    assert bench.throughput(4, 1_000_000_000, 10, 100.0) == pytest.approx(4 * one)  # weak scaling: N x the work
