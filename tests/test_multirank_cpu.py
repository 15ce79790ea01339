"""The benchmark's multi-rank plumbing with two gloo ranks on the CPU.

bench.py --gpus N runs one process per GPU; the forward is independent per
GPU, so N ranks are N replicas whose device-timed regions are combined as
the maximum over ranks (the whole-job value divides all ranks' work by it),
and the reference arm runs on rank 0 alone.  Here two processes rendezvous
over 127.0.0.1 with gloo and exercise exactly those helpers.
"""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist

    import bench

    w, r, _ = bench.dist_init()
    assert (w, r) == (world, rank) and bench._BACKEND == "gloo"
    bench.barrier(w)
    slowest = bench.max_over_ranks(0.25 * (rank + 1), w)

    class Args:
        steps, warmup = 2, 1

    line = bench.run_reference(Args(), w, r)
    with open(os.path.join(out_dir, "rank%d.txt" % rank), "w") as f:
        f.write("%r %r %r\n" % (slowest, line is None, None if line is None else (line["impl"], line["n_gpus"])))
    bench.barrier(w)
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_only_rank0_reports(tmp_path):
    import torch.multiprocessing as mp

    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    got = [open(tmp_path / ("rank%d.txt" % r)).read().split(" ", 2) for r in range(world)]
    # the max over ranks of 0.25 * (rank + 1)
    assert all(float(g[0]) == 0.5 for g in got)
    # rank 0 prints the reference line for the whole job; rank 1 prints nothing
    assert got[0][1] == "False" and "('reference', 2)" in got[0][2]
    assert got[1][1] == "True"
