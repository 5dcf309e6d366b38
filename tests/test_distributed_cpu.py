"""Multi-rank logic of the bench on CPU: two gloo ranks, max-over-ranks timing and the
weak-scaling aggregate (each rank runs its own batch; no data-path collective)."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        seconds = 1.0 + rank  # rank 1 is the slow one
        mx = bench.aggregate_max(seconds, world, torch.device("cpu"))
        val = bench.weak_scaling_value(1000, 10, world, mx)
        # each rank draws its own batch (seed = rank): the inputs differ across ranks
        x = workloads.generate(workloads.custom(1, 8, H=2, P=4, N=4, chunk=64), seed=rank).x
        gathered = [torch.zeros_like(x) for _ in range(world)]
        dist.all_gather(gathered, x)
        out[rank] = (mx, val, bool(torch.equal(gathered[0], gathered[1])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_weak_scaling():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(_rank, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        mx, val, same = out[r]
        assert mx == 2.0  # max over ranks
        assert abs(val - world * 1000 * 10 / 2.0) < 1e-9
        assert not same  # independent batches
