"""Multi-rank bookkeeping of the benchmark on CPU (gloo, world size 2):
distinct per-rank seeds, the job time is the maximum over ranks and the
whole-job throughput counts every rank's units."""
import os
import socket

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from workloads.scaling import max_over_ranks, rank_seed, weak_scaling_throughput


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        seconds = [0.5, 0.8][rank]                      # rank 1 is the slow one
        t = max_over_ranks(seconds)
        seeds = [None] * world
        dist.all_gather_object(seeds, rank_seed(5, rank))
        out[rank] = (t, weak_scaling_throughput(1000.0, t, world), tuple(seeds))
    finally:
        dist.destroy_process_group()


def test_two_ranks_weak_scaling():
    world = 2
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
        res = dict(out)
    for rank in range(world):
        t, thr, seeds = res[rank]
        assert t == 0.8                                  # max over ranks, identical on every rank
        assert thr == 1000.0 * world / 0.8
        assert len(set(seeds)) == world                  # every rank draws its own inputs


def test_single_process_identity():
    assert max_over_ranks(1.25) == 1.25
    assert rank_seed(3, 0) != rank_seed(3, 1)
