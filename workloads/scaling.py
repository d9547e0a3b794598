"""Multi-rank bookkeeping for the benchmark (no method arithmetic).

The hot path partitions by sequence: every rank runs the same per-GPU
workload on its own seeded sequences, with no data-path collective (weak
scaling).  Only the timings meet: the job time is the maximum over ranks.
"""
import torch
import torch.distributed as dist


def rank_seed(seed: int, rank: int) -> int:
    """Seed of a rank's inputs: distinct per rank, reproducible."""
    return int(seed) * 1000003 + int(rank)


def max_over_ranks(x: float) -> float:
    """Maximum of a per-rank scalar (identity without a process group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    dev = torch.device("cuda", torch.cuda.current_device()) if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_throughput(units_per_rank: float, seconds_max: float, world: int) -> float:
    """Whole-job throughput: units processed by all ranks / slowest rank's time."""
    return units_per_rank * world / seconds_max
