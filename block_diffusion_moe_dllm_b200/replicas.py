"""Replica runs over several GPUs: one process per GPU, every rank decodes its own requests (independent blocks
with their own seeds); the only cross-rank step is timing, taken as the maximum over ranks."""
import os

import torch
import torch.distributed as dist


def env():
    """(world_size, rank, local_rank) from the launcher's environment (1, 0, 0 when run directly)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def replica_seed(base_seed: int, rank: int) -> int:
    """Seed of a rank's synthetic requests: distinct per rank, reproducible."""
    return base_seed + 1000 * rank


def max_over_ranks(seconds: float, device) -> float:
    """The slowest rank's time (all ranks take part; returns the local value without a process group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return seconds
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_throughput(units_per_rank: float, seconds_max: float, world: int) -> float:
    """Whole-job throughput: units processed by all ranks over the slowest rank's time."""
    return units_per_rank * world / seconds_max
