"""Process-group plumbing for running independent replicas of the workload on N GPUs.

Heads (b, h) are independent, so a multi-GPU run is N replicas on disjoint heads with no
collective on the data path ("weak" scaling).  The only collectives are the barrier around
the timed region and the max-reduction of its duration.  torchrun provides RANK, LOCAL_RANK,
WORLD_SIZE and MASTER_ADDR/PORT.
"""
from __future__ import annotations

import datetime
import os

import torch


def world() -> tuple[int, int, int]:
    """(world_size, rank, local_rank) from the torchrun environment (1, 0, 0 without it)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: float = 120.0) -> None:
    import torch.distributed as dist

    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))


def barrier() -> None:
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float, device=None) -> float:
    """The maximum of x over all ranks (x itself without a process group)."""
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_seed(base: int, rank: int, replica: int = 0) -> int:
    """Seed of one rank's input set: every rank (and each rotating set) draws its own heads."""
    return base + 7919 * (2 * rank + replica)


def aggregate_rate(units_per_step_per_rank: int, steps: int, world_size: int, max_ms: float) -> float:
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return units_per_step_per_rank * steps * world_size / (max_ms / 1e3)
