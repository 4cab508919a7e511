"""Multi-process helpers for running the library as independent replicas.

Every (batch, head) of the attention is independent and the path has no
exchange step, so N GPUs run N replicas of the same call; the only collective
is the timing reduction: the max over ranks of the device-timed milliseconds.
"""
from __future__ import annotations

import datetime
import os


def env_ranks() -> tuple[int, int, int]:
    """(rank, world_size, local_rank) from the torchrun environment (defaults: one process)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: int = 300):
    """Initialise the default process group when WORLD_SIZE > 1; returns the module or None."""
    rank, world, _ = env_ranks()
    if world <= 1:
        return None
    import torch.distributed as dist
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return dist


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of a per-rank float over all ranks (the value itself with one process)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_ms_per_call(max_ms_per_step: float, world: int) -> float:
    """Whole-job time per call when `world` replicas each ran one call per step."""
    return max_ms_per_step / max(1, world)
