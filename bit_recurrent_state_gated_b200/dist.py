"""Multi-GPU plumbing for the decode step: one process per GPU, requests partitioned across
ranks, no collective on the data path (every request's state evolves independently).

torch.distributed is used only for the launch-time rendezvous, the barrier around the timed
region and the max-over-ranks reduction of elapsed times.
"""
from __future__ import annotations

import os
from dataclasses import dataclass


@dataclass(frozen=True)
class RankInfo:
    rank: int
    local_rank: int
    world: int


def rank_info() -> RankInfo:
    return RankInfo(int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
                    int(os.environ.get("WORLD_SIZE", 1)))


def partition(n: int, world: int, rank: int) -> tuple[int, int]:
    """[start, stop) of rank's share of n independent requests (contiguous, sizes differ by
    at most one)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def init(backend: str, timeout_s: float = 120.0):
    """Initialise the default process group when launched by torchrun (WORLD_SIZE > 1)."""
    import datetime

    import torch.distributed as dist
    info = rank_info()
    if info.world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend,
                                timeout=datetime.timedelta(seconds=timeout_s))
    return info


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank float over all ranks (identity on one process)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def finalize():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
