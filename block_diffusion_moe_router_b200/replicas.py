"""Replica (data-parallel) execution of the layer over several GPUs.

The layer works on one canvas at a time and every token is independent, so
N GPUs run N independent replicas: one process per GPU, each with its own
plan, weights and canvases, and no collective on the data path.  The only
collectives are the host-side barrier around a timed region and the max of
the per-rank device times, so the job's time is that of its slowest rank.

Rank, world size and local rank come from the torchrun environment
(RANK / WORLD_SIZE / LOCAL_RANK / MASTER_ADDR / MASTER_PORT).
"""
from __future__ import annotations

import datetime
import os
from typing import Optional, Tuple

import torch
import torch.distributed as dist


def dist_env() -> Tuple[int, int, int]:
    """(rank, world_size, local_rank) from the launcher's environment."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not (0 <= rank < world) or local < 0:
        raise ValueError(f"bad rank environment: RANK={rank} WORLD_SIZE={world} "
                         f"LOCAL_RANK={local}")
    return rank, world, local


def init(backend: str = "nccl", device: Optional[torch.device] = None,
         timeout_s: float = 120.0) -> Tuple[int, int]:
    """Join the process group when there is more than one rank.  A short
    timeout makes ranks that wait on a missing peer fail with an error."""
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
        if device is not None and backend == "nccl":
            kw["device_id"] = device
        dist.init_process_group(backend, **kw)
    return rank, world


def world_size() -> int:
    return dist.get_world_size() if dist.is_initialized() else 1


def barrier() -> None:
    if world_size() > 1:
        dist.barrier()


def max_over_ranks(value: float, device="cpu") -> float:
    """The largest of the ranks' values (every rank gets it)."""
    if world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank_step: int, world: int, steps: int, ms: float) -> float:
    """Whole-job throughput: the units all ranks processed over the job's
    (max-over-ranks) time, per second."""
    if ms <= 0:
        raise ValueError("non-positive time")
    return world * units_per_rank_step * steps / (ms * 1e-3)


def replica_seed(rank: int, i: int) -> int:
    """Seed of input set i on this rank: replicas work on distinct canvases."""
    return 777000 + 1000 * rank + i


def shutdown() -> None:
    if dist.is_initialized():
        dist.destroy_process_group()
