"""One process per GPU: rank discovery and the host-side aggregation of a
multi-GPU measurement.

The mixer's work shards with no exchange: every (batch, head) routes and
attends on its own, so N GPUs run N independent replicas of a workload (each
rank its own sequences) and the only collective is the reduction of the
timings (the maximum over ranks) and of the token counts (the sum).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_rank() -> tuple[int, int, int]:
    """(rank, local_rank, world_size) from the torchrun environment (defaults 0, 0, 1)."""
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def init(backend: str = "nccl", timeout_s: float = 120.0) -> tuple[int, int, int]:
    """Join the process group when WORLD_SIZE > 1 (MASTER_ADDR/PORT from the env)."""
    rank, local, world = env_rank()
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=timeout_s))
    return rank, local, world


def barrier():
    if dist.is_initialized():
        dist.barrier()


def reduce_max(values, device="cpu") -> list[float]:
    """Elementwise maximum over ranks of a list of floats."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def reduce_sum(values, device="cpu") -> list[float]:
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return t.tolist()


def replica_seed(seed: int, rank: int) -> int:
    """Each rank's replica draws its own sequences."""
    return int(seed) * 1009 + int(rank)


def throughput(tokens_per_rank: list[float], seconds_per_rank: list[float], device="cpu") -> float:
    """Whole-job tokens/s: all ranks' tokens over the slowest rank's time."""
    tot = reduce_sum([sum(tokens_per_rank)], device)[0]
    t = reduce_max([max(seconds_per_rank)], device)[0]
    return tot / t


def finalize():
    if dist.is_initialized():
        dist.destroy_process_group()
