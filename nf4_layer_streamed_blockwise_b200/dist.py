"""Data-parallel plumbing for the streamed trainer (one process per GPU).

Every rank streams its own copy of the frozen base from host RAM and trains on
its own micro-batch; the one exchange per step is the mean of the LoRA
gradients over the ranks (NCCL over NVLink on GPUs; gloo on CPU in tests).
All ranks take the same collective steps in the same order.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def init_from_env(backend: str = "nccl", timeout_s: int = 600):
    """Initialise the default process group from RANK / WORLD_SIZE / MASTER_* if
    WORLD_SIZE > 1; returns (rank, world, local_rank)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return rank, world, local


def average_gradients(flat_grad: torch.Tensor, world: int) -> None:
    """In place: flat_grad <- mean over ranks (sum all-reduce, then / world)."""
    if world <= 1:
        return
    dist.all_reduce(flat_grad, op=dist.ReduceOp.SUM)
    flat_grad.div_(world)


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest value across ranks (used for timing: the job is as slow as its slowest rank)."""
    if world <= 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
