"""Data-parallel plumbing for the streamed trainer (one process per GPU).

Every rank trains on its own micro-batch against the same frozen base; the
exchange per step is the mean of the LoRA gradients over the ranks (NCCL over
NVLink on GPUs; gloo on CPU in tests).  The base reaches each GPU either
whole over that GPU's host link (replicated), or as 1/world of every layer
record per rank followed by an all-gather over NVLink into every rank's slot
(sharded upload, ``gather_slot``).  All ranks take the same collective steps
in the same order: the upload order is the streaming scheduler's, which
depends only on the sequence of layer steps, the same on every rank.
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


def shard_range(nbytes: int, rank: int, world: int):
    """Bytes [lo, hi) of a record of nbytes that rank holds and copies (equal parts)."""
    if nbytes % world:
        raise ValueError(f"record of {nbytes} bytes does not split into {world} equal parts")
    per = nbytes // world
    return rank * per, (rank + 1) * per


def gather_slot(slot: torch.Tensor, nbytes: int, rank: int, world: int, stream=None) -> None:
    """Sharded upload: slot[:nbytes] holds this rank's part at shard_range(); fill
    in the other ranks' parts (in-place all-gather), ordered on `stream` when
    given (the copy stream the part was uploaded on)."""
    lo, hi = shard_range(nbytes, rank, world)
    if stream is None:
        dist.all_gather_into_tensor(slot[:nbytes], slot[lo:hi])
        return
    with torch.cuda.stream(stream):
        dist.all_gather_into_tensor(slot[:nbytes], slot[lo:hi])
