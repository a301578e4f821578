"""Process-group plumbing for multi-GPU runs of the forward pass.

The path shards by independent problems: every rank owns whole sequences
(decode) or whole prompts (prefill), so there is no data-path collective.
Ranks only meet at barriers around the timed region and in one max-reduce of
the measured time.  One process per GPU; NCCL on GPUs, gloo on CPU (tests).
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def world() -> tuple[int, int, int]:
    """(world size, rank, local rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 120.0) -> None:
    """Initialise the default process group when more than one rank runs."""
    n, _, local = world()
    if n > 1 and not dist.is_initialized():
        kw = {}
        if backend == "nccl":
            kw["device_id"] = torch.device(f"cuda:{local}")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)


def barrier() -> None:
    if dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def max_over_ranks(x: float, device="cpu") -> float:
    """The maximum of a per-rank scalar (the slowest rank's time)."""
    if not (dist.is_initialized() and dist.get_world_size() > 1):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def seed_offset(rank: int) -> int:
    """Each rank draws its own batch: the workload seed plus the rank."""
    return rank


def shard(units: int, rank: int, nranks: int) -> range:
    """Contiguous share of `units` independent problems for `rank` (used when
    a fixed total is split: strong scaling)."""
    lo = units * rank // nranks
    hi = units * (rank + 1) // nranks
    return range(lo, hi)


def finalize() -> None:
    if dist.is_initialized():
        dist.destroy_process_group()
