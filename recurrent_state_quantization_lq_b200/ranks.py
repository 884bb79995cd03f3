"""Process-per-GPU plumbing for the sharded decode.

Every (sequence, head) unit of the windowed-INT8 decode is independent of every
other: no step of the recurrence or of the per-window codec reads another
unit's state.  So N processes shard the work by sequences, each with its own
workspace and its own seeded inputs, and nothing crosses between ranks on the
data path.  What remains is host plumbing: which rank am I, which seed does my
shard draw from, one barrier around the timed region and the max over ranks of
the timer (weak scaling: the job's time is its slowest rank's).
"""
from __future__ import annotations

import datetime
import os

import torch


def env_ranks() -> tuple[int, int, int]:
    """(rank, world size, local rank) as torchrun exports them; (0, 1, 0) alone."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, device: torch.device | None = None, timeout_s: float = 300.0) -> None:
    """Join the process group (rendezvous from MASTER_ADDR / MASTER_PORT).

    A short timeout makes ranks that wait on a rank that died end with an
    error instead of waiting for good."""
    import torch.distributed as dist
    rank, world, _ = env_ranks()
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None and device.type == "cuda":
        kw["device_id"] = device
    dist.init_process_group(backend, rank=rank, world_size=world, **kw)


def shard_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s shard: distinct per rank, fixed per (workload, rank)."""
    if rank < 0 or rank >= 1000:
        raise ValueError("rank must be in [0, 1000)")
    return base_seed * 1000 + rank


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device: torch.device | str = "cpu") -> float:
    """The maximum of `x` over all ranks (every rank gets it).  `device` is the
    one the process group's backend reduces on: the rank's GPU under NCCL, the
    CPU under gloo."""
    if world == 1:
        return float(x)
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Weak-scaling throughput: every rank's units over the slowest rank's time."""
    if max_seconds <= 0:
        raise ValueError("time must be positive")
    return world * units_per_rank / max_seconds
