"""Replica plumbing for running the decode step on several GPUs of one node.

The decode step shards naturally by sequence: every GPU holds a full weight
replica and its own disjoint set of KV-cache slots, and batch invariance makes
a sequence's result independent of which GPU or batch it ran in.  There is no
collective on the data path.  The only cross-rank traffic is a barrier around
timed regions and the max of the ranks' timings (the job is as slow as its
slowest replica).  Rendezvous: torch.distributed from the usual RANK /
WORLD_SIZE / LOCAL_RANK / MASTER_ADDR / MASTER_PORT environment.
"""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_ranks():
    """(rank, world, local_rank) from the launcher's environment (1 process if unset)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, device=None, timeout_s: int = 300) -> bool:
    """Join the process group when WORLD_SIZE > 1.  Returns True if joined."""
    rank, world, _ = env_ranks()
    if world <= 1:
        return False
    kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if backend == "nccl" and device is not None:
        kw["device_id"] = device
    dist.init_process_group(backend, rank=rank, world_size=world, **kw)
    return True


def barrier() -> None:
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity in a single process)."""
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job units per second when every rank processes units_per_rank in max_ms."""
    return units_per_rank * world / (max_ms * 1e-3)


def replica_seed(base: int, rank: int) -> int:
    """Seed of a rank's own synthetic sequences (disjoint per rank)."""
    return int(base) + 1000003 * int(rank)


def finalize() -> None:
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
