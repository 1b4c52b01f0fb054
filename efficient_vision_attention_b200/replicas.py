"""Multi-GPU plumbing: one process per GPU running independent replicas.

The (batch, head) slices of the Agent Attention forward pass share nothing, so
N GPUs need no exchange on the data path: each rank processes its own slices
(its own batch, or its share of a global batch) and the only collectives are a
barrier and the max over ranks of the device-timed step.  Rendezvous comes
from the usual torch.distributed environment (RANK, WORLD_SIZE, LOCAL_RANK,
MASTER_ADDR, MASTER_PORT).
"""
from __future__ import annotations

import datetime
import os

import torch


def dist_env() -> tuple[int, int, int]:
    """(world_size, rank, local_rank) from the environment (1, 0, 0 if unset)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, device: torch.device | None = None, timeout_s: float = 120.0):
    """Initialise the process group when more than one rank runs; returns the
    torch.distributed module (or None for a single process)."""
    world, _, _ = dist_env()
    if world <= 1:
        return None
    import torch.distributed as dist
    kwargs = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if device is not None and backend == "nccl":
        kwargs["device_id"] = device
    dist.init_process_group(backend, **kwargs)
    return dist


def shard(n_items: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous share [begin, end) of n_items for `rank`; sizes differ by at most one."""
    base, extra = divmod(n_items, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of a rank's replica inputs (rank 0 keeps the workload's own seed)."""
    return base_seed + 1000 * rank


def max_over_ranks(value: float, dist, device: torch.device | None = None) -> float:
    """The maximum of `value` over all ranks (the value itself for one process)."""
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist) -> None:
    if dist is not None:
        dist.barrier()


def finalize(dist) -> None:
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
