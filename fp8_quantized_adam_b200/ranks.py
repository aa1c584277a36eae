"""Host logic of the multi-GPU run: one process per GPU, each owning an
independent shard of the parameter list.

The optimizer step has no cross-tensor dependency (each tensor's amax and
scale are its own), so shards need no collective on the data path; the only
collectives are the timing barrier and the max-over-ranks of elapsed times.
Works with the "nccl" backend on GPUs and "gloo" on CPU (tests).
"""
from __future__ import annotations

import datetime
import os
from typing import List, Sequence, Tuple

import torch
import torch.distributed as dist


def env() -> Tuple[int, int, int]:
    """(world_size, rank, local_rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, device=None, timeout_s: int = 300) -> None:
    """Join the process group when world_size > 1 (a short timeout so ranks
    waiting on a dead peer fail instead of hanging)."""
    world, _, _ = env()
    if world > 1 and not dist.is_initialized():
        kw = {"timeout": datetime.timedelta(seconds=timeout_s)}
        if device is not None and backend == "nccl":
            kw["device_id"] = device
        dist.init_process_group(backend, **kw)


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank scalar (device time) over all ranks."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier() -> None:
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def shard_seed(cfg_id: int, rank: int) -> int:
    """Seed id of a rank's shard: distinct per rank, rank 0 = the workload's."""
    return cfg_id + 100 * rank


def partition_by_numel(numels: Sequence[int], world: int) -> List[List[int]]:
    """Whole tensors to ranks, largest first onto the least-loaded rank
    (every tensor on exactly one rank, so its amax never crosses ranks)."""
    load = [0] * world
    parts: List[List[int]] = [[] for _ in range(world)]
    for i in sorted(range(len(numels)), key=lambda k: (-numels[k], k)):
        r = min(range(world), key=lambda q: (load[q], q))
        parts[r].append(i)
        load[r] += int(numels[i])
    return [sorted(p) for p in parts]


def finish() -> None:
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
