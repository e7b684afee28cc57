"""Host-side plumbing for running the forward on several GPUs of one node.

The packed-THD forward shards by pack: every rank (one process per GPU) runs
its own pack of the same shape -- the same document lengths, tensor values
seeded by the rank -- with no collective on the data path.  The only
collectives are the barrier around the timed region and the max-over-ranks
reduction of its device time.
"""
from __future__ import annotations

import os
from dataclasses import dataclass
from typing import Optional

import torch
import torch.distributed as dist


@dataclass
class RankInfo:
    rank: int
    world: int
    local_rank: int

    @property
    def is_root(self) -> bool:
        return self.rank == 0


def rank_info() -> RankInfo:
    return RankInfo(int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
                    int(os.environ.get("LOCAL_RANK", 0)))


def init(backend: str, timeout_s: float = 120.0) -> RankInfo:
    """Initialise the process group when launched with WORLD_SIZE > 1."""
    info = rank_info()
    if info.world > 1 and not dist.is_initialized():
        import datetime
        kw = {}
        if backend == "nccl":
            kw["device_id"] = torch.device("cuda", info.local_rank)
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return info


def tensor_seed(base_seed: int, rank: int) -> int:
    """Seed of rank `rank`'s tensor values (document lengths keep base_seed)."""
    return base_seed + 7919 * rank


def barrier(device: Optional[torch.device] = None) -> None:
    if dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(value: float, device: Optional[torch.device] = None) -> float:
    """Maximum of a per-rank float over all ranks (identity when single rank)."""
    if not (dist.is_initialized() and dist.get_world_size() > 1):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / max_seconds


def shutdown() -> None:
    if dist.is_initialized():
        dist.destroy_process_group()
