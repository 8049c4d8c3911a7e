"""Host-side multi-GPU plumbing: one process per GPU (torchrun), no data-path
collective.

The attention heads (b, h) and the regrid's targets are independent
problems, so N ranks run N independent replicas of the workload, each on
its own seeded batch (weak scaling).  The only collectives are a barrier
around the timed region and a MAX reduction of each rank's elapsed time.
"""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass

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
    """RANK / WORLD_SIZE / LOCAL_RANK from the environment (torchrun), else 0/1/0."""
    return RankInfo(int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
                    int(os.environ.get("LOCAL_RANK", 0)))


def init(backend: str, info: RankInfo, timeout_s: float = 120.0) -> None:
    """Join the process group when there is more than one rank (short timeout
    so a rank that never arrives ends the others with an error)."""
    if info.world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        kw = {}
        if backend == "nccl":
            kw["device_id"] = torch.device("cuda", info.local_rank)
        dist.init_process_group(backend, rank=info.rank, world_size=info.world,
                                timeout=datetime.timedelta(seconds=timeout_s), **kw)


def shutdown() -> None:
    if dist.is_initialized():
        dist.destroy_process_group()


def replica_seed(base_seed: int, rank: int) -> int:
    """Seed of rank r's batch: rank 0 keeps the workload's own seed."""
    return base_seed + 1000 * rank


def barrier(device: torch.device | None = None) -> None:
    if dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def max_over_ranks(value: float, device: torch.device | None = None) -> float:
    """The maximum of a per-rank scalar (elapsed device time) over all ranks."""
    if not dist.is_initialized():
        return float(value)
    dev = device if device is not None else torch.device("cpu")
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device: torch.device | None = None) -> float:
    if not dist.is_initialized():
        return float(value)
    dev = device if device is not None else torch.device("cpu")
    t = torch.tensor([float(value)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())
