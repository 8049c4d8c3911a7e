"""Host-side multi-GPU plumbing: one process per GPU (torchrun), no data-path
collective.

The attention heads (b, h) and the regrid's targets are independent
problems, so one problem is split across ranks without any exchange: at
world size W the problem is a batch of B*W sequences (and W blocks of
regrid targets against one shared source set), and rank r computes
sequences [r*B, (r+1)*B) -- the heads [r*B*H, (r+1)*B*H) of the flattened
batch -- and target block r.  The per-rank work is fixed as W grows (weak
scaling).  Every sequence is drawn from a seed of its own, so a rank draws
its block alone and the global batch does not depend on W.  The only
collectives are a barrier around the timed region and a MAX reduction of
each rank's elapsed time.
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


def shard(units: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous block (first, count) of `units` independent units for
    `rank`; the blocks of ranks 0..world-1 partition [0, units) in order."""
    base, extra = divmod(units, world)
    first = rank * base + min(rank, extra)
    return first, base + (1 if rank < extra else 0)


def sequence_block(per_rank: int, rank: int) -> int:
    """First sequence of rank r when every rank takes `per_rank` sequences."""
    return per_rank * rank


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
