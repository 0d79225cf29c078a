"""Data-parallel replicas: one process per GPU, independent batches, no collective on the
data path. The only communication is host plumbing: a barrier around timed regions and a
max over ranks of a timing (torch.distributed; NCCL on GPUs, gloo on CPU)."""
from __future__ import annotations

import datetime
import os
from dataclasses import dataclass
from typing import Optional


@dataclass
class Rank:
    rank: int
    world: int
    local: int


def from_env() -> Rank:
    return Rank(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                int(os.environ.get("LOCAL_RANK", "0")))


def init(r: Rank, backend: str, device=None, timeout_s: float = 120.0) -> None:
    """Joins the process group when world > 1 (short timeout, so a rank that waits for a
    missing peer ends with an error rather than waiting for good)."""
    if r.world <= 1:
        return
    import torch.distributed as dist
    kw = {}
    if device is not None and backend == "nccl":
        kw["device_id"] = device
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)


def shutdown(r: Rank) -> None:
    if r.world <= 1:
        return
    import torch.distributed as dist
    if dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()


def barrier(r: Rank) -> None:
    if r.world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(r: Rank, value: float, device=None) -> float:
    """Maximum of a per-rank scalar (a duration) over all ranks."""
    if r.world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard(n_units: int, r: Rank) -> range:
    """Contiguous share of n_units independent units (batch rows) for this rank; shares
    differ in size by at most one and cover every unit exactly once."""
    base, extra = divmod(n_units, r.world)
    start = r.rank * base + min(r.rank, extra)
    return range(start, start + base + (1 if r.rank < extra else 0))


def seed_for(r: Rank, base: Optional[int] = 0) -> int:
    """Each replica draws its own independent batch."""
    return (base or 0) + r.rank
