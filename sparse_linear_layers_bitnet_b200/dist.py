"""Multi-process plumbing for the benchmark (one process per GPU).

The hot path shards without any data exchange: every rank packs and
multiplies its own layers (weak scaling).  The only cross-rank operations are
host-side bookkeeping: a barrier around the timed region and the maximum of
the per-rank device times.  torch.distributed provides both (NCCL on GPUs,
gloo on CPU for tests).
"""
from __future__ import annotations

import os
from dataclasses import dataclass


@dataclass
class DistInfo:
    rank: int
    world: int
    local_rank: int


def env_info() -> DistInfo:
    return DistInfo(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str | None = None, timeout_s: float = 120.0) -> DistInfo:
    """Join the process group when launched by torchrun (WORLD_SIZE > 1)."""
    import datetime

    import torch
    import torch.distributed as dist
    info = env_info()
    if info.world > 1 and not dist.is_initialized():
        if backend is None:
            backend = "nccl" if torch.cuda.is_available() else "gloo"
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(info.local_rank)
            kw["device_id"] = torch.device("cuda", info.local_rank)
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return info


def barrier() -> None:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(value: float, device=None) -> float:
    """Maximum of a per-rank scalar (e.g. a device-timed duration)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def shard(n_units: int, rank: int, world: int) -> range:
    """Contiguous share of n_units for this rank (sizes differ by at most one)."""
    base, extra = divmod(n_units, world)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def finalize() -> None:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()
