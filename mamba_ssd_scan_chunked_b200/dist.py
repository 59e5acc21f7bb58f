"""Process-group plumbing for running the SSD core on several GPUs of a node.

Every (batch, head) recurrence is independent, so the batch is sharded across
ranks (one process per GPU) with no collective on the data path; the only
collectives are the barrier around a timed region and the max-over-ranks
reduction of its duration.
"""
from __future__ import annotations

import datetime


def init(world: int, rank: int, local_rank: int, backend: str = "nccl", timeout_s: float = 120.0):
    """Join the default process group (None when world == 1)."""
    if world <= 1:
        return None
    import torch
    import torch.distributed as td
    kw = {}
    if backend == "nccl":
        kw["device_id"] = torch.device("cuda", local_rank)
    td.init_process_group(backend, rank=rank, world_size=world,
                          timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return td.group.WORLD


def shard(global_batch: int, rank: int, world: int) -> list:
    """Contiguous block of batch indices owned by `rank` (sizes differ by at most one)."""
    if world < 1 or not 0 <= rank < world or global_batch < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(global_batch, world)
    start = rank * base + min(rank, extra)
    return list(range(start, start + base + (1 if rank < extra else 0)))


def _device(pg):
    import torch
    import torch.distributed as td
    return torch.device("cuda", torch.cuda.current_device()) if td.get_backend(pg) == "nccl" else torch.device("cpu")


def barrier(pg) -> None:
    if pg is None:
        return
    import torch
    import torch.distributed as td
    t = torch.zeros(1, device=_device(pg))
    td.all_reduce(t, group=pg)   # a collective every rank takes in the same order


def max_over_ranks(pg, value: float) -> float:
    if pg is None:
        return float(value)
    import torch
    import torch.distributed as td
    t = torch.tensor([float(value)], dtype=torch.float64, device=_device(pg))
    td.all_reduce(t, op=td.ReduceOp.MAX, group=pg)
    return float(t.item())


def finish(pg) -> None:
    if pg is None:
        return
    import torch.distributed as td
    td.destroy_process_group()
