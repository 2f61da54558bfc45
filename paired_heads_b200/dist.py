"""Data-parallel plumbing for running the forward on N GPUs, one process per GPU.

The forward has no exchange step: every rank holds whole documents of its own and runs the same
two library calls on them. Only timing crosses ranks (barriers and a max-reduce of the elapsed
device time). Rank and world size come from the torchrun environment.
"""
from __future__ import annotations

import datetime
import os


def env():
    """(rank, world_size, local_rank) from the launcher's environment (1 process: 0, 1, 0)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, device=None, timeout_s: float = 120.0):
    """Join the process group (no-op for a single process). Returns the torch.distributed
    module or None."""
    _, world, _ = env()
    if world <= 1:
        return None
    import torch.distributed as dist

    kw = dict(timeout=datetime.timedelta(seconds=timeout_s))
    if device is not None and backend == "nccl":
        kw["device_id"] = device
    dist.init_process_group(backend, **kw)
    return dist


def max_over_ranks(dist, value: float, device=None) -> float:
    """The largest value over all ranks (identity for a single process)."""
    if dist is None:
        return value
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def gather_ints(dist, value: int) -> list:
    """Every rank's integer, in rank order (a one-element list for a single process)."""
    if dist is None:
        return [int(value)]
    import torch

    t = torch.tensor([int(value)], dtype=torch.int64)
    out = [torch.zeros_like(t) for _ in range(dist.get_world_size())]
    dist.all_gather(out, t)
    return [int(x.item()) for x in out]


def barrier(dist):
    if dist is not None:
        dist.barrier()


def finalize(dist):
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
