"""Multi-process plumbing for running the coupling on several GPUs of one node.

The coupling of one shape pair runs on one GPU; a batch of independent shape
pairs is split across ranks (weak scaling, no collective on the data path).
torch.distributed is used only for the barrier around the timed region and to
take the maximum of the ranks' device times.
"""
from __future__ import annotations

import datetime
import os


def world():
    """(world_size, rank, local_rank) from the torchrun environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: int = 120):
    """Initialise the process group when running under torchrun."""
    ws, rank, local = world()
    if ws > 1:
        import torch
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return ws, rank, local


def shard(num_items: int, ws: int, rank: int):
    """Indices of the independent problems (shape pairs) this rank owns: a
    contiguous block, sizes differing by at most one."""
    base, extra = divmod(num_items, ws)
    start = rank * base + min(rank, extra)
    return list(range(start, start + base + (1 if rank < extra else 0)))


def max_over_ranks(x: float, ws: int, device=None) -> float:
    if ws == 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(ws: int):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def finalize(ws: int):
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
