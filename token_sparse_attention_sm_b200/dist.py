"""Multi-process plumbing: one process per GPU, launched by torchrun.

The decode path shards into independent units (sequences, or whole KV heads)
with no exchange step, so the data path needs no collective.  torch
distributed is used only for the barrier around a timed region and for the
max-over-ranks of its duration."""
from __future__ import annotations

import datetime
import os

import torch
import torch.distributed as dist


def env_rank_world():
    """(rank, world_size, local_rank) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: int = 120) -> bool:
    """Initialise the default process group when WORLD_SIZE > 1."""
    rank, world, _ = env_rank_world()
    if world <= 1 or dist.is_initialized():
        return dist.is_initialized()
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    dist.init_process_group(backend, rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=timeout_s))
    return True


def shard_range(n: int, world: int, rank: int):
    """Contiguous [lo, hi) share of n units for `rank`; shares differ by at
    most one unit and cover 0..n-1 exactly once."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    return n * rank // world, n * (rank + 1) // world


def _device():
    if dist.is_initialized() and dist.get_backend() == "nccl":
        return torch.device("cuda", torch.cuda.current_device())
    return torch.device("cpu")


def barrier():
    if dist.is_initialized():
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[torch.cuda.current_device()])
        else:
            dist.barrier()


def max_over_ranks(x: float) -> float:
    if not dist.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float) -> float:
    if not dist.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_device())
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def finalize():
    if dist.is_initialized():
        dist.destroy_process_group()
