"""Host-side helpers for running the forward on several GPUs, one process per GPU.

The Sparse-BitLinear forward has no cross-GPU exchange in its data path: linears (or
batches) are independent problems, so N ranks each take a share of them, or each run a
replica of the same workload on its own inputs ("weak" scaling, no collective).  The
collectives here are for control only: a barrier and the max of the ranks' device times.
"""
import datetime
import os
from typing import Tuple

import torch


def env_world() -> Tuple[int, int, int]:
    """(world_size, rank, local_rank) from the torchrun environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str = "nccl", timeout_s: float = 120.0) -> Tuple[int, int, int]:
    """Joins the process group when WORLD_SIZE > 1 (one process per GPU; the rendezvous comes
    from MASTER_ADDR / MASTER_PORT).  Sets the local CUDA device for the nccl backend.
    Returns (world_size, rank, local_rank)."""
    world, rank, local = env_world()
    if world > 1 and not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        if backend == "nccl":
            torch.cuda.set_device(local)
        torch.distributed.init_process_group(backend,
                                             timeout=datetime.timedelta(seconds=timeout_s))
    return world, rank, local


def shutdown():
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.destroy_process_group()


def shard_range(n_units: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous [begin, end) share of n_units for `rank`; sizes differ by at most one."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    base, extra = divmod(n_units, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar (device times are reported as the slowest rank)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def barrier(device=None):
    """All ranks meet (host side), then this rank's device work is finished."""
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()
    if device is not None and torch.cuda.is_available():
        torch.cuda.synchronize(device)
