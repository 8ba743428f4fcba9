"""Host-side helpers for running the forward on several GPUs, one process per GPU.

The Sparse-BitLinear forward has no cross-GPU exchange in its data path: linears (or
batches) are independent problems, so N ranks each take a share of them ("weak" scaling,
no collective).  The only collectives here are for control: a barrier and the max of the
ranks' device times.
"""
import os
from typing import Tuple

import torch


def env_world() -> Tuple[int, int, int]:
    """(world_size, rank, local_rank) from the torchrun environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


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


def barrier(device=None):
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.barrier()
    if device is not None and torch.cuda.is_available():
        torch.cuda.synchronize(device)
