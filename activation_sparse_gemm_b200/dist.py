"""Multi-GPU plumbing for the RT-Lynx linear layer: one process per GPU.

Tokens are independent in every step of the layer (the 2-of-4 mask, s and
T are per token, and so is each row of Y), so N GPUs run the layer on
disjoint contiguous token blocks with replicated weights and no data-path
collective.  These helpers cover the host side: the token split, process-group
setup from the torchrun environment, and the max-over-ranks reduction used to
time a step.
"""
from __future__ import annotations

import datetime
import os


def token_block(M: int, world: int, rank: int, align: int = 1):
    """[start, stop) of rank's contiguous share of M tokens.  Blocks hold whole
    `align`-token units (the last one may end at M inside a unit), their unit
    counts differ by at most one, and together they cover [0, M) without
    overlap."""
    if world <= 0 or not 0 <= rank < world or M < 0 or align <= 0:
        raise ValueError("bad split")
    units = -(-M // align)
    base, extra = divmod(units, world)
    start_u = rank * base + min(rank, extra)
    stop_u = start_u + base + (1 if rank < extra else 0)
    return min(start_u * align, M), min(stop_u * align, M)


def env_ranks():
    """(world, rank, local_rank) from the torchrun environment (1, 0, 0 without one)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(backend: str, timeout_s: float = 120.0):
    """Initialises the default process group when WORLD_SIZE > 1; returns (world, rank, local_rank)."""
    import torch.distributed as dist
    world, rank, local = env_ranks()
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s))
    return world, rank, local


def max_over_ranks(value: float, device=None) -> float:
    """Largest value over all ranks (the value itself without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.barrier()


def shutdown():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
