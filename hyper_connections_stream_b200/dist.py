"""Multi-process plumbing for running the HC step on several GPUs of a node.

The step shards with no collective: every token is independent (the mixes act
within a token's n streams and RMSNorm within one token), so N ranks each run
their own tokens. torch.distributed carries only the barrier and the
max-over-ranks timing. Works with NCCL (tensors on the rank's GPU) and gloo
(CPU tensors, used by the CPU tests).
"""
from __future__ import annotations

import os

import torch


def env():
    """(world_size, rank, local_rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def seed_offset(rank: int) -> int:
    """Seed shift that gives every rank its own synthetic batch."""
    return 7919 * rank


def token_shard(T: int, rank: int, world: int):
    """(start, count) of rank's contiguous share of T tokens (strong scaling):
    the first T % world ranks take one extra token."""
    base, extra = divmod(T, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The maximum of `value` over all ranks (the slowest rank's time)."""
    if world == 1:
        return float(value)
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64,
                     device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
