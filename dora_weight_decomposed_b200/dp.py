"""Data-parallel DoRA layer: tokens are sharded across ranks, the frozen W0 and
the trainable A, B, m are replicated, and the one exchange per step is a sum of
the per-rank gradients dm, dA, dB (dx stays local to its tokens). The norm
depends on the weights only, so every rank computes it for itself.

The collectives are torch.distributed (NCCL over NVLink on GPUs, gloo on CPU).
"""
from __future__ import annotations


def token_shard(T_total: int, rank: int, world: int) -> tuple[int, int]:
    """[start, stop) of this rank's tokens; shards differ in size by at most one."""
    if world < 1 or not 0 <= rank < world or T_total < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(T_total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_gradients(dm, dA, dB, group=None) -> None:
    """Sum dm, dA and dB over the data-parallel group, in place."""
    import torch.distributed as dist
    for t in (dm, dA, dB):
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
