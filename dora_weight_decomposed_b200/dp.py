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
    """Sum dm, dA and dB over the data-parallel group, in place, in one float32 all-reduce.

    bf16 gradients are widened to float32 before the sum and rounded once after
    it: a bf16 all-reduce would round at every hop of the ring, so its error
    would grow with the number of ranks. dm is float32 already. One flat buffer
    carries all three, so the exchange is a single collective (float64 when
    any of them is float64).
    """
    import torch
    import torch.distributed as dist
    ts = (dm, dA, dB)
    acc = torch.float64 if any(t.dtype == torch.float64 for t in ts) else torch.float32
    flat = torch.cat([t.reshape(-1).to(acc) for t in ts])
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    off = 0
    for t in ts:
        n = t.numel()
        t.copy_(flat[off:off + n].view(t.shape))
        off += n
