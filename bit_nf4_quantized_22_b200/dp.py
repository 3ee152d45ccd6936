"""Data-parallel plumbing for the layer (one process per GPU).

The frozen NF4 weight is replicated; each rank takes its own contiguous run of
token rows.  The only exchange of a data-parallel QLoRA step is the sum of the
adapter gradients over ranks (the frozen weight has none): one all-reduce
each for dA and dB on the default process group (NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations


def shard_rows(M: int, rank: int, world: int) -> slice:
    """Contiguous token rows of `rank` when M rows are split over `world` ranks."""
    base, extra = divmod(M, world)
    start = rank * base + min(rank, extra)
    return slice(start, start + base + (1 if rank < extra else 0))


def allreduce_adapter_grads(dA, dB, group=None) -> None:
    """Sum dA and dB over the ranks of `group`, in place."""
    import torch.distributed as dist
    dist.all_reduce(dA, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(dB, op=dist.ReduceOp.SUM, group=group)
