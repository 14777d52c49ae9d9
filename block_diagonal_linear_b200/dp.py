"""Data-parallel plumbing for the Monarch training step (one process per GPU).

Rows of X are independent, so a batch shards by rows with the factors R and L
replicated.  The forward needs no exchange; the backward's weight gradients are
sums over rows, so each rank's dR and dL are summed over ranks with one
all-reduce (NCCL on GPUs, gloo on CPU).  dX needs no exchange.
"""
from __future__ import annotations


def shard_rows(rows: int, rank: int, world: int) -> tuple[int, int]:
    """[start, stop) of this rank's rows; shards differ in size by at most one row."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank %d of world %d" % (rank, world))
    return rows * rank // world, rows * (rank + 1) // world


def allreduce_weight_grads(dR, dL, group=None) -> None:
    """Sum dR and dL over the ranks of `group` in place (every rank gets the total)."""
    import torch.distributed as dist
    dist.all_reduce(dR, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(dL, op=dist.ReduceOp.SUM, group=group)
