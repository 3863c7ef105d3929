"""Data parallelism for the FP8 blockwise linear layer (host side).

The layer shards over tokens: forward and data-gradient GEMMs need no
exchange, and every rank quantises the replicated weights identically.  The
weight gradient dW = dY^T X contracts over tokens, so each rank produces a
partial dW over its own tokens and the partials are summed across ranks with
one all-reduce (NCCL over NVLink on GPUs).  Shards are whole 128-token
blocks, so no quantisation group (128 consecutive tokens) straddles two ranks
and every rank's codes equal the corresponding slice of a single-GPU run.
"""
from __future__ import annotations


def shard_tokens(tokens: int, rank: int, world: int, block: int = 128) -> tuple[int, int]:
    """[start, stop) of this rank's tokens: whole blocks, as even as possible."""
    if tokens % block:
        raise ValueError(f"token count {tokens} is not a multiple of {block}")
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    nblocks = tokens // block
    base, extra = divmod(nblocks, world)
    start = rank * base + min(rank, extra)
    count = base + (1 if rank < extra else 0)
    return start * block, (start + count) * block


def allreduce_weight_grads(grads, group=None) -> None:
    """Sum the per-rank partial weight gradients in place across the process group."""
    import torch.distributed as dist
    for g in grads:
        dist.all_reduce(g, op=dist.ReduceOp.SUM, group=group)
