"""Data parallelism for the FP8 blockwise linear layer (host side).

The layer shards over tokens: forward and data-gradient GEMMs need no
exchange, and every rank quantises the replicated weights identically.  The
weight gradient dW = dY^T X contracts over tokens, so each rank produces a
partial dW over its own tokens, in fp32, and the partials are summed across
ranks with one all-reduce (NCCL over NVLink on GPUs) and rounded to bf16 once.  Shards are whole 128-token
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


def allreduce_weight_grads(grads, group=None, round_fn=None) -> None:
    """Sum the per-rank partial weight gradients across the process group.

    grads: (partial, out) pairs.  `partial` is this rank's fp32 dW over its own
    tokens (the WGRAD GEMM with fp32 output); it is summed in place in fp32 by
    one all-reduce per gradient, and the sum is rounded once into `out` (bf16)
    by round_fn(partial, out) -- on the GPU the library's
    fp8blk_round_f32_to_bf16.  A single-precision sum followed by one rounding
    differs from a one-GPU run only in the order of the fp32 additions.
    """
    import torch
    import torch.distributed as dist
    if round_fn is None:
        from . import fp8blk_round_f32_to_bf16

        def round_fn(x, y):
            fp8blk_round_f32_to_bf16(x, y)
    for partial, out in grads:
        if partial.dtype != torch.float32 or out.dtype != torch.bfloat16:
            raise ValueError("weight-gradient partials are float32 and their sums bfloat16")
        dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)
        round_fn(partial, out)
