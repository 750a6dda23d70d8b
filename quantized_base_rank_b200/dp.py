"""Data parallelism over tokens for the quantised linear.

Every rank holds the same quantised weight and adapter and its own shard of the tokens.
The forward and dX need nothing from other ranks. The adapter gradients are sums over
tokens (dA = s U^T X, dB = s dY^T T), so the full-batch gradients are the sums of the
ranks' partial gradients: the only exchange is one all-reduce of dA and dB. Both go in
one flat fp32 bucket, so the exchange is one collective per layer.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_rows(M: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous token range [start, end) of `rank`: the first M % world ranks get one
    extra row, so the shards differ by at most one row and cover [0, M) exactly once."""
    if world < 1 or not 0 <= rank < world or M < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(M, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_adapter_grads(dA: torch.Tensor, dB: torch.Tensor, group=None) -> None:
    """Sum dA [r, K] and dB [N, r] (fp32) over the ranks of `group`, in place, with one
    collective on a flat bucket."""
    if dA.dtype != torch.float32 or dB.dtype != torch.float32:
        raise TypeError("adapter gradients are fp32")
    bucket = torch.cat([dA.reshape(-1), dB.reshape(-1)])
    dist.all_reduce(bucket, op=dist.ReduceOp.SUM, group=group)
    dA.copy_(bucket[:dA.numel()].view_as(dA))
    dB.copy_(bucket[dA.numel():].view_as(dB))
