"""Data parallelism for the quantised linear: tokens sharded over ranks, and a weight's
quantisation sharded over ranks.

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


GROUP_ELEMS = 64 * 256        # elements per double-quantisation group


def shard_elems(n: int, world: int, rank: int) -> tuple[int, int]:
    """Contiguous element range [start, end) of `rank` for quantising a weight of n
    elements across `world` ranks: whole groups of 256 blocks, split as evenly as
    possible, the ragged tail on the last rank."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError("bad shard request")
    groups = -(-n // GROUP_ELEMS)
    g0, g1 = shard_rows(groups, world, rank)
    return min(n, g0 * GROUP_ELEMS), min(n, g1 * GROUP_ELEMS)


def allreduce_bins(bins: torch.Tensor, group=None) -> None:
    """Sum the exact DQ bins (int64 holding non-negative sums below 2^63) over the ranks."""
    if bins.dtype != torch.int64:
        raise TypeError("bins are int64")
    dist.all_reduce(bins, op=dist.ReduceOp.SUM, group=group)


def quantize_nf4_dq_sharded(W: torch.Tensor, group=None):
    """NF4 + double quantisation of a flattened weight W, each rank quantising its
    shard_elems range, with one integer all-reduce of the exact DQ bins so that the
    per-tensor mean is the whole weight's. Returns this rank's (range, codes, absmax,
    qabsmax, group_scale, mean); every rank's arrays are slices of the single-GPU
    nf4_dq_quantize result, bit for bit."""
    from . import binding as bd
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    flat = W.reshape(-1)
    n = flat.numel()
    s0, s1 = shard_elems(n, world, rank)
    if s1 <= s0:
        raise ValueError("a rank with no elements: use fewer ranks for this weight")
    codes, absmax, bins = bd.nf4_quantize_shard(flat[s0:s1])
    if world > 1:
        allreduce_bins(bins, group)
    qa, gs, mu = bd.dq_quantize_shard(absmax, bins, -(-n // 64))
    return (s0, s1), codes, absmax, qa, gs, mu
