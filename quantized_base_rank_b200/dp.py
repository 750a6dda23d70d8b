"""Data parallelism for the quantised linear: tokens sharded over ranks, and a weight's
quantisation sharded over ranks.

Every rank holds the same quantised weight and adapter and its own shard of the tokens.
The forward and dX need nothing from other ranks. The adapter gradients are sums over
tokens (dA = s U^T X, dB = s dY^T T), so the full-batch gradients are the sums of the
ranks' partial gradients: the only exchange is one all-reduce of dA and dB. For one layer
both go in one flat fp32 bucket (allreduce_adapter_grads). For a stack of layers,
BucketedGradExchange puts several layers' gradients in each bucket and issues each
bucket's all-reduce as soon as its layers' backward has been issued, so the exchange
overlaps the backward of the layers that follow.
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


class BucketedGradExchange:
    """The adapter-gradient exchange of a whole stack, bucketed across layers and
    overlapped with the rest of the backward.

    The backward visits the layers last to first. Each layer's dA [r, K] and dB [N, r]
    (fp32) are views into one flat bucket, so the backward kernels write them in place
    and nothing is copied. Buckets are filled in the order the gradients become ready,
    up to `bucket_cap_bytes` each (a layer never straddles two buckets). As soon as every
    layer of a bucket has reported ready(), the bucket's sum over ranks is issued as an
    asynchronous all-reduce. With NCCL it runs on the library's communication stream after
    the work already queued on the current stream, while the following layers' backward
    kernels run. finish() makes the current stream wait for every bucket. Each bucket is
    summed in one collective with the same element layout on every rank, and a sum of
    world-size-2 contributions has one rounding, so the result is the same bit for bit as
    one all-reduce per layer (allreduce_adapter_grads).

    layers: (r, K, N) per layer, in the order their gradients become ready.
    """

    def __init__(self, layers, bucket_cap_bytes: int = 25 << 20, group=None, device=None):
        if bucket_cap_bytes <= 0:
            raise ValueError("bucket_cap_bytes must be positive")
        self.group = group
        sizes = [r * K + N * r for (r, K, N) in layers]
        if any(r < 1 or K < 1 or N < 1 for (r, K, N) in layers):
            raise ValueError("every layer needs r, K, N >= 1")
        self.layer_bucket, self.layer_offset = [], []
        bucket_elems = []
        for n in sizes:
            if not bucket_elems or (bucket_elems[-1] > 0 and 4 * (bucket_elems[-1] + n) > bucket_cap_bytes):
                bucket_elems.append(0)
            self.layer_bucket.append(len(bucket_elems) - 1)
            self.layer_offset.append(bucket_elems[-1])
            bucket_elems[-1] += n
        self.buckets = [torch.zeros(n, dtype=torch.float32, device=device) for n in bucket_elems]
        self._views = []
        for (r, K, N), b, off in zip(layers, self.layer_bucket, self.layer_offset):
            flat = self.buckets[b]
            self._views.append((flat[off:off + r * K].view(r, K), flat[off + r * K:off + r * K + N * r].view(N, r)))
        self._members = [sum(1 for b in self.layer_bucket if b == i) for i in range(len(self.buckets))]
        self._left = list(self._members)
        self._reported = [False] * len(layers)
        self.works = [None] * len(self.buckets)
        self.launch_order = []                   # bucket indices, in the order they were issued

    def grads(self, layer: int):
        """(dA, dB) of `layer`: the views its backward writes."""
        return self._views[layer]

    def ready(self, layer: int) -> None:
        """The backward of `layer` has been issued on the current stream."""
        if self._reported[layer]:
            raise RuntimeError(f"layer {layer} reported twice in one step")
        self._reported[layer] = True
        b = self.layer_bucket[layer]
        self._left[b] -= 1
        if self._left[b] == 0:
            if dist.is_initialized() and dist.get_world_size(self.group) > 1:
                self.works[b] = dist.all_reduce(self.buckets[b], op=dist.ReduceOp.SUM, group=self.group,
                                                async_op=True)
            self.launch_order.append(b)

    def finish(self) -> None:
        """Wait (on the current stream) for every bucket, then reset for the next step."""
        if not all(self._reported):
            missing = [i for i, r in enumerate(self._reported) if not r]
            raise RuntimeError(f"layers {missing} never reported ready")
        for w in self.works:
            if w is not None:
                w.wait()
        self.works = [None] * len(self.buckets)
        self._left = list(self._members)
        self._reported = [False] * len(self._reported)
        self.launch_order = []


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
