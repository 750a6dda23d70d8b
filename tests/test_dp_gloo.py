"""Data parallelism over tokens, world size 2 on CPU with the gloo backend.

Each rank takes its token shard, computes its partial adapter gradients with the oracle
(fp64 on the host; the GPU kernels compute the same partial sums on the device), and the
ranks exchange them with dp.allreduce_adapter_grads. The sum must equal the full-batch
gradients, and each rank's dX rows must equal the full-batch rows of its shard."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle.qlora_oracle as o
from quantized_base_rank_b200 import dp, synth


def test_shards_cover_every_row_once():
    for M in (0, 1, 2, 3, 7, 64, 8191, 8192):
        for world in (1, 2, 3, 4, 8):
            spans = [dp.shard_rows(M, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == M
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [e - s for s, e in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        dp.shard_rows(8, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CASE = synth.LinearCase("dp-ragged", N=192, K=256, M=131, r=8, alpha=16.0, seed=3)


def _worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = synth.make_inputs(CASE)
        wd = o.quantize_weight(inp["W"].float().numpy(), CASE.fmt)["wdeq"].reshape(CASE.N, CASE.K)
        s0, s1 = dp.shard_rows(CASE.M, world, rank)
        f = lambda t: t.float().numpy().astype(np.float64)
        X, dY, A, B = f(inp["X"])[s0:s1], f(inp["dY"])[s0:s1], f(inp["A"]), f(inp["B"])
        dX, dA, dB = o.linear_bwd(X, dY, wd, A, B, CASE.alpha, CASE.r)
        tA = torch.from_numpy(dA.astype(np.float32))
        tB = torch.from_numpy(dB.astype(np.float32))
        dp.allreduce_adapter_grads(tA, tB)
        results[rank] = (s0, s1, dX, tA.numpy(), tB.numpy())
    finally:
        dist.destroy_process_group()


def test_allreduce_of_partial_gradients_equals_full_batch():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), results), nprocs=world, join=True,
                       start_method="spawn")
    inp = synth.make_inputs(CASE)
    wd = o.quantize_weight(inp["W"].float().numpy(), CASE.fmt)["wdeq"].reshape(CASE.N, CASE.K)
    f = lambda t: t.float().numpy().astype(np.float64)
    dX, dA, dB = o.linear_bwd(f(inp["X"]), f(inp["dY"]), wd, f(inp["A"]), f(inp["B"]), CASE.alpha, CASE.r)
    covered = 0
    for rank in range(world):
        s0, s1, dXr, dAr, dBr = results[rank]
        covered += s1 - s0
        np.testing.assert_allclose(dXr, dX[s0:s1], rtol=0, atol=1e-12)
        # the exchange sums fp32 partials; the reference is the fp64 full batch
        np.testing.assert_allclose(dAr, dA, rtol=1e-5, atol=1e-6 * np.abs(dA).max())
        np.testing.assert_allclose(dBr, dB, rtol=1e-5, atol=1e-6 * np.abs(dB).max())
        if rank:
            assert np.array_equal(dAr, results[0][3]) and np.array_equal(dBr, results[0][4])
    assert covered == CASE.M


def test_quantise_shards_are_whole_groups():
    for n in (1, 64, 16384, 16385, 3 * 16384 + 5, 4096 * 4096, 22016 * 8192):
        for world in (1, 2, 3, 8):
            spans = [dp.shard_elems(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            assert all(a % dp.GROUP_ELEMS == 0 for a, b in spans if b > a)   # empty shards are refused


def _bins_worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # values near 2^62: the sum must stay exact in int64
        bins = torch.tensor([(1 << 61) + 12345 * (rank + 1) + i for i in range(16)], dtype=torch.int64)
        dp.allreduce_bins(bins)
        results[rank] = bins.tolist()
    finally:
        dist.destroy_process_group()


def test_bin_allreduce_is_exact():
    world = 2
    results = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_bins_worker, args=(world, _free_port(), results), nprocs=world, join=True,
                       start_method="spawn")
    want = [sum((1 << 61) + 12345 * (r + 1) + i for r in range(world)) for i in range(16)]
    assert results[0] == want and results[1] == want


def _step_worker(rank, world, port, results):
    """A data-parallel training step of the adapter: partial gradients of the shard, the
    all-reduce, then the optimiser step with the 1/world gradient scale (AdamW) and the
    Lion INT8 step on the averaged gradient, both with the oracle on the host."""
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = synth.make_inputs(CASE)
        wd = o.quantize_weight(inp["W"].float().numpy(), CASE.fmt)["wdeq"].reshape(CASE.N, CASE.K)
        s0, s1 = dp.shard_rows(CASE.M, world, rank)
        f = lambda t: t.float().numpy().astype(np.float64)
        A, B = f(inp["A"]), f(inp["B"])
        _, dA, dB = o.linear_bwd(f(inp["X"])[s0:s1], f(inp["dY"])[s0:s1], wd, A, B, CASE.alpha, CASE.r)
        tA = torch.from_numpy(dA.astype(np.float32))
        tB = torch.from_numpy(dB.astype(np.float32))
        dp.allreduce_adapter_grads(tA, tB)
        g = np.concatenate([tA.numpy().ravel(), tB.numpy().ravel()])
        theta0 = np.concatenate([A.ravel(), B.ravel()]).astype(np.float32)
        n = theta0.size
        th_adam = o.adamw_step(theta0, g, np.zeros(n), np.zeros(n), 1, 1e-3, 0.9, 0.999, 1e-8, 0.01,
                               grad_scale=1.0 / world)[0]
        g_mean = (g / np.float32(world)).astype(np.float32)
        th_lion, codes, amax, _ = o.lion_int8_step(theta0, g_mean, np.zeros(n, np.int8),
                                                   np.zeros((n + 63) // 64, np.float32), 1e-4, 0.9, 0.99, 0.1)
        results[rank] = (th_adam, th_lion, codes, amax)
    finally:
        dist.destroy_process_group()


def test_data_parallel_step_with_optimisers_keeps_replicas_identical():
    """After the exchange every rank takes the same optimiser step: the replicas are
    bit-identical, and equal (within the fp32 exchange's rounding) to one process stepping
    on the averaged full-batch gradient."""
    world = 2
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_step_worker, args=(world, _free_port(), results), nprocs=world, join=True,
                       start_method="spawn")
    r0, r1 = results[0], results[1]
    for a, b in zip(r0, r1):
        assert np.array_equal(np.asarray(a), np.asarray(b))
    inp = synth.make_inputs(CASE)
    wd = o.quantize_weight(inp["W"].float().numpy(), CASE.fmt)["wdeq"].reshape(CASE.N, CASE.K)
    f = lambda t: t.float().numpy().astype(np.float64)
    A, B = f(inp["A"]), f(inp["B"])
    _, dA, dB = o.linear_bwd(f(inp["X"]), f(inp["dY"]), wd, A, B, CASE.alpha, CASE.r)
    g = np.concatenate([dA.ravel(), dB.ravel()]) / world
    theta0 = np.concatenate([A.ravel(), B.ravel()])
    n = theta0.size
    th_ref = o.adamw_step(theta0, g, np.zeros(n), np.zeros(n), 1, 1e-3, 0.9, 0.999, 1e-8, 0.01)[0]
    np.testing.assert_allclose(r0[0], th_ref, rtol=1e-6, atol=1e-9)
    # Lion moves every element by lr against sign(c); the same signs as the single process
    # wherever the averaged gradient is not within the exchange's rounding of zero
    sure = np.abs(g) > 1e-6 * np.abs(g).max()
    step = r0[1].astype(np.float64) - theta0.astype(np.float32).astype(np.float64) * (1 - 1e-5)
    assert np.all(np.sign(step[sure]) == -np.sign(g[sure]))


# ---- bucketed, overlapped exchange across the layers of a stack ----------------------

STACK = [synth.LinearCase(f"dp-stack-{i}", N=N, K=K, M=97, r=r, alpha=16.0, seed=20 + i)
         for i, (N, K, r) in enumerate([(128, 192, 8), (256, 128, 16), (64, 256, 4), (192, 64, 32),
                                        (128, 128, 8)])]
CAP = 4 * (8 * 192 + 128 * 8 + 16 * 128 + 256 * 16)   # the first two layers fill one bucket


def _stack_worker(rank, world, port, results):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        order = list(reversed(range(len(STACK))))          # the backward goes last layer first
        ex = dp.BucketedGradExchange([(STACK[i].r, STACK[i].K, STACK[i].N) for i in order], CAP)
        partial = {}
        issued_before_last = []
        for j, i in enumerate(order):
            c = STACK[i]
            inp = synth.make_inputs(c)
            wd = o.quantize_weight(inp["W"].float().numpy(), c.fmt)["wdeq"].reshape(c.N, c.K)
            s0, s1 = dp.shard_rows(c.M, world, rank)
            f = lambda t: t.float().numpy().astype(np.float64)
            _, dA, dB = o.linear_bwd(f(inp["X"])[s0:s1], f(inp["dY"])[s0:s1], wd, f(inp["A"]), f(inp["B"]),
                                     c.alpha, c.r)
            gA, gB = ex.grads(j)
            gA.copy_(torch.from_numpy(dA.astype(np.float32)))
            gB.copy_(torch.from_numpy(dB.astype(np.float32)))
            partial[i] = (gA.clone(), gB.clone())
            ex.ready(j)
            if j < len(order) - 1:
                issued_before_last.append(list(ex.launch_order))
        ex.finish()
        seq = {}
        for i in order:                                      # one all-reduce per layer
            tA, tB = partial[i]
            dp.allreduce_adapter_grads(tA, tB)
            seq[i] = (tA.numpy(), tB.numpy())
        got = {i: tuple(t.clone().numpy() for t in ex.grads(j)) for j, i in enumerate(order)}
        results[rank] = (got, seq, issued_before_last, ex.layer_bucket, len(ex.buckets))
    finally:
        dist.destroy_process_group()


def test_bucketed_overlapped_exchange_equals_per_layer_allreduce():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    results = mgr.dict()
    mp.start_processes(_stack_worker, args=(world, _free_port(), results), nprocs=world, join=True,
                       start_method="spawn")
    for rank in range(world):
        got, seq, issued, layer_bucket, nb = results[rank]
        assert nb >= 3 and layer_bucket == sorted(layer_bucket)
        # each bucket's collective is issued as soon as its last layer is ready, before the
        # backward of the remaining layers has been issued
        assert issued[-1] == list(range(nb - 1))
        for i in got:
            assert np.array_equal(got[i][0], seq[i][0]) and np.array_equal(got[i][1], seq[i][1])
            if rank:
                assert np.array_equal(got[i][0], results[0][0][i][0])
    # and the summed gradients are the full-batch ones
    got = results[0][0]
    for i, c in enumerate(STACK):
        inp = synth.make_inputs(c)
        wd = o.quantize_weight(inp["W"].float().numpy(), c.fmt)["wdeq"].reshape(c.N, c.K)
        f = lambda t: t.float().numpy().astype(np.float64)
        _, dA, dB = o.linear_bwd(f(inp["X"]), f(inp["dY"]), wd, f(inp["A"]), f(inp["B"]), c.alpha, c.r)
        np.testing.assert_allclose(got[i][0], dA, rtol=1e-5, atol=1e-6 * np.abs(dA).max())
        np.testing.assert_allclose(got[i][1], dB, rtol=1e-5, atol=1e-6 * np.abs(dB).max())


def test_bucket_plan_without_a_process_group():
    layers = [(8, 192, 128), (16, 128, 256), (4, 256, 64)]
    ex = dp.BucketedGradExchange(layers, bucket_cap_bytes=1)      # one layer per bucket
    assert ex.layer_bucket == [0, 1, 2]
    ex = dp.BucketedGradExchange(layers, bucket_cap_bytes=1 << 30)
    assert ex.layer_bucket == [0, 0, 0] and ex.buckets[0].numel() == sum(r * (K + N) for r, K, N in layers)
    dA, dB = ex.grads(1)
    assert dA.shape == (16, 128) and dB.shape == (256, 16) and dA.is_contiguous() and dB.is_contiguous()
    for i in range(3):
        ex.ready(i)
    with pytest.raises(RuntimeError):
        ex.ready(0)
    ex.finish()
    with pytest.raises(RuntimeError):
        ex.finish()                                              # nothing reported this step
