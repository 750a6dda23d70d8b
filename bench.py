#!/usr/bin/env python
"""Benchmark of the QLoRA-style quantised linear on B200.

One step = the whole hot path on one batch: NF4 quantisation + double quantisation of
the frozen bf16 weight, the fused forward Y = X W'^T + s (X A^T) B^T, and the backward
(dX, dA, dB). Workload: the fine-tune-shaped MLP up-projection (W 11008x4096 ~N(0,0.02),
X 8192x4096 ~N(0,1), LoRA r=64, alpha=16, dY ~N(0,1)), seeded synthetic data.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun (N > 1) every rank runs its own batch (weak scaling) and the adapter
gradients dA, dB are summed across ranks with NCCL, the data-parallel exchange step.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused NF4+LoRA linear TFLOP/s & HBM GB/s (% of roofline); quantize GB/s"
NF4_DQ_BYTES_PER_PARAM = 2.0 + 0.5 + 1.0 / 64 + 4.0 / 16384   # bf16 read + codes + consts

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the fused
# forward GEMM on this workload, from one ncu capture (profiles/fwd_main_gemm_upproj_11008x4096_M8192.md),
# valid only for the kernel sources it was taken on: reported as null once they change.
FWD_MAIN_TRAFFIC = {"bytes": 99780096 + 149417216, "sources_sha256_16": "8c3563e70db2e8d6"}
FWD_MAIN_SOURCES = ("quantized_base_rank_b200/csrc/gemm.cuh", "quantized_base_rank_b200/csrc/sm100.cuh",
                    "quantized_base_rank_b200/csrc/linear.cu", "quantized_base_rank_b200/csrc/common.cuh")


def sources_sha256_16(paths) -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def fwd_main_traffic():
    ok = sources_sha256_16(FWD_MAIN_SOURCES) == FWD_MAIN_TRAFFIC["sources_sha256_16"]
    return FWD_MAIN_TRAFFIC["bytes"] if ok else None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def linear_flops(M, N, K, r):
    fwd = 2 * M * N * K + 2 * M * K * r + 2 * M * N * r
    bwd = (2 * M * N * K + 2 * M * N * r + 2 * M * r * K) + 2 * M * r * K + 2 * M * N * r
    return fwd, bwd


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples taken while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            target = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            target = str(device_index)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", target], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# --------------------------------------------------------------------------------------
# CPU oracle leg (reported baseline / reference arm)
# --------------------------------------------------------------------------------------

def oracle_step(inp_np, case, m_rows: int, n_rows: int):
    """One bounded sample of the step on the host: quantise n_rows rows of W (NF4 + DQ),
    then forward + backward in fp64 for m_rows tokens over the full weight."""
    import oracle.qlora_oracle as o
    w = inp_np["W"]
    t0 = time.perf_counter()
    o.quantize_weight(w[:n_rows], "nf4_dq")
    wd = inp_np["Wd"]
    X = inp_np["X"][:m_rows]
    dY = inp_np["dY"][:m_rows]
    o.linear_fwd(X, wd, inp_np["A"], inp_np["B"], case.alpha, case.r)
    o.linear_bwd(X, dY, wd, inp_np["A"], inp_np["B"], case.alpha, case.r)
    dt = time.perf_counter() - t0
    f, b = linear_flops(m_rows, case.N, case.K, case.r)
    return dt, f + b


def oracle_inputs(case):
    """The oracle's inputs, with the full-weight quantisations timed on the way (NF4+DQ,
    which also gives the dequantised weight, and blockwise int8), as GB/s of algorithmic
    bytes (2.516 and 3.0625 B/param) on the host's cores."""
    import oracle.qlora_oracle as o
    from quantized_base_rank_b200 import synth
    inp = synth.make_inputs(case)
    f = lambda t: t.float().numpy()
    w = f(inp["W"])
    t0 = time.perf_counter()
    wd = o.quantize_weight(w, "nf4_dq")["wdeq"].reshape(case.N, case.K).astype(np.float64)
    t_nf4 = time.perf_counter() - t0
    t0 = time.perf_counter()
    o.quantize_weight(w, "int8")
    t_i8 = time.perf_counter() - t0
    n = w.size
    timing = {"nf4_dq_quantize_and_dequant": {"s": t_nf4, "GB/s": NF4_DQ_BYTES_PER_PARAM * n / t_nf4 / 1e9},
              "int8_quantize_and_dequant": {"s": t_i8, "GB/s": 3.0625 * n / t_i8 / 1e9}}
    return {"W": w, "Wd": wd, "X": f(inp["X"]).astype(np.float64), "A": f(inp["A"]).astype(np.float64),
            "B": f(inp["B"]).astype(np.float64), "dY": f(inp["dY"]).astype(np.float64), "timing": timing}


def blas_threads() -> int:
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        return max(i.get("num_threads", 1) for i in info) if info else os.cpu_count()
    except Exception:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return "unknown"


def run_reference(args, case, world, rank):
    if rank != 0:
        return
    inp = oracle_inputs(case)
    # per step: 256 weight rows quantised, 32 tokens through fwd + bwd over the full weight
    m_rows, n_rows = 32, 256
    for _ in range(args.warmup):
        oracle_step(inp, case, m_rows, n_rows)
    tot_t, tot_f = 0.0, 0.0
    for _ in range(args.steps):
        dt, fl = oracle_step(inp, case, m_rows, n_rows)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    sample = (f"each step: NF4+DQ quantise of {n_rows} of {case.N} weight rows, fp64 forward + "
              f"backward for {m_rows} of {case.M} tokens over the full {case.N}x{case.K} weight")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * tot_t / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": case.name, "M": case.M, "N": case.N, "K": case.K, "r": case.r,
                       "alpha": case.alpha, "format": "nf4_dq"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": blas_threads(),
                             "kind": "oracle", "sample": sample, "cpu": cpu_model(),
                             "components": inp["timing"]},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------------------
# GPU leg
# --------------------------------------------------------------------------------------

def decode_bench(dev, peaks, reps: int = 20):
    """Decode-shaped forward (7B 4096x4096 NF4+DQ linear, r=16, M in {1, 4, 16}): GB/s of
    algorithmic bytes per call. Back-to-back calls rotate over enough quantised weight
    copies to exceed three times the L2 size, inside one CUDA graph, so each call reads its
    weight from HBM; the graph is replayed `reps` times and timed with CUDA events."""
    from quantized_base_rank_b200 import binding as B
    from quantized_base_rank_b200 import synth
    out = {}
    base = synth.CFG2[0]
    W = synth.weight_with_outliers(base.N, base.K, base.w_std, base.outlier_frac, base.outlier_mult,
                                   base.seed).to(dev)
    q0 = B.quantize_weight(W, "nf4_dq")
    del W
    n = base.N * base.K
    wbytes = n * (0.5 + 1.0 / 64) + 4.0 * n / 16384
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copies = max(4, int(np.ceil(3 * l2 / wbytes)))
    qws = [B.QuantWeight("nf4_dq", base.N, base.K, q0.codes.clone(), None, q0.qabsmax.clone(),
                         q0.group_scale.clone(), q0.mean.clone()) for _ in range(copies)]
    for case in synth.CFG2:
        M, N, K, r = case.M, case.N, case.K, case.r
        inp = synth.make_inputs(case)
        X, A, Bm = (inp[k].to(dev) for k in ("X", "A", "B"))
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        T = torch.empty((M, r), dtype=torch.bfloat16, device=dev)
        for qw in qws[:2]:
            B.linear_fwd(qw, X, A, Bm, case.alpha, Y=Y, T=T)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream(dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for qw in qws:
                    B.linear_fwd(qw, X, A, Bm, case.alpha, Y=Y, T=T)
        torch.cuda.synchronize()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / (reps * copies)
        nbytes = wbytes + 2 * M * K + 2 * r * K + 2 * N * r + 2 * M * N
        gbs = nbytes / (us * 1e-6) / 1e9
        out[f"M{M}"] = {"us_per_call": us, "bytes": nbytes, "GB/s": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
                        "frac_8tbs": gbs / 8000.0, "weight_copies": copies}
        del g
    return out


def lordba_bench(dev, peaks, qw_up, X_up, reps: int = 10):
    """The LoRDBA double-binary adapter branch: (1) the up-projection forward (8192 tokens,
    R = 64, one envelope term) against the same forward with a dense r = 64 adapter;
    (2) the decode-shaped 4096x4096 NF4+DQ layer at M = 1, R = 16, timed like the dense
    decode component (a CUDA graph over weight copies exceeding 3x L2)."""
    from quantized_base_rank_b200 import binding as B
    from quantized_base_rank_b200 import synth
    out = {}
    N, K = qw_up.N, qw_up.K
    ad = synth.lordba_inputs(N, K, 64, 1, 3)
    B1p, B2p = B.pack_signs(ad["B1"].to(dev)), B.pack_signs(ad["B2"].to(dev))
    al, be, ga = (ad[k].to(dev) for k in ("alpha", "beta", "gamma"))
    Y = torch.empty((X_up.shape[0], N), dtype=torch.bfloat16, device=dev)
    A_d = synth.normal_bf16((64, K), 0.02, 7, 0).to(dev)
    B_d = synth.normal_bf16((N, 64), 0.02, 7, 1).to(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(call):
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            call()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    # the dense rank-64 forward timed the same way, right before, as the comparison
    ms_dense = timed(lambda: B.linear_fwd(qw_up, X_up, A_d, B_d, 64.0, save_T=False, Y=Y))
    ms = timed(lambda: B.linear_fwd_lordba(qw_up, X_up, B1p, B2p, al, be, ga, 64, Y=Y))
    M = X_up.shape[0]
    flops = 2 * M * N * K + 2 * M * K * 64 + 2 * M * N * 64
    carrier_bytes = (N * 64 + 64 * K) / 8 + 2 * (N + 64 + K)
    out["upproj_R64"] = {"ms": ms, "TFLOP/s": flops / (ms * 1e-3) / 1e12, "dense_r64_ms": ms_dense,
                         "adapter_bytes": carrier_bytes, "dense_adapter_bytes": 2 * 64 * (N + K)}
    # decode-shaped
    base = synth.CFG2[0]
    W = synth.weight_with_outliers(base.N, base.K, base.w_std, base.outlier_frac, base.outlier_mult,
                                   base.seed).to(dev)
    q0 = B.quantize_weight(W, "nf4_dq")
    del W
    n = base.N * base.K
    ad = synth.lordba_inputs(base.N, base.K, 16, 1, 4)
    B1p, B2p = B.pack_signs(ad["B1"].to(dev)), B.pack_signs(ad["B2"].to(dev))
    al, be, ga = (ad[k].to(dev) for k in ("alpha", "beta", "gamma"))
    wbytes = n * (0.5 + 1.0 / 64) + 4.0 * n / 16384
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copies = max(4, int(np.ceil(3 * l2 / wbytes)))
    qws = [B.QuantWeight("nf4_dq", base.N, base.K, q0.codes.clone(), None, q0.qabsmax.clone(),
                         q0.group_scale.clone(), q0.mean.clone()) for _ in range(copies)]
    X = synth.normal_bf16((1, base.K), 1.0, 5, 0).to(dev)
    Y = torch.empty((1, base.N), dtype=torch.bfloat16, device=dev)
    for qw in qws[:2]:
        B.linear_fwd_lordba(qw, X, B1p, B2p, al, be, ga, 16, Y=Y)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    st = torch.cuda.Stream(dev)
    st.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(st):
        with torch.cuda.graph(g, stream=st):
            for qw in qws:
                B.linear_fwd_lordba(qw, X, B1p, B2p, al, be, ga, 16, Y=Y)
    torch.cuda.synchronize()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    us = e0.elapsed_time(e1) * 1e3 / (reps * copies)
    nbytes = wbytes + 2 * base.K + (base.N * 16 + 16 * base.K) / 8 + 2 * (base.N + 16 + base.K) + 2 * base.N
    out["decode_7b_4096x4096_M1_R16"] = {"us_per_call": us, "bytes": nbytes,
                                        "GB/s": nbytes / (us * 1e-6) / 1e9,
                                        "frac_hbm": nbytes / (us * 1e-6) / 1e9 / peaks["hbm_gbs"]}
    del g
    return out


def qwha_bench(dev, peaks, qw_up, X_up, reps: int = 10):
    """The Walsh-Hadamard adapter (Delta W = F H^{-1}, sparse F): (1) the up-projection
    forward at 8192 tokens with a budget of a rank-64 LoRA (64 (N + K) values), beside the
    dense rank-64 forward timed the same way, and the transform kernel alone; (2) the
    decode-shaped 4096x4096 NF4+DQ layer at M = 1 with a rank-16 budget, timed like the
    dense decode component (a CUDA graph over weight copies exceeding 3x L2), beside the
    dense rank-16 adapter timed the same way."""
    from quantized_base_rank_b200 import binding as B
    from quantized_base_rank_b200 import synth
    out = {}
    N, K = qw_up.N, qw_up.K
    M = X_up.shape[0]
    ad = synth.qwha_inputs(N, K, 64, 5)
    rp, col, c = ad["row_ptr"].to(dev), ad["col"].to(dev), ad["c"].to(dev)
    nnz = c.numel()
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    A_d = synth.normal_bf16((64, K), 0.02, 7, 0).to(dev)
    B_d = synth.normal_bf16((N, 64), 0.02, 7, 1).to(dev)
    Z = torch.empty_like(X_up)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(call, n=reps):
        for _ in range(3):
            call()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(n):
            call()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    ms_dense = timed(lambda: B.linear_fwd(qw_up, X_up, A_d, B_d, 64.0, save_T=False, Y=Y))
    ms = timed(lambda: B.linear_fwd_qwha(qw_up, X_up, rp, col, c, Y=Y))
    ms_wht = timed(lambda: B.wht(X_up, Z))
    wht_bytes = 2 * M * K * 2
    useful = 2 * M * N * K + 2 * M * nnz
    out["upproj_r64_budget"] = {
        "ms": ms, "TFLOP/s_useful": useful / (ms * 1e-3) / 1e12, "dense_lora_r64_ms": ms_dense, "nnz": nnz,
        "adapter_bytes": nnz * 4 + (N + 1) * 4, "dense_lora_bytes": 2 * 64 * (N + K),
        "wht_us": ms_wht * 1e3, "wht_GB/s": wht_bytes / (ms_wht * 1e-3) / 1e9,
        "wht_frac_hbm": wht_bytes / (ms_wht * 1e-3) / 1e9 / peaks["hbm_gbs"]}
    del Y, Z
    # decode-shaped
    base = synth.CFG2[0]
    W = synth.weight_with_outliers(base.N, base.K, base.w_std, base.outlier_frac, base.outlier_mult,
                                   base.seed).to(dev)
    q0 = B.quantize_weight(W, "nf4_dq")
    del W
    n = base.N * base.K
    ad = synth.qwha_inputs(base.N, base.K, 16, 6)
    rp, col, c = ad["row_ptr"].to(dev), ad["col"].to(dev), ad["c"].to(dev)
    nnz = c.numel()
    A16 = synth.normal_bf16((16, base.K), 0.02, 8, 0).to(dev)
    B16 = synth.normal_bf16((base.N, 16), 0.02, 8, 1).to(dev)
    wbytes = n * (0.5 + 1.0 / 64) + 4.0 * n / 16384
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copies = max(4, int(np.ceil(3 * l2 / wbytes)))
    qws = [B.QuantWeight("nf4_dq", base.N, base.K, q0.codes.clone(), None, q0.qabsmax.clone(),
                         q0.group_scale.clone(), q0.mean.clone()) for _ in range(copies)]
    X = synth.normal_bf16((1, base.K), 1.0, 5, 0).to(dev)
    Y = torch.empty((1, base.N), dtype=torch.bfloat16, device=dev)

    def graph_us(call):
        for qw in qws[:2]:
            call(qw)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        st = torch.cuda.Stream(dev)
        st.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(st):
            with torch.cuda.graph(g, stream=st):
                for qw in qws:
                    call(qw)
        torch.cuda.synchronize()
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(2 * reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) * 1e3 / (2 * reps * copies)

    us = graph_us(lambda qw: B.linear_fwd_qwha(qw, X, rp, col, c, Y=Y))
    us_lora = graph_us(lambda qw: B.linear_fwd(qw, X, A16, B16, 32.0, save_T=False, Y=Y))
    nbytes = wbytes + 2 * base.K + nnz * 4 + (base.N + 1) * 4 + 2 * base.N
    out["decode_7b_4096x4096_M1_r16_budget"] = {
        "us_per_call": us, "dense_lora_r16_us": us_lora, "nnz": nnz, "bytes": nbytes,
        "GB/s": nbytes / (us * 1e-6) / 1e9, "frac_hbm": nbytes / (us * 1e-6) / 1e9 / peaks["hbm_gbs"]}
    return out


def optim_bench(dev, peaks, reps: int = 10):
    """The adapter optimiser step (AdamW) over every adapter parameter of the 7B stack at
    rank 64 (one flat vector), 30 bytes per parameter. States (theta, m, v) in paged
    (managed) memory resident on the device, beside the same step on plain device memory;
    and once with the states paged out to the host before the step (the migration cost)."""
    from quantized_base_rank_b200 import binding as B
    from quantized_base_rank_b200 import stack
    n = sum(sp.r * (sp.N + sp.K) for sp in stack.stack_7b())
    n = (n + 3) // 4 * 4
    g = torch.empty(n, device=dev).normal_(0.0, 1e-3, generator=torch.Generator(dev).manual_seed(3))
    param = torch.empty(n, dtype=torch.bfloat16, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    hp = dict(lr=1e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0)

    def timed(theta, m, v, before=None, n_steps=reps):
        B.adamw_step(theta, param, g, m, v, 1, **hp)
        torch.cuda.synchronize()
        total = 0.0
        for t in range(n_steps):
            if before is not None:
                before()
                torch.cuda.synchronize()
            e0.record()
            B.adamw_step(theta, param, g, m, v, t + 2, **hp)
            e1.record()
            torch.cuda.synchronize()
            total += e0.elapsed_time(e1)
        return total / n_steps

    dense = [torch.zeros(n, device=dev) for _ in range(3)]
    ms_dev = timed(*dense)
    del dense
    buf = B.PagedBuffer(3 * n * 4)
    th, m, v = (buf.view(torch.float32, n, i * n * 4) for i in range(3))
    th.zero_()
    m.zero_()
    v.zero_()
    buf.prefetch(to_host=False)
    ms_paged = timed(th, m, v)
    ms_paged_in = timed(th, m, v, before=lambda: buf.prefetch(to_host=True), n_steps=2)
    buf.prefetch(to_host=False)
    torch.cuda.synchronize()
    del th, m, v
    buf.free()
    # Lion with INT8 momentum on the same parameters: 16 bytes per parameter
    theta = torch.zeros(n, device=dev)
    codes = torch.zeros(n, dtype=torch.int8, device=dev)
    amax = torch.zeros((n + 63) // 64, device=dev)
    for _ in range(3):
        B.lion_int8_step(theta, param, g, codes, amax, 1e-4)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps):
        B.lion_int8_step(theta, param, g, codes, amax, 1e-4)
    e1.record()
    torch.cuda.synchronize()
    ms_lion = e0.elapsed_time(e1) / reps
    lion_bytes = 16 * n + 8 * ((n + 63) // 64)
    del theta, codes, amax
    nbytes = 30 * n
    return {"params": n, "bytes_per_step": nbytes,
            "lion_int8": {"ms": ms_lion, "bytes_per_step": lion_bytes,
                          "GB/s": lion_bytes / (ms_lion * 1e-3) / 1e9,
                          "frac_hbm": lion_bytes / (ms_lion * 1e-3) / 1e9 / peaks["hbm_gbs"]},
            "paged_resident": {"ms": ms_paged, "GB/s": nbytes / (ms_paged * 1e-3) / 1e9,
                               "frac_hbm": nbytes / (ms_paged * 1e-3) / 1e9 / peaks["hbm_gbs"]},
            "device_memory": {"ms": ms_dev, "GB/s": nbytes / (ms_dev * 1e-3) / 1e9},
            "paged_in_from_host": {"ms": ms_paged_in, "state_bytes_migrated": 12 * n}}


def run_ours(args, case, world, rank, local_rank):
    from quantized_base_rank_b200 import binding as B
    from quantized_base_rank_b200 import dp, synth

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    B.lib().ql_set_gemm_pair(1 if args.gemm == "pair" else 0)
    dist = None
    if world > 1:
        import torch.distributed as dist

    peaks = load_peaks()
    seed_case = synth.LinearCase(**{**case.__dict__, "seed": case.seed + rank})
    inp = synth.make_inputs(seed_case)
    M, N, K, r = case.M, case.N, case.K, case.r
    W = inp["W"].to(dev)
    X, A, Bm, dY = (inp[k].to(dev) for k in ("X", "A", "B", "dY"))
    n = N * K
    codes = torch.empty(n // 2, dtype=torch.uint8, device=dev)
    absmax = torch.empty(n // 64, dtype=torch.float32, device=dev)
    qa = torch.empty(n // 64, dtype=torch.int8, device=dev)
    gs = torch.empty((n // 64 + 255) // 256, dtype=torch.float32, device=dev)
    mu = torch.empty(1, dtype=torch.float32, device=dev)
    qw = B.QuantWeight("nf4_dq", N, K, codes, None, qa, gs, mu)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    T = torch.empty((M, r), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    dA = torch.empty((r, K), dtype=torch.float32, device=dev)
    dB = torch.empty((N, r), dtype=torch.float32, device=dev)

    def step():
        B.nf4_dq_quantize(W, codes, absmax, qa, gs, mu)
        B.linear_fwd(qw, X, A, Bm, case.alpha, Y=Y, T=T)
        B.linear_bwd(qw, X, dY, A, Bm, T, case.alpha, dX=dX, dA=dA, dB=dB)
        if dist is not None:
            dp.allreduce_adapter_grads(dA, dB)

    def barrier():
        if dist is not None:
            dist.barrier()

    def timed(fn, steps):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(steps):
            fn()
        e.record()
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        ms = s.elapsed_time(e) / steps
        if dist is not None:
            t = torch.tensor([ms], device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ms = float(t.item())
        return ms

    # ---- device-resident timed region ----
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier()
    for g in B.PROFILE_GROUPS:
        B.profile_read(g)                     # drop anything recorded so far
    clocks = ClockSampler(dev.index) if rank == 0 else None
    B.profile_enable(True)
    c0 = B.launch_count()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ev_s, ev_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev_s.record()
    for _ in range(args.steps):
        step()
    ev_e.record()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    B.profile_enable(False)
    launches = B.launch_count() - c0
    clk = clocks.stop() if clocks else None
    ms = ev_s.elapsed_time(ev_e) / args.steps
    if dist is not None:
        t = torch.tensor([ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    prof = {g: B.profile_read(g) for g in B.PROFILE_GROUPS}
    assert B.device_status() == B.QL_OK

    fwd_f, bwd_f = linear_flops(M, N, K, r)
    value = world * (fwd_f + bwd_f) / (ms * 1e-3) / 1e12

    def avg(g):
        t, c = prof[g]
        return t / c if c else float("nan")

    fwd_ms = sum(avg(g) for g in ("fwd_prep", "fwd_xa", "fwd_main"))
    bwd_ms = sum(avg(g) for g in ("bwd_prep", "bwd_dyb", "bwd_db", "bwd_da", "bwd_dx"))
    # the one-launch NF4+DQ path records no separate DQ group
    q_ms = avg("nf4") + (avg("dq") if prof["dq"][1] else 0.0)
    main_flops = 2 * M * N * (K + r)                # algorithmic work of the fused forward GEMM
    main_ms = avg("fwd_main")
    achieved = main_flops / (main_ms * 1e-3) / 1e12
    dx_ms = avg("bwd_dx")
    dx_flops = 2 * M * N * K + 2 * M * r * K

    # ---- end-to-end through the public API with host buffers ----
    pin = lambda t: t.pin_memory()
    hW, hX, hA, hB, hdY = (pin(inp[k]) for k in ("W", "X", "A", "B", "dY"))
    hdA = torch.empty_like(dA, device="cpu").pin_memory()
    hdB = torch.empty_like(dB, device="cpu").pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (hW, hX, hA, hB, hdY))
    d2h = hdA.numel() * 4 + hdB.numel() * 4

    # Pipelined through two input sets: step i computes on set i % 2 while a copy stream
    # brings step i + 1's inputs from pinned host memory into the other set. Every step's
    # inputs are copied once; a timed region of K steps holds K full input copies (the
    # first timed step's set arrives in the step before it). Events keep a set's copy after
    # the compute that last read it, and the compute after its copy.
    sets = [(W, X, A, Bm, dY), tuple(torch.empty_like(t) for t in (W, X, A, Bm, dY))]
    hsets = (hW, hX, hA, hB, hdY)
    copy_stream = torch.cuda.Stream(dev)
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    used = [torch.cuda.Event(), torch.cuda.Event()]
    e2e_state = {"i": 0}

    def copy_set(j):
        copy_stream.wait_event(used[j])
        with torch.cuda.stream(copy_stream):
            for d, h in zip(sets[j], hsets):
                d.copy_(h, non_blocking=True)
            copied[j].record(copy_stream)

    def e2e_step():
        i = e2e_state["i"]
        j = i % 2
        cur = torch.cuda.current_stream(dev)
        if i == 0:
            copy_set(j)
            cur.wait_event(copied[j])
        copy_set(1 - j)                                  # the next step's inputs
        Wj, Xj, Aj, Bj, dYj = sets[j]
        B.nf4_dq_quantize(Wj, codes, absmax, qa, gs, mu)
        B.linear_fwd(qw, Xj, Aj, Bj, case.alpha, Y=Y, T=T)
        B.linear_bwd(qw, Xj, dYj, Aj, Bj, T, case.alpha, dX=dX, dA=dA, dB=dB)
        if dist is not None:
            dp.allreduce_adapter_grads(dA, dB)
        used[j].record(cur)
        hdA.copy_(dA, non_blocking=True)
        hdB.copy_(dB, non_blocking=True)
        # the step ends when the next step's inputs are in, so a timed region that closes
        # after this step holds every copy it started
        cur.wait_event(copied[1 - j])
        e2e_state["i"] = i + 1

    e2e_steps = max(3, args.steps // 10)
    e2e_ms = timed(e2e_step, e2e_steps)
    e2e_value = world * (fwd_f + bwd_f) / (e2e_ms * 1e-3) / 1e12

    # ---- decode-shaped forward (small M, HBM-bound) ----
    decode = decode_bench(dev, peaks)

    # ---- LoRDBA double-binary adapter branch ----
    lordba = lordba_bench(dev, peaks, qw, X)

    # ---- Walsh-Hadamard (QWHA) adapter ----
    qwha = qwha_bench(dev, peaks, qw, X)

    # ---- adapter optimiser step with paged states ----
    optim = optim_bench(dev, peaks)

    # ---- CPU oracle baseline (rank 0, one GPU only) ----
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        o_inp = oracle_inputs(case)
        m_rows, n_rows = 1024, case.N
        dt, fl = oracle_step(o_inp, case, m_rows, n_rows)
        cpu = {"value": fl / dt / 1e12, "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": (f"one step with the full {N}x{K} weight quantised (NF4+DQ) and fp64 "
                          f"forward + backward for {m_rows} of {M} tokens; {dt:.1f} s"),
               "cpu": cpu_model(), "components": o_inp["timing"]}

    if rank != 0:
        return
    if peaks.get("bf16_tflops_sustained"):
        peak_fwd = peaks["bf16_tflops_sustained"]
        peak_fwd_source = f"{peaks['source']} bf16 sustained (kernel timed inside {args.steps} steps)"
    else:
        peak_fwd = peaks["bf16_tflops"]
        peak_fwd_source = f"{peaks['source']} bf16 burst (no sustained figure)"
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": case.name, "M": M, "N": N, "K": K, "r": r, "alpha": case.alpha,
                   "format": "nf4_dq", "step": "quantise(NF4+DQ) + fwd + bwd(dX,dA,dB)",
                   "l2": "inputs larger than L2 (X 64 MB, W 90 MB, dY 180 MB > 126 MB)",
                   "parallelism": f"dp{world}" if world > 1 else "single",
                   "fused_gemm": "cta_pair" if args.gemm == "pair" else "single_cta"},
        # the kernel is timed inside a long run of steps under the power cap, so its
        # denominator is the measured sustained bf16 throughput; the burst figure is beside it
        "roofline": {"kernel": "fused forward GEMM (NF4 decode + X W'^T + P B^T)", "bound": "tensor",
                     "achieved": achieved, "peak": peak_fwd, "unit": "TFLOP/s",
                     "frac": achieved / peak_fwd, "traffic": fwd_main_traffic(),
                     "traffic_unit": "bytes per launch (ncu dram read + write)",
                     "peak_source": peak_fwd_source,
                     "frac_of_burst": achieved / peaks["bf16_tflops"],
                     "frac_of_datasheet_2250": achieved / 2250.0},
        "components": {
            "quantize_nf4_dq": {"ms": q_ms, "GB/s": n * NF4_DQ_BYTES_PER_PARAM / (q_ms * 1e-3) / 1e9,
                                "frac_hbm": n * NF4_DQ_BYTES_PER_PARAM / (q_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                "frac_8tbs": n * NF4_DQ_BYTES_PER_PARAM / (q_ms * 1e-3) / 1e9 / 8000.0},
            "forward": {"ms": fwd_ms, "TFLOP/s": fwd_f / (fwd_ms * 1e-3) / 1e12},
            "backward": {"ms": bwd_ms, "TFLOP/s": bwd_f / (bwd_ms * 1e-3) / 1e12},
            "fwd_main_gemm": {"ms": main_ms, "TFLOP/s": achieved},
            "bwd_dx_gemm": {"ms": dx_ms, "TFLOP/s": dx_flops / (dx_ms * 1e-3) / 1e12},
            "per_group_ms": {g: avg(g) for g in B.PROFILE_GROUPS if prof[g][1]},
            "decode_7b_4096x4096_nf4": decode,
            "lordba": lordba,
            "qwha": qwha,
            "optimizer_adamw_7b_r64": optim,
        },
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches,
        "clocks": clk,
        "cpu_baseline": cpu,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--gemm", choices=["pair", "single"], default="single",
                    help="fused weight GEMM on CTA pairs (cta_group::2) or on single CTAs")
    ap.add_argument("--part", choices=["all", "decode", "qwha", "optim"], default="all",
                    help="decode / qwha / optim: only that component (a short run for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    from quantized_base_rank_b200 import synth
    case = synth.CFG3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, case, world, rank)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if args.part == "decode":
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        out = decode_bench(dev, load_peaks(), reps=args.steps)
        if rank == 0:
            print(json.dumps({"part": "decode", "decode_7b_4096x4096_nf4": out}), flush=True)
        return
    if args.part == "optim":
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        out = optim_bench(dev, load_peaks(), reps=args.steps)
        if rank == 0:
            print(json.dumps({"part": "optim", "optimizer_adamw_7b_r64": out}), flush=True)
        return
    if args.part == "qwha":
        from quantized_base_rank_b200 import binding as B
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        inp = synth.make_inputs(dataclasses.replace(case, backward=False))
        qw = B.quantize_weight(inp["W"].to(dev), "nf4_dq")
        out = qwha_bench(dev, load_peaks(), qw, inp["X"].to(dev), reps=args.steps)
        if rank == 0:
            print(json.dumps({"part": "qwha", "qwha": out}), flush=True)
        return
    try:
        run_ours(args, case, world, rank, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
