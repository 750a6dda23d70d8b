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
FWD_MAIN_TRAFFIC = {"bytes": 112071168 + 149585664, "sources_sha256_16": "24736b26d741c823"}
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
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured",
                "sustained_sm_mhz": (d.get("clocks_under_load") or {}).get("sm_mhz_median")}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def linear_flops(M, N, K, r):
    fwd = 2 * M * N * K + 2 * M * K * r + 2 * M * N * r
    bwd = (2 * M * N * K + 2 * M * N * r + 2 * M * r * K) + 2 * M * r * K + 2 * M * N * r
    return fwd, bwd


class ClockSampler:
    """SM clock and throttle-reason samples taken while the timed region runs: a thread
    reads NVML every `period_s` (10 ms) from start() to stop(), so even a timed region of a
    few tens of milliseconds gets several samples. Read-only queries; nothing is set. Falls
    back to nvidia-smi at its shortest loop period if NVML cannot be loaded."""
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int, period_s: float = 0.01):
        import threading
        self.period = period_s
        self.samples = []                      # (sm_mhz, sm_max_mhz, reason bits, watts)
        self.err = None
        self._stop = threading.Event()
        self._thread = None
        self._nv = None
        self._smi = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
            self._h = nv.nvmlDeviceGetHandleByUUID(uuid.encode() if isinstance(uuid, str) else uuid)
            self._nv = nv
            self._bits = {"hw_slowdown": nv.nvmlClocksEventReasonHwSlowdown,
                          "hw_thermal_slowdown": nv.nvmlClocksEventReasonHwThermalSlowdown,
                          "sw_thermal_slowdown": nv.nvmlClocksEventReasonSwThermalSlowdown,
                          "sw_power_cap": nv.nvmlClocksEventReasonSwPowerCap}
            self._max = nv.nvmlDeviceGetMaxClockInfo(self._h, nv.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception as e:                   # no NVML: nvidia-smi at 100 ms
            self.err = f"nvml: {e}"
            q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
            try:
                self._smi = subprocess.Popen(
                    ["nvidia-smi", f"--query-gpu={q}", "--format=csv,noheader,nounits", "-lms", "100",
                     "-i", str(device_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except Exception:
                self._smi = None

    def _sample(self):
        nv = self._nv
        sm = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
        bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        try:
            w = nv.nvmlDeviceGetPowerUsage(self._h) / 1000.0
        except Exception:
            w = None
        self.samples.append((float(sm), float(self._max), int(bits), w))

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception as e:
                self.err = str(e)
                return
            self._stop.wait(self.period)

    def stop(self) -> dict:
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=5)
            try:
                self._sample()                   # one more at the end of the region
            except Exception:
                pass
            sm = [x[0] for x in self.samples]
            reasons = sorted({nm for x in self.samples for nm, b in self._bits.items() if x[2] & b})
            watts = [x[3] for x in self.samples if x[3] is not None]
            return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": float(self._max),
                    "sm_mhz_min": min(sm) if sm else None, "reasons": reasons, "samples": len(sm),
                    "period_ms": 1e3 * self.period, "power_w_max": max(watts) if watts else None,
                    "source": "nvml"}
        if self._smi is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no clock source"], "samples": 0}
        self._smi.terminate()
        try:
            out, _ = self._smi.communicate(timeout=5)
        except Exception:
            self._smi.kill()
            out, _ = self._smi.communicate()
        sm, smax, reasons = [], [], set()
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(self.NAMES, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": sorted(reasons),
                "samples": len(sm), "period_ms": 100.0, "source": "nvidia-smi"}


# cuBLAS's bf16 throughput per GHz of SM clock, from the sustained measurement (its median
# clock under load is recorded beside it); the per-clock comparison of a kernel timed at
# another clock
def cublas_tflops_per_ghz(peaks):
    if peaks.get("bf16_tflops_sustained") and peaks.get("sustained_sm_mhz"):
        return peaks["bf16_tflops_sustained"] / (peaks["sustained_sm_mhz"] / 1e3)
    return None


def pick_tensor_peak(peaks, timed_s: float, clk: dict | None):
    """The bf16 denominator that matches how the kernel was timed. The burst figure is
    cuBLAS timed alone, before the power cap pulls the clock down; the sustained one is
    cuBLAS held for seconds under the cap. A timed region shorter than a second, or one
    whose median SM clock stayed at the maximum with no power cap active, is a burst."""
    reasons = (clk or {}).get("reasons") or []
    sm, smax = (clk or {}).get("sm_mhz"), (clk or {}).get("sm_max_mhz")
    at_max = sm is not None and smax and sm >= 0.97 * smax and "sw_power_cap" not in reasons
    if timed_s < 1.0 or at_max or not peaks.get("bf16_tflops_sustained"):
        why = "timed region under 1 s" if timed_s < 1.0 else "SM clock at max, no power cap"
        if not peaks.get("bf16_tflops_sustained"):
            why = "no sustained figure"
        return peaks["bf16_tflops"], f"{peaks['source']} bf16 burst ({why}; {timed_s:.3f} s timed)"
    return (peaks["bf16_tflops_sustained"],
            f"{peaks['source']} bf16 sustained ({timed_s:.2f} s timed under the power cap)")


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


INT8_BYTES_PER_PARAM = 2.0 + 1.0 + 4.0 / 64                      # bf16 read + codes + fp32 absmax


def quant_outputs(fmt, n, dev):
    if fmt == "nf4_dq":
        nb = n // 64
        return (torch.empty(n // 2, dtype=torch.uint8, device=dev), torch.empty(nb, dtype=torch.float32, device=dev),
                torch.empty(nb, dtype=torch.int8, device=dev),
                torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev),
                torch.empty(1, dtype=torch.float32, device=dev))
    return (torch.empty(n, dtype=torch.int8, device=dev), torch.empty(n // 64, dtype=torch.float32, device=dev))


def quantize_into(fmt, W, outs):
    from quantized_base_rank_b200 import binding as B
    if fmt == "nf4_dq":
        B.nf4_dq_quantize(W, *outs)
    else:
        B.int8_quantize(W, *outs)


def as_weight(fmt, N, K, outs):
    from quantized_base_rank_b200 import binding as B
    if fmt == "nf4_dq":
        codes, _, qa, gs, mu = outs
        return B.QuantWeight(fmt, N, K, codes, None, qa, gs, mu)
    codes, absmax = outs
    return B.QuantWeight(fmt, N, K, codes, absmax)


def graph_us(fn, reps: int = 20) -> float:
    """Device time of one fn() call: reps calls captured in one CUDA graph and replayed, so
    the host's launch overhead is not in the figure."""
    for _ in range(3):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        with torch.cuda.graph(g, stream=st):
            for _ in range(reps):
                fn()
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    del g
    return e0.elapsed_time(e1) * 1e3 / reps


def quant_bench(dev, peaks, reps: int = 20, shapes=((4096, 4096), (11008, 4096), (22016, 8192))):
    """Quantise alone, device time per weight (CUDA-graph replay of back-to-back calls over
    three bf16 source copies, so each call reads its source from HBM): NF4 + double
    quantisation in one call, and blockwise int8, on the 7B-shaped 4096x4096 and 11008x4096
    weights and the 65B-shaped 22016x8192 one. GB/s of algorithmic bytes (2.516 and 3.0625
    B/param)."""
    from quantized_base_rank_b200 import synth
    out = {}
    for (N, K) in shapes:
        n = N * K
        Ws = [synth.device_normal_bf16((N, K), 0.02, 0, 400 + c, dev) for c in range(3)]
        i = [0]

        def nxt():
            i[0] += 1
            return Ws[i[0] % 3]

        for fmt, bpp in (("nf4_dq", NF4_DQ_BYTES_PER_PARAM), ("int8", INT8_BYTES_PER_PARAM)):
            outs = quant_outputs(fmt, n, dev)
            us = graph_us(lambda: quantize_into(fmt, nxt(), outs), reps)
            gbs = bpp * n / (us * 1e-6) / 1e9
            out[f"{N}x{K}_{fmt}"] = {"us": us, "GB/s": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
                                     "hbm_floor_us": bpp * n / (peaks["hbm_gbs"] * 1e3)}
            del outs
        del Ws
        torch.cuda.empty_cache()
    return out


def layer_bench(dev, peaks, N, K, M, r, fmt, reps: int = 5, seed: int = 0, idx: int = 0):
    """One quantised linear W [N, K] in format `fmt` at M tokens and rank r: the quantise
    (GB/s of algorithmic bytes; the bf16 source rotates over enough copies to exceed 3x
    L2, so it is read from HBM), then forward and backward, each kernel group timed by
    the library's event hooks over `reps` calls. Inputs are device Philox draws."""
    from quantized_base_rank_b200 import binding as B
    from quantized_base_rank_b200 import synth
    n = N * K
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    copies = min(4, max(1, int(np.ceil(3 * l2 / (2 * n)))))
    Ws = [synth.device_normal_bf16((N, K), 0.02, seed, idx + c, dev) for c in range(copies)]
    outs = quant_outputs(fmt, n, dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    qi = [0]

    def nxt():
        qi[0] += 1
        return Ws[qi[0] % copies]

    q_us = graph_us(lambda: quantize_into(fmt, nxt(), outs), max(4, reps * copies))
    bpp = NF4_DQ_BYTES_PER_PARAM if fmt == "nf4_dq" else INT8_BYTES_PER_PARAM
    q_gbs = bpp * n / (q_us * 1e-6) / 1e9
    del Ws
    qw = as_weight(fmt, N, K, outs)
    X = synth.device_normal_bf16((M, K), 1.0, seed, idx + 10, dev)
    A = synth.device_normal_bf16((r, K), 1.0 / K, seed, idx + 11, dev)
    Bm = synth.device_normal_bf16((N, r), 0.01, seed, idx + 12, dev)
    dY = synth.device_normal_bf16((M, N), 1.0, seed, idx + 13, dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    T = torch.empty((M, r), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    dA = torch.empty((r, K), dtype=torch.float32, device=dev)
    dB = torch.empty((N, r), dtype=torch.float32, device=dev)

    def fb():
        B.linear_fwd(qw, X, A, Bm, 16.0, Y=Y, T=T)
        B.linear_bwd(qw, X, dY, A, Bm, T, 16.0, dX=dX, dA=dA, dB=dB)

    for _ in range(3):
        fb()
    torch.cuda.synchronize()
    for g in B.PROFILE_GROUPS:
        B.profile_read(g)
    B.profile_enable(True)
    e0.record()
    for _ in range(reps):
        fb()
    e1.record()
    torch.cuda.synchronize()
    B.profile_enable(False)
    step_ms = e0.elapsed_time(e1) / reps
    prof = {g: B.profile_read(g) for g in B.PROFILE_GROUPS}
    avg = lambda g: prof[g][0] / prof[g][1] if prof[g][1] else 0.0
    fwd_f, bwd_f = linear_flops(M, N, K, r)
    fwd_ms = sum(avg(g) for g in ("fwd_prep", "fwd_xa", "fwd_main", "fwd_small"))
    bwd_ms = sum(avg(g) for g in ("bwd_prep", "bwd_dyb", "bwd_db", "bwd_da", "bwd_dx"))
    main_f, dx_f = 2 * M * N * (K + r), 2 * M * N * K + 2 * M * r * K
    tf = lambda f, ms: f / (ms * 1e-3) / 1e12 if ms > 0 else None
    burst = peaks["bf16_tflops"]
    assert B.device_status() == B.QL_OK
    return {"N": N, "K": K, "M": M, "r": r, "format": fmt,
            "quantize": {"us": q_us, "GB/s": q_gbs, "frac_hbm": q_gbs / peaks["hbm_gbs"],
                         "bytes_per_param": bpp, "source_copies": copies},
            "fwd_bwd_ms": step_ms, "TFLOP/s": tf(fwd_f + bwd_f, step_ms),
            "forward": {"ms": fwd_ms, "TFLOP/s": tf(fwd_f, fwd_ms)},
            "backward": {"ms": bwd_ms, "TFLOP/s": tf(bwd_f, bwd_ms)},
            "fwd_main_gemm": {"ms": avg("fwd_main"), "TFLOP/s": tf(main_f, avg("fwd_main")),
                              "frac_of_burst": tf(main_f, avg("fwd_main")) / burst},
            "bwd_dx_gemm": {"ms": avg("bwd_dx"), "TFLOP/s": tf(dx_f, avg("bwd_dx")),
                            "frac_of_burst": tf(dx_f, avg("bwd_dx")) / burst},
            "per_group_ms": {g: avg(g) for g in B.PROFILE_GROUPS if prof[g][1]}}


def layers_bench(dev, peaks, reps: int = 5):
    """The layers the step leaves out: the same up-projection in the int8 format, and the
    65B-shaped 22016x8192 (gate/up) and 8192x22016 (down) linears at 2048 tokens, in both
    formats, rank 64."""
    out = {"upproj_11008x4096_M8192_int8": layer_bench(dev, peaks, 11008, 4096, 8192, 64, "int8", reps,
                                                       idx=200)}
    for (N, K) in ((22016, 8192), (8192, 22016)):
        for fmt in ("nf4_dq", "int8"):
            out[f"llama65b_{N}x{K}_M2048_{fmt}"] = layer_bench(dev, peaks, N, K, 2048, 64, fmt, reps,
                                                               idx=300 + N % 97 + (fmt == "int8"))
            torch.cuda.empty_cache()
    return out


def stack_bench(dev, peaks, M: int = 4096, reps: int = 2):
    """The 32-layer 7B-shaped stack: every one of its 224 bf16 weights is drawn on the
    device (13 GB of sources), then (1) the whole stack is quantised to NF4+DQ by the batched
    entry, timed as one region (16.3 GB of algorithmic traffic), with one call per weight
    timed beside it, and (2) every linear runs its forward at M tokens with a rank-64
    adapter, timed as one region."""
    from quantized_base_rank_b200 import binding as B
    from quantized_base_rank_b200 import stack, synth
    specs = stack.stack_7b()
    srcs = [synth.device_normal_bf16((sp.N, sp.K), 0.02, 0, synth.stack_index(sp.layer, sp.which, synth.W_IDX),
                                     dev) for sp in specs]
    outs = [quant_outputs("nf4_dq", sp.N * sp.K, dev) for sp in specs]
    n_total = sum(sp.N * sp.K for sp in specs)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed_ms(fn):
        fn()
        torch.cuda.synchronize()
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    # the whole stack in one batched call (three launches per 128 weights), and, beside it,
    # one nf4_dq_quantize call per weight
    q_ms = timed_ms(lambda: B.nf4_dq_quantize_batch(srcs, outs))
    q_ms_each = timed_ms(lambda: [quantize_into("nf4_dq", Wc, o) for Wc, o in zip(srcs, outs)])
    q_gbs = NF4_DQ_BYTES_PER_PARAM * n_total / (q_ms * 1e-3) / 1e9
    del srcs
    torch.cuda.empty_cache()
    qws = [as_weight("nf4_dq", sp.N, sp.K, o) for sp, o in zip(specs, outs)]
    Xs = {K: synth.device_normal_bf16((M, K), 1.0, 0, 990 + K % 7, dev) for K in {sp.K for sp in specs}}
    Ys = {N: torch.empty((M, N), dtype=torch.bfloat16, device=dev) for N in {sp.N for sp in specs}}
    ads = [(synth.device_normal_bf16((sp.r, sp.K), 1.0 / sp.K, 0, synth.stack_index(sp.layer, sp.which, synth.A_IDX),
                                     dev),
            synth.device_normal_bf16((sp.N, sp.r), 0.01, 0, synth.stack_index(sp.layer, sp.which, synth.B_IDX), dev))
           for sp in specs]

    def fwd_all():
        for sp, qw, (A, Bm) in zip(specs, qws, ads):
            B.linear_fwd(qw, Xs[sp.K], A, Bm, sp.alpha, save_T=False, Y=Ys[sp.N])

    fwd_all()
    torch.cuda.synchronize()
    for g in B.PROFILE_GROUPS:
        B.profile_read(g)
    B.profile_enable(True)
    e0.record()
    for _ in range(reps):
        fwd_all()
    e1.record()
    torch.cuda.synchronize()
    B.profile_enable(False)
    f_ms = e0.elapsed_time(e1) / reps
    prof = {g: B.profile_read(g) for g in B.PROFILE_GROUPS}
    flops = sum(stack.linear_flops(sp, M)[0] for sp in specs)
    main_flops = sum(2 * M * sp.N * (sp.K + sp.r) for sp in specs)
    main_ms = prof["fwd_main"][0] / reps
    assert B.device_status() == B.QL_OK
    acct = stack.accounting(specs)
    return {"linears": len(specs), "params": n_total, "stored_bytes": acct["weight_bytes"],
            "bits_per_param": acct["bits_per_param"],
            "quantize_all": {"ms": q_ms, "GB/s": q_gbs, "frac_hbm": q_gbs / peaks["hbm_gbs"],
                             "algorithmic_bytes": NF4_DQ_BYTES_PER_PARAM * n_total, "call": "nf4_dq_quantize_batch",
                             "one_call_per_weight_ms": q_ms_each},
            "forward_all_M4096_r64": {"ms": f_ms, "TFLOP": flops / 1e12, "TFLOP/s": flops / (f_ms * 1e-3) / 1e12,
                                      "main_gemm_ms": main_ms,
                                      "main_gemm_TFLOP/s": main_flops / (main_ms * 1e-3) / 1e12,
                                      "main_gemm_frac_of_burst":
                                          main_flops / (main_ms * 1e-3) / 1e12 / peaks["bf16_tflops"]}}


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
    # the adapter gradients live in the data-parallel exchange's bucket (written in place)
    exchange = dp.BucketedGradExchange([(r, K, N)], device=dev) if dist is not None else None
    if exchange is not None:
        dA, dB = exchange.grads(0)
    else:
        dA = torch.empty((r, K), dtype=torch.float32, device=dev)
        dB = torch.empty((N, r), dtype=torch.float32, device=dev)

    def exchange_grads():
        if exchange is not None:
            exchange.ready(0)
            exchange.finish()

    def step():
        B.nf4_dq_quantize(W, codes, absmax, qa, gs, mu)
        B.linear_fwd(qw, X, A, Bm, case.alpha, Y=Y, T=T)
        B.linear_bwd(qw, X, dY, A, Bm, T, case.alpha, dX=dX, dA=dA, dB=dB)
        exchange_grads()

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
        exchange_grads()
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

    # ---- quantise alone, device time (CUDA graphs) ----
    quant = quant_bench(dev, peaks)

    # ---- the int8 format and the 65B-shaped layers; the whole 7B stack ----
    layers = layers_bench(dev, peaks) if not args.skip_extra else None
    torch.cuda.empty_cache()
    stack7b = stack_bench(dev, peaks) if not args.skip_extra else None
    torch.cuda.empty_cache()

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
    timed_s = ms * args.steps / 1e3
    peak_fwd, peak_fwd_source = pick_tensor_peak(peaks, timed_s, clk)
    per_ghz = cublas = None
    if clk and clk.get("sm_mhz"):
        per_ghz = achieved / (clk["sm_mhz"] / 1e3)
        cublas = cublas_tflops_per_ghz(peaks)
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": case.name, "M": M, "N": N, "K": K, "r": r, "alpha": case.alpha,
                   "format": "nf4_dq", "step": "quantise(NF4+DQ) + fwd + bwd(dX,dA,dB)",
                   "l2": "inputs larger than L2 (X 64 MB, W 90 MB, dY 180 MB > 126 MB)",
                   "parallelism": f"dp{world}" if world > 1 else "single",
                   "fused_gemm": "cta_pair" if args.gemm == "pair" else "single_cta"},
        # the denominator follows the timed region: the burst figure for a short region at
        # full clock, the sustained one for seconds under the power cap; both are beside it,
        # with the per-clock comparison against cuBLAS
        "roofline": {"kernel": "fused forward GEMM (NF4 decode + X W'^T + P B^T)", "bound": "tensor",
                     "achieved": achieved, "peak": peak_fwd, "unit": "TFLOP/s",
                     "frac": achieved / peak_fwd, "traffic": fwd_main_traffic(),
                     "traffic_unit": "bytes per launch (ncu dram read + write)",
                     "algorithmic_flops_per_launch": main_flops,
                     "peak_source": peak_fwd_source,
                     "frac_of_burst": achieved / peaks["bf16_tflops"],
                     "frac_of_sustained": (achieved / peaks["bf16_tflops_sustained"]
                                           if peaks.get("bf16_tflops_sustained") else None),
                     "frac_of_datasheet_2250": achieved / 2250.0,
                     "tflops_per_ghz": per_ghz, "cublas_tflops_per_ghz": cublas,
                     "per_clock_frac_of_cublas": per_ghz / cublas if per_ghz and cublas else None},
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
            "quantize_alone": quant,
            "layers": layers,
            "stack_7b_32x7": stack7b,
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
    ap.add_argument("--part", choices=["all", "decode", "qwha", "optim", "layers", "stack", "quantize"],
                    default="all", help="decode / qwha / optim / layers / stack / quantize: only that "
                                        "component (a short run for profiling)")
    ap.add_argument("--shape", default=None, help="NxK: the one weight shape of --part quantize")
    ap.add_argument("--skip-extra", action="store_true",
                    help="leave out the int8, 65B-shaped and whole-stack components")
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
    if args.part in ("layers", "stack", "quantize"):
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        fn = {"layers": layers_bench, "stack": stack_bench, "quantize": quant_bench}[args.part]
        kw = {}
        if args.part == "quantize" and args.shape:
            kw["shapes"] = (tuple(int(v) for v in args.shape.lower().split("x")),)
        out = fn(dev, load_peaks(), reps=max(1, args.steps), **kw)
        if rank == 0:
            print(json.dumps({"part": args.part, args.part: out}), flush=True)
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
