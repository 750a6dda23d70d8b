"""Seeded synthetic inputs for the quantised linear layer.

This module only draws random tensors with the shapes and distributions of the
workloads below; it holds none of the method's arithmetic. Both the test suite's
CPU oracle and the CUDA path take their inputs from here.

Conventions:
* ``N(0, s)`` names the standard deviation s.
* Every tensor has its own stream, seeded ``seed * 1000 + index`` in the order
  W, outlier positions/signs, X, A, B, dY.
* Values are drawn in fp32 and rounded to bf16 (nearest-even); the bf16 bit
  patterns are what both sides consume.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

W_IDX, OUTLIER_IDX, X_IDX, A_IDX, B_IDX, DY_IDX = range(6)


def _rng(seed: int, idx: int) -> np.random.Generator:
    return np.random.default_rng(seed * 1000 + idx)


def to_bf16(x: np.ndarray) -> torch.Tensor:
    """fp32 numpy -> bf16 torch CPU tensor (round to nearest even)."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)


def normal_bf16(shape, std: float, seed: int, idx: int) -> torch.Tensor:
    x = _rng(seed, idx).standard_normal(size=shape, dtype=np.float32) * np.float32(std)
    return to_bf16(x)


def weight_with_outliers(N: int, K: int, std: float, frac: float, mult: float,
                         seed: int) -> torch.Tensor:
    """W ~ N(0, std) with round(frac * N * K) positions, drawn without replacement,
    set to +-mult*std (random sign)."""
    w = _rng(seed, W_IDX).standard_normal(size=(N, K), dtype=np.float32) * np.float32(std)
    n_out = int(round(frac * N * K))
    if n_out:
        g = _rng(seed, OUTLIER_IDX)
        pos = g.choice(N * K, size=n_out, replace=False)
        sign = np.where(g.integers(0, 2, size=n_out) == 1, 1.0, -1.0).astype(np.float32)
        w.reshape(-1)[pos] = sign * np.float32(mult * std)
    return to_bf16(w)


@dataclasses.dataclass(frozen=True)
class LinearCase:
    """One quantised linear: weight [N, K], tokens M, rank r, alpha, format."""
    name: str
    N: int
    K: int
    M: int
    r: int
    alpha: float
    fmt: str = "nf4_dq"          # "nf4_dq" or "int8"
    w_std: float = 0.02
    outlier_frac: float = 0.0
    outlier_mult: float = 20.0
    a_std: float | None = None   # None -> 1/K
    b_std: float = 0.01
    backward: bool = True
    seed: int = 0

    @property
    def s(self) -> float:
        return self.alpha / self.r


def make_inputs(case: LinearCase) -> dict:
    """All bf16 CPU tensors of one case: W, X, A, B and (if backward) dY."""
    seed = case.seed
    W = weight_with_outliers(case.N, case.K, case.w_std, case.outlier_frac,
                             case.outlier_mult, seed)
    X = normal_bf16((case.M, case.K), 1.0, seed, X_IDX)
    a_std = case.a_std if case.a_std is not None else 1.0 / case.K
    A = normal_bf16((case.r, case.K), a_std, seed, A_IDX)
    B = normal_bf16((case.N, case.r), case.b_std, seed, B_IDX)
    out = {"W": W, "X": X, "A": A, "B": B}
    if case.backward:
        out["dY"] = normal_bf16((case.M, case.N), 1.0, seed, DY_IDX)
    return out


def device_normal_bf16(shape, std: float, seed: int, idx: int,
                       device="cuda") -> torch.Tensor:
    """Large tensors drawn on the device with torch's Philox generator (for the
    multi-layer stacks, whose bf16 sources are too big to draw on the host)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000 + idx)
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    return (x * std).to(torch.bfloat16)


# The five workloads: a single small linear, a decode-shaped 7B linear, a
# fine-tune-shaped MLP up-projection, a 32-layer 7B-shaped stack and 80 layers of
# 65B-shaped linears with a per-layer (format, rank) mix.
CFG1 = LinearCase("single-256", N=256, K=256, M=64, r=8, alpha=16.0, a_std=1.0 / 256)
CFG2 = [LinearCase(f"decode-7b-M{m}", N=4096, K=4096, M=m, r=16, alpha=32.0,
                   outlier_frac=0.001, outlier_mult=20.0, backward=False)
        for m in (1, 4, 16)]
CFG3 = LinearCase("upproj-11008x4096-M8192", N=11008, K=4096, M=8192, r=64, alpha=16.0)

STACK_7B = [("q", 4096, 4096), ("k", 4096, 4096), ("v", 4096, 4096), ("o", 4096, 4096),
            ("gate", 11008, 4096), ("up", 11008, 4096), ("down", 4096, 11008)]
STACK_65B = [("q", 8192, 8192), ("k", 8192, 8192), ("v", 8192, 8192), ("o", 8192, 8192),
             ("gate", 22016, 8192), ("up", 22016, 8192), ("down", 8192, 22016)]


def layer_mix_65b(n_layers: int = 80, seed: int = 0):
    """Per decoder layer: (format, rank) drawn uniformly from {nf4_dq, int8} x
    {8, 16, 32, 64} by a seed-0 generator, shared by the layer's 7 linears."""
    g = np.random.default_rng(seed * 1000 + 900)
    fmts = g.integers(0, 2, size=n_layers)
    ranks = g.integers(0, 4, size=n_layers)
    return [("nf4_dq" if f == 0 else "int8", (8, 16, 32, 64)[r]) for f, r in zip(fmts, ranks)]


def stack_index(layer: int, which: int, slot: int) -> int:
    """Sub-stream of tensor `slot` (W_IDX, X_IDX, A_IDX, B_IDX or DY_IDX) of linear `which`
    of decoder layer `layer` in a multi-layer stack."""
    return 100000 + (layer * 8 + which) * 8 + slot


def stack_linear_inputs(layer: int, which: int, N: int, K: int, M: int, r: int, seed: int = 0,
                        device="cuda", backward: bool = True) -> dict:
    """Device bf16 tensors of one linear of a stack: W ~ N(0, 0.02) [N, K], X ~ N(0, 1)
    [M, K], A ~ N(0, 1/K) [r, K], B ~ N(0, 0.01) [N, r] and dY ~ N(0, 1) [M, N], each from
    its own Philox sub-stream."""
    idx = lambda slot: stack_index(layer, which, slot)
    out = {"W": device_normal_bf16((N, K), 0.02, seed, idx(W_IDX), device),
           "X": device_normal_bf16((M, K), 1.0, seed, idx(X_IDX), device),
           "A": device_normal_bf16((r, K), 1.0 / K, seed, idx(A_IDX), device),
           "B": device_normal_bf16((N, r), 0.01, seed, idx(B_IDX), device)}
    if backward:
        out["dY"] = device_normal_bf16((M, N), 1.0, seed, idx(DY_IDX), device)
    return out


def lordba_inputs(N: int, K: int, R: int, ell: int, seed: int = 0) -> dict:
    """A LoRDBA adapter for a weight [N, K]: sign carriers B1 [N, R], B2 [R, K] (+-1,
    fp32) and fp16 channel scales alpha [ell, N] ~ U(0.5, 1) * 0.02 / sqrt(R),
    beta [ell, R] ~ U(0.5, 1), gamma [ell, K] ~ U(0.5, 1), so that the branch is of the
    same order as a N(0, 0.02) weight."""
    g = _rng(seed, 40)
    B1 = np.where(g.random((N, R)) < 0.5, -1.0, 1.0).astype(np.float32)
    B2 = np.where(g.random((R, K)) < 0.5, -1.0, 1.0).astype(np.float32)
    alpha = (g.uniform(0.5, 1.0, (ell, N)) * 0.02 / np.sqrt(R)).astype(np.float16)
    beta = g.uniform(0.5, 1.0, (ell, R)).astype(np.float16)
    gamma = g.uniform(0.5, 1.0, (ell, K)).astype(np.float16)
    return {"B1": torch.from_numpy(B1), "B2": torch.from_numpy(B2), "alpha": torch.from_numpy(alpha),
            "beta": torch.from_numpy(beta), "gamma": torch.from_numpy(gamma)}


def qwha_inputs(N: int, K: int, r_equiv: int, seed: int = 0, c_std: float = 0.02) -> dict:
    """A Walsh-Hadamard adapter for a weight [N, K] in compressed-row form.

    Budget: p = r_equiv * (N + K) coefficients, the trainable-parameter count of a rank
    r_equiv LoRA adapter on the same weight. Per-row counts: a floor of max(1, p / (4N))
    per output channel, the rest spread in proportion to a log-normal(0, 1) channel weight
    (a heavy-tailed stand-in for a per-channel error magnitude), each capped at K.
    Positions: distinct columns drawn uniformly per row, sorted ascending. Values:
    c ~ N(0, c_std) rounded to bf16.

    Returns row_ptr (int32 [N+1]), col (uint16 [nnz]), c (bf16 [nnz]) as CPU tensors."""
    assert 1 <= K <= 65536 and N >= 1
    g = _rng(seed, 50)
    p = min(r_equiv * (N + K), N * K)
    floor = max(1, p // (4 * N))
    w = g.lognormal(0.0, 1.0, N)
    extra = max(p - floor * N, 0)
    share = extra * w / w.sum()
    cnt = floor + np.floor(share).astype(np.int64)
    short = p - int(cnt.sum())
    if short > 0:                                   # largest remainders take the rest
        order = np.argsort(-(share - np.floor(share)), kind="stable")
        cnt[order[:short]] += 1
    cnt = np.minimum(cnt, K)
    row_ptr = np.zeros(N + 1, np.int64)
    row_ptr[1:] = np.cumsum(cnt)
    col = np.empty(int(row_ptr[-1]), np.uint16)
    for n in range(N):
        col[row_ptr[n]:row_ptr[n + 1]] = np.sort(g.choice(K, int(cnt[n]), replace=False))
    c = g.standard_normal(int(row_ptr[-1]), dtype=np.float32) * np.float32(c_std)
    return {"row_ptr": torch.from_numpy(row_ptr.astype(np.int32)), "col": torch.from_numpy(col),
            "c": to_bf16(c)}
