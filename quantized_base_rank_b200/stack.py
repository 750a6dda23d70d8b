"""A stack of quantised linears with a per-layer choice of weight format and adapter rank,
and the memory accounting of the stored formats.

AutoQRA page (gist.science/ko/paper/2602.22268), section 3.1: every layer l of the frozen
backbone gets its own bit-width q_l and adapter rank r_l. Here q_l is NF4 with double
quantisation (QLoRA page, aizip.shop/methodologies/qlora, sections "1. 4-bit NormalFloat
(NF4)" and "2. Double Quantization") or blockwise int8, and r_l is one of {8, 16, 32, 64}.
One decoder layer's seven linears share the layer's choice. The stack is a list of
independent linears: each call goes through the library's C ABI (binding.py), and nothing
here computes the method.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import binding as bd
from . import synth

FORMATS = ("nf4_dq", "int8")
BLOCK = 64          # elements per quantisation block
GROUP = 256         # blocks per double-quantisation group


@dataclass(frozen=True)
class LinearSpec:
    """One linear of a stack: weight [N, K] in format `fmt`, adapter rank `r`."""
    layer: int
    which: int      # position in the decoder layer's list of linears
    name: str
    N: int
    K: int
    fmt: str
    r: int
    alpha: float

    @property
    def params(self) -> int:
        return self.N * self.K


def _layer(layer: int, shapes, fmt: str, r: int, alpha: float):
    return [LinearSpec(layer, i, name, N, K, fmt, r, alpha) for i, (name, N, K) in enumerate(shapes)]


def stack_7b(n_layers: int = 32, r: int = 64, alpha: float = 16.0) -> list[LinearSpec]:
    """The 7B-shaped stack: 32 decoder layers of q, k, v, o (4096x4096), gate, up
    (11008x4096) and down (4096x11008), all NF4 + double quantisation at rank r."""
    return [s for l in range(n_layers) for s in _layer(l, synth.STACK_7B, "nf4_dq", r, alpha)]


def stack_65b_mix(n_layers: int = 80, alpha: float = 16.0, seed: int = 0) -> list[LinearSpec]:
    """The 65B-shaped stack with a per-layer (format, rank) drawn by synth.layer_mix_65b."""
    mix = synth.layer_mix_65b(n_layers, seed)
    return [s for l, (fmt, r) in enumerate(mix) for s in _layer(l, synth.STACK_65B, fmt, r, alpha)]


def weight_bytes(fmt: str, n: int) -> int:
    """Stored bytes of one weight of n parameters (n/64 blocks rounded up). NF4 + DQ:
    n/2 bytes of codes, one int8 constant per block, one fp32 scale per group of 256
    blocks and one fp32 mean. int8: n bytes of codes and one fp32 absmax per block."""
    nb = -(-n // BLOCK)
    if fmt == "nf4_dq":
        return -(-n // 2) + nb + 4 * -(-nb // GROUP) + 4
    if fmt == "int8":
        return n + 4 * nb
    raise ValueError(fmt)


def adapter_bytes(spec: LinearSpec) -> int:
    """bf16 A [r, K] and B [N, r]."""
    return 2 * spec.r * (spec.K + spec.N)


def accounting(specs) -> dict:
    """Parameters, stored weight bytes, bits per parameter and adapter bytes of a stack."""
    params = sum(s.params for s in specs)
    wbytes = sum(weight_bytes(s.fmt, s.params) for s in specs)
    by_fmt = {f: sum(weight_bytes(s.fmt, s.params) for s in specs if s.fmt == f) for f in FORMATS}
    return {"linears": len(specs), "params": params, "weight_bytes": wbytes,
            "bits_per_param": 8.0 * wbytes / params, "weight_bytes_by_format": by_fmt,
            "adapter_bytes": sum(adapter_bytes(s) for s in specs)}


def linear_flops(spec: LinearSpec, M: int) -> tuple[int, int]:
    """(forward, backward) flops of one call with M tokens; dequantisation not counted."""
    N, K, r = spec.N, spec.K, spec.r
    fwd = 2 * M * N * K + 2 * M * K * r + 2 * M * N * r
    bwd = (2 * M * N * K + 2 * M * N * r + 2 * M * r * K) + 2 * M * r * K + 2 * M * N * r
    return fwd, bwd


class QuantizedLinear:
    """One linear of the stack on the device: the quantised weight in the spec's format
    (the dispatch of the per-layer choice) and the bf16 adapter A, B."""

    def __init__(self, spec: LinearSpec, W: torch.Tensor, A: torch.Tensor, B: torch.Tensor):
        if tuple(W.shape) != (spec.N, spec.K):
            raise ValueError(f"weight shape {tuple(W.shape)} is not {(spec.N, spec.K)}")
        if tuple(A.shape) != (spec.r, spec.K) or tuple(B.shape) != (spec.N, spec.r):
            raise ValueError("adapter shapes do not match the spec")
        self.spec = spec
        self.qw = bd.quantize_weight(W, spec.fmt)
        self.A, self.B = A, B

    def stored_bytes(self) -> int:
        return self.qw.nbytes()

    def forward(self, X: torch.Tensor, save_T: bool = True):
        """(Y, T): Y = X W'^T + (alpha/r) (X A^T) B^T, T = bf16(X A^T) for the backward."""
        return bd.linear_fwd(self.qw, X, self.A, self.B, self.spec.alpha, save_T=save_T)

    def backward(self, X: torch.Tensor, dY: torch.Tensor, T: torch.Tensor):
        """(dX, dA, dB) with the quantised weight frozen."""
        return bd.linear_bwd(self.qw, X, dY, self.A, self.B, T, self.spec.alpha)
