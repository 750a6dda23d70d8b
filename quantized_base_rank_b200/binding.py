"""ctypes binding of libqlora_b200.so: the C entry points under the same names, with
torch tensors marshalled to device pointers. No computation happens here; every step
of the path runs in the library's CUDA kernels. The library must be built
(``python -m quantized_base_rank_b200.build``); loading fails loudly otherwise.
"""
from __future__ import annotations

import ctypes
import os
import re
import threading

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqlora_b200.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "qlora.h")

QL_OK, QL_ERR_INVALID_ARG, QL_ERR_UNSUPPORTED, QL_ERR_WORKSPACE, QL_ERR_NONFINITE, \
    QL_ERR_TIMEOUT, QL_ERR_CUDA = range(7)
QL_FMT_NF4_DQ, QL_FMT_INT8_B64 = 0, 1
QL_OP_DQ, QL_OP_FWD, QL_OP_BWD, QL_OP_FWD_LORDBA, QL_OP_FWD_QWHA, QL_OP_DQ_BATCH = 0, 1, 2, 3, 4, 5
FORMATS = {"nf4_dq": QL_FMT_NF4_DQ, "int8": QL_FMT_INT8_B64}


class QLError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


class QLWeight(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("codes", ctypes.c_void_p), ("absmax", ctypes.c_void_p),
                ("qabsmax", ctypes.c_void_p), ("group_scale", ctypes.c_void_p),
                ("mean", ctypes.c_void_p)]


class QLNf4DqItem(ctypes.Structure):
    """ql_nf4_dq_item: one weight of nf4_dq_quantize_batch."""
    _fields_ = [("W", ctypes.c_void_p), ("n", ctypes.c_int64), ("codes", ctypes.c_void_p),
                ("absmax", ctypes.c_void_p), ("qabsmax", ctypes.c_void_p), ("group_scale", ctypes.c_void_p),
                ("mean", ctypes.c_void_p)]


class QLQwha(ctypes.Structure):
    """ql_qwha: the sparse coefficients of a Walsh-Hadamard adapter in compressed rows."""
    _fields_ = [("row_ptr", ctypes.c_void_p), ("col", ctypes.c_void_p), ("c", ctypes.c_void_p),
                ("nnz", ctypes.c_int64)]


class QLLordba(ctypes.Structure):
    """ql_lordba: packed sign carriers and fp16 channel scales of a LoRDBA adapter."""
    _fields_ = [("R", ctypes.c_int32), ("ell", ctypes.c_int32), ("B1", ctypes.c_void_p),
                ("B2", ctypes.c_void_p), ("alpha", ctypes.c_void_p), ("beta", ctypes.c_void_p),
                ("gamma", ctypes.c_void_p)]


class QLAdamw(ctypes.Structure):
    """ql_adamw: the hyperparameters of one AdamW step."""
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float), ("grad_scale", ctypes.c_float),
                ("step", ctypes.c_int64)]


class QLLion(ctypes.Structure):
    """ql_lion: the hyperparameters of one Lion step."""
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("weight_decay", ctypes.c_float)]


_lib = None
_lock = threading.Lock()
P, I64, I32, F32, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
_SIGS = {
    "nf4_quantize": ([P, I64, P, P, P], I32),
    "int8_quantize": ([P, I64, P, P, P], I32),
    "dq_quantize": ([P, I64, P, P, P, P, SZ, P], I32),
    "nf4_dq_quantize": ([P, I64, P, P, P, P, P, P, SZ, P], I32),
    "nf4_dq_quantize_batch": ([P, I32, P, SZ, P], I32),
    "nf4_quantize_shard": ([P, I64, P, P, P, P, SZ, P], I32),
    "qlora_linear_fwd_lordba": ([ctypes.POINTER(QLWeight), P, I64, ctypes.c_void_p, P, P, SZ, P], I32),
    "qlora_linear_fwd_qwha": ([ctypes.POINTER(QLWeight), P, I64, ctypes.c_void_p, P, P, SZ, P], I32),
    "ql_wht": ([P, I64, I64, P, P], I32),
    "ql_adamw_step": ([P, P, P, P, P, I64, ctypes.c_void_p, P], I32),
    "ql_lion_int8_step": ([P, P, P, P, P, I64, ctypes.c_void_p, P], I32),
    "ql_paged_alloc": ([SZ, ctypes.POINTER(ctypes.c_void_p)], I32),
    "ql_paged_free": ([ctypes.c_void_p], I32),
    "ql_paged_prefetch": ([ctypes.c_void_p, SZ, I32, P], I32),
    "dq_quantize_shard": ([P, I64, P, I64, P, P, P, P], I32),
    "ql_dequantize": ([ctypes.POINTER(QLWeight), P, P], I32),
    "qlora_linear_fwd": ([ctypes.POINTER(QLWeight), P, I64, P, P, I32, F32, P, P, P, SZ, P], I32),
    "qlora_linear_bwd": ([ctypes.POINTER(QLWeight), P, P, I64, P, P, P, I32, F32, P, P, P, P, SZ, P], I32),
    "ql_workspace_bytes": ([I32, I64, I64, I64, I32], SZ),
    "ql_get_device_status": ([P], I32),
    "ql_status_string": ([I32], ctypes.c_char_p),
    "ql_nf4_codebook": ([ctypes.POINTER(ctypes.c_float)], None),
    "ql_set_wait_timeout_ns": ([ctypes.c_uint64], None),
    "ql_set_gemm_pair": ([ctypes.c_int], None),
    "ql_profile_enable": ([ctypes.c_int], None),
    "ql_profile_read": ([ctypes.c_int, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64)], ctypes.c_int),
    "ql_launch_count": ([], ctypes.c_uint64),
    "qlora_linear_fwd_static": ([ctypes.POINTER(QLWeight), P, I64, P, P, I32, F32, P, P, P], I32),
}

# kernel groups of ql_profile_read
PROFILE_GROUPS = ["nf4", "dq", "int8", "dequant", "fwd_prep", "fwd_xa", "fwd_main", "bwd_prep",
                  "bwd_dyb", "bwd_db", "bwd_da", "bwd_dx", "fwd_small", "fwd_adapter", "optim"]


def lib() -> ctypes.CDLL:
    """Load the shared library (once). Raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m quantized_base_rank_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            for name, (args, res) in _SIGS.items():
                f = getattr(L, name)
                f.argtypes = args
                f.restype = res
            _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/qlora.h declares."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s+([A-Za-z_][A-Za-z0-9_]*)\s*\(",
                      src, flags=re.M)


def status_string(s: int) -> str:
    return lib().ql_status_string(int(s)).decode()


def _check(status: int, where: str):
    if status != QL_OK:
        raise QLError(status, where)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(device: torch.device | None = None) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _is_cuda(t: torch.Tensor) -> bool:
    return t.is_cuda


def _need(t: torch.Tensor, dtype: torch.dtype, name: str, shape=None, device=None):
    """Refuse, before the library is called, what its kernels would read or write out of
    bounds: t must be a contiguous CUDA tensor of `dtype`; with `shape`, of exactly that
    shape (an int: that many elements, any shape); with `device`, on that device. The C
    entry points take bare pointers and cannot see a buffer's size."""
    if not isinstance(t, torch.Tensor) or t.dtype != dtype or not _is_cuda(t) or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA {dtype} tensor")
    if shape is not None:
        ok = t.numel() == shape if isinstance(shape, int) else tuple(t.shape) == tuple(shape)
        if not ok:
            raise ValueError(f"{name} has shape {tuple(t.shape)}; expected {shape}")
    if device is not None and t.device != torch.device(device):
        raise ValueError(f"{name} is on {t.device}; expected {device}")


# ---- workspace: caller-owned device memory, allocated by torch, reused ----------------
_ws = {}


def workspace(nbytes: int, device: torch.device) -> torch.Tensor:
    key = (device.index, torch.cuda.current_stream(device).cuda_stream)
    buf = _ws.get(key)
    if buf is None or buf.numel() < nbytes:
        buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
        _ws[key] = buf
    return buf


def workspace_bytes(op: int, M: int, N: int, K: int, r: int) -> int:
    return int(lib().ql_workspace_bytes(op, M, N, K, r))


def _need_dq_outputs(nb: int, qabsmax, group_scale, mean, dev):
    _need(qabsmax, torch.int8, "qabsmax", nb, dev)
    _need(group_scale, torch.float32, "group_scale", (nb + 255) // 256, dev)
    _need(mean, torch.float32, "mean", 1, dev)


def _need_weight(qw: "QuantWeight", K: int, dev):
    if qw.K != K:
        raise ValueError(f"X has {K} columns; the weight has K = {qw.K}")
    if qw.device != dev:
        raise ValueError(f"the weight is on {qw.device}; X is on {dev}")


# ---- entry points ---------------------------------------------------------------------

def nf4_quantize(W: torch.Tensor, codes: torch.Tensor | None = None,
                 absmax: torch.Tensor | None = None):
    _need(W, torch.bfloat16, "W")
    n = W.numel()
    if codes is None:
        codes = torch.empty((n + 1) // 2, dtype=torch.uint8, device=W.device)
    if absmax is None:
        absmax = torch.empty((n + 63) // 64, dtype=torch.float32, device=W.device)
    _need(codes, torch.uint8, "codes", (n + 1) // 2, W.device)
    _need(absmax, torch.float32, "absmax", (n + 63) // 64, W.device)
    _check(lib().nf4_quantize(_ptr(W), n, _ptr(codes), _ptr(absmax), _stream(W.device)),
           "nf4_quantize")
    return codes, absmax


def int8_quantize(W: torch.Tensor, codes: torch.Tensor | None = None,
                  absmax: torch.Tensor | None = None):
    _need(W, torch.bfloat16, "W")
    n = W.numel()
    if codes is None:
        codes = torch.empty(n, dtype=torch.int8, device=W.device)
    if absmax is None:
        absmax = torch.empty((n + 63) // 64, dtype=torch.float32, device=W.device)
    _need(codes, torch.int8, "codes", n, W.device)
    _need(absmax, torch.float32, "absmax", (n + 63) // 64, W.device)
    _check(lib().int8_quantize(_ptr(W), n, _ptr(codes), _ptr(absmax), _stream(W.device)),
           "int8_quantize")
    return codes, absmax


def dq_quantize(absmax: torch.Tensor, qabsmax=None, group_scale=None, mean=None):
    _need(absmax, torch.float32, "absmax")
    nb = absmax.numel()
    dev = absmax.device
    if qabsmax is None:
        qabsmax = torch.empty(nb, dtype=torch.int8, device=dev)
    if group_scale is None:
        group_scale = torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev)
    if mean is None:
        mean = torch.empty(1, dtype=torch.float32, device=dev)
    _need_dq_outputs(nb, qabsmax, group_scale, mean, dev)
    nws = workspace_bytes(QL_OP_DQ, 0, 0, 0, 0)
    ws = workspace(nws, dev)
    _check(lib().dq_quantize(_ptr(absmax), nb, _ptr(qabsmax), _ptr(group_scale), _ptr(mean),
                             _ptr(ws), ws.numel(), _stream(dev)), "dq_quantize")
    return qabsmax, group_scale, mean


def nf4_dq_quantize(W: torch.Tensor, codes=None, absmax=None, qabsmax=None, group_scale=None,
                    mean=None):
    """NF4 + double quantisation in one call; same results as nf4_quantize then dq_quantize."""
    _need(W, torch.bfloat16, "W")
    n = W.numel()
    dev = W.device
    nb = (n + 63) // 64
    if codes is None:
        codes = torch.empty((n + 1) // 2, dtype=torch.uint8, device=dev)
    if absmax is None:
        absmax = torch.empty(nb, dtype=torch.float32, device=dev)
    if qabsmax is None:
        qabsmax = torch.empty(nb, dtype=torch.int8, device=dev)
    if group_scale is None:
        group_scale = torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev)
    if mean is None:
        mean = torch.empty(1, dtype=torch.float32, device=dev)
    _need(codes, torch.uint8, "codes", (n + 1) // 2, dev)
    _need(absmax, torch.float32, "absmax", nb, dev)
    _need_dq_outputs(nb, qabsmax, group_scale, mean, dev)
    ws = workspace(workspace_bytes(QL_OP_DQ, 0, 0, 0, 0), dev)
    _check(lib().nf4_dq_quantize(_ptr(W), n, _ptr(codes), _ptr(absmax), _ptr(qabsmax), _ptr(group_scale),
                                 _ptr(mean), _ptr(ws), ws.numel(), _stream(dev)), "nf4_dq_quantize")
    return codes, absmax, qabsmax, group_scale, mean


def nf4_dq_quantize_batch(Ws, outs=None):
    """NF4 + double quantisation of several weights in one call (four launches per 128
    weights). Ws: list of bf16 tensors on one device. outs: optional list of (codes,
    absmax, qabsmax, group_scale, mean) per weight. Returns that list; each entry equals
    nf4_dq_quantize of its weight bit for bit."""
    if not Ws:
        return []
    dev = Ws[0].device
    if outs is None:
        outs = []
        for W in Ws:
            n = W.numel()
            nb = (n + 63) // 64
            outs.append((torch.empty((n + 1) // 2, dtype=torch.uint8, device=dev),
                         torch.empty(nb, dtype=torch.float32, device=dev),
                         torch.empty(nb, dtype=torch.int8, device=dev),
                         torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev),
                         torch.empty(1, dtype=torch.float32, device=dev)))
    if len(outs) != len(Ws):
        raise ValueError("one output tuple per weight")
    items = (QLNf4DqItem * len(Ws))()
    for i, (W, (codes, absmax, qa, gs, mu)) in enumerate(zip(Ws, outs)):
        _need(W, torch.bfloat16, f"W[{i}]", None, dev)
        n = W.numel()
        nb = (n + 63) // 64
        _need(codes, torch.uint8, f"codes[{i}]", (n + 1) // 2, dev)
        _need(absmax, torch.float32, f"absmax[{i}]", nb, dev)
        _need_dq_outputs(nb, qa, gs, mu, dev)
        items[i] = QLNf4DqItem(_ptr(W), n, _ptr(codes), _ptr(absmax), _ptr(qa), _ptr(gs), _ptr(mu))
    ws = workspace(workspace_bytes(QL_OP_DQ_BATCH, len(Ws), 0, 0, 0), dev)
    _check(lib().nf4_dq_quantize_batch(items, len(Ws), _ptr(ws), ws.numel(), _stream(dev)),
           "nf4_dq_quantize_batch")
    return outs


def nf4_quantize_shard(W: torch.Tensor, codes=None, absmax=None, bins=None):
    """Step 1 of the sharded NF4 + double quantisation: codes, absmax and the shard's exact
    DQ bins (int64 [16] holding the unsigned 64-bit sums, each below 2^63)."""
    _need(W, torch.bfloat16, "W")
    n = W.numel()
    dev = W.device
    if codes is None:
        codes = torch.empty((n + 1) // 2, dtype=torch.uint8, device=dev)
    if absmax is None:
        absmax = torch.empty((n + 63) // 64, dtype=torch.float32, device=dev)
    if bins is None:
        bins = torch.empty(16, dtype=torch.int64, device=dev)
    _need(codes, torch.uint8, "codes", (n + 1) // 2, dev)
    _need(absmax, torch.float32, "absmax", (n + 63) // 64, dev)
    _need(bins, torch.int64, "bins", 16, dev)
    ws = workspace(workspace_bytes(QL_OP_DQ, 0, 0, 0, 0), dev)
    _check(lib().nf4_quantize_shard(_ptr(W), n, _ptr(codes), _ptr(absmax), _ptr(bins), _ptr(ws),
                                    ws.numel(), _stream(dev)), "nf4_quantize_shard")
    return codes, absmax, bins


def dq_quantize_shard(absmax: torch.Tensor, bins: torch.Tensor, nblocks_total: int, qabsmax=None,
                      group_scale=None, mean=None):
    """Step 3: the mean from bins summed over all shards, then this shard's groups."""
    _need(absmax, torch.float32, "absmax")
    nb = absmax.numel()
    dev = absmax.device
    _need(bins, torch.int64, "bins", 16, dev)
    if qabsmax is None:
        qabsmax = torch.empty(nb, dtype=torch.int8, device=dev)
    if group_scale is None:
        group_scale = torch.empty((nb + 255) // 256, dtype=torch.float32, device=dev)
    if mean is None:
        mean = torch.empty(1, dtype=torch.float32, device=dev)
    _need_dq_outputs(nb, qabsmax, group_scale, mean, dev)
    _check(lib().dq_quantize_shard(_ptr(absmax), nb, _ptr(bins), int(nblocks_total), _ptr(qabsmax),
                                   _ptr(group_scale), _ptr(mean), _stream(dev)), "dq_quantize_shard")
    return qabsmax, group_scale, mean


def pack_signs(S: torch.Tensor) -> torch.Tensor:
    """Pack a +-1 matrix [rows, cols] 1 bit per entry, the ql_lordba carrier layout:
    bit j%32 of word j/32 of a row is 1 for +1. Returns int32 [rows, ceil(cols/32)]."""
    rows, cols = S.shape
    words = (cols + 31) // 32
    bits = torch.zeros((rows, words * 32), dtype=torch.int64, device=S.device)
    bits[:, :cols] = (S > 0).to(torch.int64)
    shifts = torch.arange(32, device=S.device, dtype=torch.int64)
    packed = (bits.view(rows, words, 32) << shifts).sum(dim=2)
    packed = torch.where(packed >= 2 ** 31, packed - 2 ** 32, packed)
    return packed.to(torch.int32).contiguous()


def linear_fwd_lordba(qw: "QuantWeight", X: torch.Tensor, B1p: torch.Tensor, B2p: torch.Tensor,
                      alpha: torch.Tensor, beta: torch.Tensor, gamma: torch.Tensor, R: int,
                      Y: torch.Tensor | None = None) -> torch.Tensor:
    """Y = X W'^T + X Delta W^T with the LoRDBA adapter given by packed carriers B1p
    [N, ceil(R/32)], B2p [R, ceil(K/32)] (int32 words) and fp16 scales alpha [ell, N],
    beta [ell, R], gamma [ell, K]."""
    _need(X, torch.bfloat16, "X")
    for t, nm in ((alpha, "alpha"), (beta, "beta"), (gamma, "gamma")):
        _need(t, torch.float16, nm)
    for t, nm in ((B1p, "B1"), (B2p, "B2")):
        _need(t, torch.int32, nm)
    M, K = X.shape
    ell = alpha.shape[0]
    dev = X.device
    N = qw.N
    _need_weight(qw, K, dev)
    _need(B1p, torch.int32, "B1", (N, (R + 31) // 32), dev)
    _need(B2p, torch.int32, "B2", (R, (K + 31) // 32), dev)
    _need(alpha, torch.float16, "alpha", (ell, N), dev)
    _need(beta, torch.float16, "beta", (ell, R), dev)
    _need(gamma, torch.float16, "gamma", (ell, K), dev)
    if Y is None:
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    _need(Y, torch.bfloat16, "Y", (M, N), dev)
    ad = QLLordba(R, ell, _ptr(B1p), _ptr(B2p), _ptr(alpha), _ptr(beta), _ptr(gamma))
    ws = workspace(workspace_bytes(QL_OP_FWD_LORDBA, M, qw.N, K, R * ell), dev)
    _check(lib().qlora_linear_fwd_lordba(ctypes.byref(qw.desc), _ptr(X), M, ctypes.addressof(ad), _ptr(Y),
                                         _ptr(ws), ws.numel(), _stream(dev)), "qlora_linear_fwd_lordba")
    return Y


def linear_fwd_qwha(qw: "QuantWeight", X: torch.Tensor, row_ptr: torch.Tensor, col: torch.Tensor,
                    c: torch.Tensor, Y: torch.Tensor | None = None) -> torch.Tensor:
    """Y = X W'^T + X (F H^{-1})^T with the Walsh-Hadamard adapter F given in compressed
    rows: row_ptr int32 [N+1], col uint16 [nnz], c bf16 [nnz]."""
    _need(X, torch.bfloat16, "X")
    _need(row_ptr, torch.int32, "row_ptr")
    _need(col, torch.uint16, "col")
    _need(c, torch.bfloat16, "c")
    M, K = X.shape
    dev = X.device
    nnz = c.numel()
    _need_weight(qw, K, dev)
    _need(row_ptr, torch.int32, "row_ptr", qw.N + 1, dev)
    _need(col, torch.uint16, "col", nnz, dev)
    _need(c, torch.bfloat16, "c", nnz, dev)
    if Y is None:
        Y = torch.empty((M, qw.N), dtype=torch.bfloat16, device=dev)
    _need(Y, torch.bfloat16, "Y", (M, qw.N), dev)
    ad = QLQwha(_ptr(row_ptr), _ptr(col) if nnz else None, _ptr(c) if nnz else None, nnz)
    ws = workspace(workspace_bytes(QL_OP_FWD_QWHA, M, qw.N, K, 0), dev)
    _check(lib().qlora_linear_fwd_qwha(ctypes.byref(qw.desc), _ptr(X), M, ctypes.addressof(ad), _ptr(Y),
                                       _ptr(ws), ws.numel(), _stream(dev)), "qlora_linear_fwd_qwha")
    return Y


def wht(X: torch.Tensor, Z: torch.Tensor | None = None) -> torch.Tensor:
    """Z = X H^{-T}: the orthonormal (blockwise) Walsh-Hadamard transform of each row."""
    _need(X, torch.bfloat16, "X")
    M, K = X.shape
    if Z is None:
        Z = torch.empty_like(X)
    _need(Z, torch.bfloat16, "Z", (M, K), X.device)
    _check(lib().ql_wht(_ptr(X), M, K, _ptr(Z), _stream(X.device)), "ql_wht")
    return Z


def adamw_step(theta: torch.Tensor, param: torch.Tensor, grad: torch.Tensor, m: torch.Tensor,
               v: torch.Tensor, step: int, lr: float, beta1: float = 0.9, beta2: float = 0.999,
               eps: float = 1e-8, weight_decay: float = 0.0, grad_scale: float = 1.0):
    """One AdamW step over flat adapter parameters: theta, grad, m, v fp32 [n] (theta the
    trained copy), param bf16 [n] (rewritten as bf16(theta)). Tensors may be views of a
    PagedBuffer."""
    n = theta.numel()
    for t, nm in ((theta, "theta"), (grad, "grad"), (m, "m"), (v, "v")):
        _need(t, torch.float32, nm, n, theta.device)
    _need(param, torch.bfloat16, "param", n, theta.device)
    h = QLAdamw(lr, beta1, beta2, eps, weight_decay, grad_scale, step)
    _check(lib().ql_adamw_step(_ptr(theta), _ptr(param), _ptr(grad), _ptr(m), _ptr(v), n, ctypes.addressof(h),
                               _stream(theta.device)), "ql_adamw_step")


def lion_int8_step(theta: torch.Tensor, param: torch.Tensor, grad: torch.Tensor, m_codes: torch.Tensor,
                   m_absmax: torch.Tensor, lr: float, beta1: float = 0.9, beta2: float = 0.99,
                   weight_decay: float = 0.0):
    """One Lion step with INT8 momentum: theta, grad fp32 [n]; m_codes int8 [n] and m_absmax
    fp32 [ceil(n/64)] updated in place; param bf16 [n] rewritten as bf16(theta)."""
    n = theta.numel()
    dev = theta.device
    for t, nm in ((theta, "theta"), (grad, "grad")):
        _need(t, torch.float32, nm, n, dev)
    _need(param, torch.bfloat16, "param", n, dev)
    _need(m_codes, torch.int8, "m_codes", n, dev)
    _need(m_absmax, torch.float32, "m_absmax", (n + 63) // 64, dev)
    h = QLLion(lr, beta1, beta2, weight_decay)
    _check(lib().ql_lion_int8_step(_ptr(theta), _ptr(param), _ptr(grad), _ptr(m_codes), _ptr(m_absmax), n,
                                   ctypes.addressof(h), _stream(theta.device)), "ql_lion_int8_step")


class _CudaArray:
    """A CUDA Array Interface view of memory the library owns (torch.as_tensor reads it
    without a copy)."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr, "data": (ptr, False),
                                         "version": 3, "strides": None, "stream": None}


class PagedBuffer:
    """Paged (CUDA managed) memory from ql_paged_alloc, for optimiser states: the driver
    moves its pages between device and host memory on demand; prefetch() moves them
    explicitly. float32 views are plain CUDA tensors over the same memory, valid while the
    buffer is alive."""

    _TYPES = {torch.float32: ("<f4", 4), torch.int8: ("|i1", 1), torch.int32: ("<i4", 4)}

    def __init__(self, nbytes: int):
        self.nbytes = int(nbytes)
        p = ctypes.c_void_p()
        _check(lib().ql_paged_alloc(self.nbytes, ctypes.byref(p)), "ql_paged_alloc")
        self.ptr = p.value or 0

    def view(self, dtype: torch.dtype, numel: int, offset_bytes: int = 0) -> torch.Tensor:
        code, size = self._TYPES[dtype]
        if offset_bytes < 0 or offset_bytes % size or offset_bytes + numel * size > self.nbytes:
            raise ValueError("view outside the buffer")
        return torch.as_tensor(_CudaArray(self.ptr + offset_bytes, (numel,), code), device="cuda")

    def prefetch(self, to_host: bool, stream_device: torch.device | None = None, offset_bytes: int = 0,
                 nbytes: int | None = None):
        n = self.nbytes - offset_bytes if nbytes is None else nbytes
        _check(lib().ql_paged_prefetch(self.ptr + offset_bytes, n, 1 if to_host else 0, _stream(stream_device)),
               "ql_paged_prefetch")

    def host_array(self, dtype=np.float32, numel: int | None = None, offset_bytes: int = 0) -> np.ndarray:
        """The same memory read from the host (unified memory): a numpy view, valid after
        the stream that wrote it has been synchronised."""
        item = np.dtype(dtype).itemsize
        n = (self.nbytes - offset_bytes) // item if numel is None else numel
        buf = (ctypes.c_char * (n * item)).from_address(self.ptr + offset_bytes)
        return np.frombuffer(buf, dtype=dtype, count=n)

    def free(self):
        if self.ptr:
            _check(lib().ql_paged_free(self.ptr), "ql_paged_free")
            self.ptr = 0

    def __del__(self):
        try:
            self.free()
        except Exception:
            pass


class QuantWeight:
    """A quantised weight W [N, K] held in device tensors, plus its ABI descriptor."""

    def __init__(self, fmt: str, N: int, K: int, codes, absmax=None, qabsmax=None,
                 group_scale=None, mean=None):
        self.fmt, self.N, self.K = fmt, N, K
        self.codes, self.absmax = codes, absmax
        self.qabsmax, self.group_scale, self.mean = qabsmax, group_scale, mean
        self.desc = QLWeight(FORMATS[fmt], 0, N, K, _ptr(codes), _ptr(absmax), _ptr(qabsmax),
                             _ptr(group_scale), _ptr(mean))

    @property
    def device(self):
        return self.codes.device

    def nbytes(self) -> int:
        ts = [self.codes, self.qabsmax, self.group_scale, self.mean] if self.fmt == "nf4_dq" \
            else [self.codes, self.absmax]
        return sum(t.numel() * t.element_size() for t in ts)


def quantize_weight(W: torch.Tensor, fmt: str = "nf4_dq", keep_absmax: bool = False) -> QuantWeight:
    """Quantise a bf16 [N, K] weight: NF4 + double quantisation, or blockwise int8."""
    N, K = W.shape
    if fmt == "nf4_dq":
        codes, absmax, qa, gs, mu = nf4_dq_quantize(W)
        return QuantWeight(fmt, N, K, codes, absmax if keep_absmax else None, qa, gs, mu)
    if fmt == "int8":
        codes, absmax = int8_quantize(W)
        return QuantWeight(fmt, N, K, codes, absmax)
    raise ValueError(fmt)


def dequantize(qw: QuantWeight) -> torch.Tensor:
    out = torch.empty((qw.N, qw.K), dtype=torch.bfloat16, device=qw.device)
    _check(lib().ql_dequantize(ctypes.byref(qw.desc), _ptr(out), _stream(qw.device)),
           "ql_dequantize")
    return out


def linear_fwd(qw: QuantWeight, X: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
               alpha: float, save_T: bool = True, Y: torch.Tensor | None = None,
               T: torch.Tensor | None = None):
    """Y = X W'^T + (alpha/r) (X A^T) B^T. Returns (Y, T) with T = bf16(X A^T) or None."""
    for t, nm in ((X, "X"), (A, "A"), (B, "B")):
        _need(t, torch.bfloat16, nm)
    M, K = X.shape
    r = A.shape[0]
    dev = X.device
    _need_weight(qw, K, dev)
    _need(A, torch.bfloat16, "A", (r, K), dev)
    _need(B, torch.bfloat16, "B", (qw.N, r), dev)
    if Y is None:
        Y = torch.empty((M, qw.N), dtype=torch.bfloat16, device=dev)
    if T is None and save_T:
        T = torch.empty((M, r), dtype=torch.bfloat16, device=dev)
    _need(Y, torch.bfloat16, "Y", (M, qw.N), dev)
    if T is not None:
        _need(T, torch.bfloat16, "T", (M, r), dev)
    ws = workspace(workspace_bytes(QL_OP_FWD, M, qw.N, K, r), dev)
    _check(lib().qlora_linear_fwd(ctypes.byref(qw.desc), _ptr(X), M, _ptr(A), _ptr(B), r,
                                  float(alpha), _ptr(Y), _ptr(T), _ptr(ws), ws.numel(),
                                  _stream(dev)), "qlora_linear_fwd")
    return Y, T


def linear_bwd(qw: QuantWeight, X, dY, A, B, T, alpha: float, dX=None, dA=None, dB=None):
    """Returns (dX bf16 [M,K], dA fp32 [r,K], dB fp32 [N,r])."""
    for t, nm in ((X, "X"), (dY, "dY"), (A, "A"), (B, "B"), (T, "T")):
        _need(t, torch.bfloat16, nm)
    M, K = X.shape
    r = A.shape[0]
    dev = X.device
    N = qw.N
    _need_weight(qw, K, dev)
    for t, nm, shape in ((dY, "dY", (M, N)), (A, "A", (r, K)), (B, "B", (N, r)), (T, "T", (M, r))):
        _need(t, torch.bfloat16, nm, shape, dev)
    if dX is None:
        dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    if dA is None:
        dA = torch.empty((r, K), dtype=torch.float32, device=dev)
    if dB is None:
        dB = torch.empty((N, r), dtype=torch.float32, device=dev)
    _need(dX, torch.bfloat16, "dX", (M, K), dev)
    _need(dA, torch.float32, "dA", (r, K), dev)
    _need(dB, torch.float32, "dB", (N, r), dev)
    ws = workspace(workspace_bytes(QL_OP_BWD, M, qw.N, K, r), dev)
    _check(lib().qlora_linear_bwd(ctypes.byref(qw.desc), _ptr(X), _ptr(dY), M, _ptr(A), _ptr(B),
                                  _ptr(T), r, float(alpha), _ptr(dX), _ptr(dA), _ptr(dB),
                                  _ptr(ws), ws.numel(), _stream(dev)), "qlora_linear_bwd")
    return dX, dA, dB


def device_status(device: torch.device | None = None) -> int:
    """Synchronise and return (and clear) the library's sticky device flag."""
    return int(lib().ql_get_device_status(_stream(device)))


def profile_enable(on: bool = True):
    lib().ql_profile_enable(1 if on else 0)


def profile_read(group: str):
    """(total milliseconds, launches) of one kernel group since the last read."""
    ms = ctypes.c_double(0.0)
    cnt = ctypes.c_int64(0)
    lib().ql_profile_read(PROFILE_GROUPS.index(group), ctypes.byref(ms), ctypes.byref(cnt))
    return ms.value, cnt.value


def launch_count() -> int:
    return int(lib().ql_launch_count())


def nf4_codebook() -> list[float]:
    buf = (ctypes.c_float * 16)()
    lib().ql_nf4_codebook(buf)
    return list(buf)
