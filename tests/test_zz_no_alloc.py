"""The forward entry point that allocates nothing (qlora_linear_fwd_static).

It is for callers that cannot allocate device memory where they run the layer, such as
a plugin whose host framework owns every allocation or a loop that must not touch the
allocator. It keeps its scratch in one fixed array inside the library. This file is
collected last so that a failure here comes after every other test has run.

Each call goes straight through the C ABI and is compared with the workspace-taking
qlora_linear_fwd. Both run the same kernels on the same inputs, so the outputs must be
identical bit for bit (a stale or aliased scratch region would show up as a difference).
The larger shape runs first, so the small one that follows reads scratch that a bigger
call has already filled, and the small one runs twice in a row through the shared array.
"""
import ctypes
import os

import pytest
import torch

from quantized_base_rank_b200 import binding as B
from quantized_base_rank_b200 import build as build_mod
from quantized_base_rank_b200 import synth


def _static_fwd(qw, X, A, Bm, alpha):
    M, r = X.shape[0], A.shape[0]
    Y = torch.full((M, qw.N), float("nan"), dtype=torch.bfloat16, device=X.device)
    T = torch.full((M, r), float("nan"), dtype=torch.bfloat16, device=X.device)
    st = B.lib().qlora_linear_fwd_static(ctypes.byref(qw.desc), X.data_ptr(), M, A.data_ptr(),
                                         Bm.data_ptr(), r, float(alpha), Y.data_ptr(), T.data_ptr(),
                                         torch.cuda.current_stream().cuda_stream)
    assert st == B.QL_OK, B.status_string(st)
    return Y, T


def _prepare(case):
    inp = synth.make_inputs(case)
    qw = B.quantize_weight(inp["W"].cuda(), case.fmt)
    return qw, inp["X"].cuda(), inp["A"].cuda(), inp["B"].cuda()


@pytest.mark.gpu
def test_static_scratch_forward_equals_workspace_forward():
    big = synth.LinearCase("no-alloc-300x1024x768", N=1024, K=768, M=300, r=64, alpha=16.0, seed=4)
    small = synth.CFG1
    qb = _prepare(big)
    qs = _prepare(small)
    # the big shape first: it fills more of the shared array than the small one uses
    Yb, Tb = _static_fwd(*qb, big.alpha)
    Ys1, Ts1 = _static_fwd(*qs, small.alpha)
    Ys2, Ts2 = _static_fwd(*qs, small.alpha)       # a second call in a row on the same array
    Yb_ref, Tb_ref = B.linear_fwd(*qb, big.alpha)
    Ys_ref, Ts_ref = B.linear_fwd(*qs, small.alpha)
    torch.cuda.synchronize()
    assert B.device_status() == B.QL_OK
    for got, ref in ((Yb, Yb_ref), (Tb, Tb_ref), (Ys1, Ys_ref), (Ts1, Ts_ref), (Ys2, Ys_ref), (Ts2, Ts_ref)):
        assert torch.equal(got, ref)


@pytest.mark.gpu
def test_static_scratch_decode_shaped_call():
    """A decode-shaped call (one token) takes the path that needs no scratch."""
    case = synth.LinearCase("no-alloc-decode", N=1024, K=768, M=1, r=16, alpha=32.0, seed=5)
    assert B.workspace_bytes(B.QL_OP_FWD, case.M, case.N, case.K, case.r) == 0
    q = _prepare(case)
    Y, T = _static_fwd(*q, case.alpha)
    Y2, T2 = _static_fwd(*q, case.alpha)
    Y_ref, T_ref = B.linear_fwd(*q, case.alpha)
    torch.cuda.synchronize()
    assert B.device_status() == B.QL_OK
    assert torch.equal(Y, Y_ref) and torch.equal(T, T_ref)
    assert torch.equal(Y2, Y_ref) and torch.equal(T2, T_ref)


@pytest.mark.gpu
def test_static_scratch_refuses_oversize_shapes():
    case = synth.LinearCase("too-big", N=8192, K=4096, M=16384, r=256, alpha=16.0)
    need = B.workspace_bytes(B.QL_OP_FWD, case.M, case.N, case.K, case.r)
    assert need > 8 << 20
    n = case.N * case.K
    w = B.QuantWeight("nf4_dq", case.N, case.K,
                      torch.zeros(n // 2, dtype=torch.uint8, device="cuda"), None,
                      torch.zeros(n // 64, dtype=torch.int8, device="cuda"),
                      torch.zeros(n // 64 // 256, dtype=torch.float32, device="cuda"),
                      torch.zeros(1, dtype=torch.float32, device="cuda"))
    st = B.lib().qlora_linear_fwd_static(ctypes.byref(w.desc), 16, case.M, 16, 16, case.r, 16.0,
                                         16, None, None)
    assert st == B.QL_ERR_WORKSPACE


def test_static_scratch_status_matches_workspace_entry_without_a_device():
    """Shapes that the workspace entry refuses as unsupported get the same status here,
    before the scratch-size limit is looked at (no CUDA call is made)."""
    if not os.path.exists(B.LIB_PATH):
        build_mod.build()
    lib = B.lib()
    w = B.QLWeight(0, 0, 4096, 4096, 16, 0, 16, 16, 16)
    for M, r in (((1 << 31) + 1, 16), (64, 257)):
        a = lib.qlora_linear_fwd(ctypes.byref(w), 16, M, 16, 16, r, 16.0, 16, None, 16, 1 << 40, None)
        b = lib.qlora_linear_fwd_static(ctypes.byref(w), 16, M, 16, 16, r, 16.0, 16, None, None)
        assert a == b == B.QL_ERR_UNSUPPORTED
    # a null or misaligned operand: the same refusal from both
    for X in (None, 18):
        a = lib.qlora_linear_fwd(ctypes.byref(w), X, 64, 16, 16, 16, 16.0, 16, None, 256, 1 << 40, None)
        b = lib.qlora_linear_fwd_static(ctypes.byref(w), X, 64, 16, 16, 16, 16.0, 16, None, None)
        assert a == b == B.QL_ERR_INVALID_ARG
