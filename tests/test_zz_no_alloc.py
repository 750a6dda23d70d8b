"""The forward entry point that allocates nothing (qlora_linear_fwd_static).

It is for callers that cannot allocate device memory where they run the layer, such as
a plugin whose host framework owns every allocation or a loop that must not touch the
allocator.
It keeps its scratch in one fixed array inside the library. This file is collected last
so that a failure here comes after every other test has run. Each call goes straight
through the C ABI and is compared with the workspace-taking qlora_linear_fwd, on two
calls in a row that share the fixed array, within the tolerance the other tests use."""
import ctypes

import numpy as np
import pytest
import torch

from quantized_base_rank_b200 import binding as B
from quantized_base_rank_b200 import synth

pytestmark = pytest.mark.gpu


def _static_fwd(qw, X, A, Bm, alpha):
    M, r = X.shape[0], A.shape[0]
    Y = torch.empty((M, qw.N), dtype=torch.bfloat16, device=X.device)
    T = torch.empty((M, r), dtype=torch.bfloat16, device=X.device)
    st = B.lib().qlora_linear_fwd_static(ctypes.byref(qw.desc), X.data_ptr(), M, A.data_ptr(),
                                         Bm.data_ptr(), r, float(alpha), Y.data_ptr(), T.data_ptr(),
                                         torch.cuda.current_stream().cuda_stream)
    assert st == B.QL_OK, B.status_string(st)
    return Y, T


def _close(got, ref):
    got = got.float().cpu().numpy().astype(np.float64)
    ref = ref.float().cpu().numpy().astype(np.float64)
    err = got - ref
    assert np.linalg.norm(err) <= 5e-3 * np.linalg.norm(ref)
    assert np.max(np.abs(err)) <= 1e-2 * np.max(np.abs(ref))


def test_static_scratch_forward_matches_workspace_forward_twice():
    cases = [synth.CFG1,
             synth.LinearCase("no-alloc-300x1024x768", N=1024, K=768, M=300, r=64, alpha=16.0, seed=4)]
    for case in cases:                       # two calls in a row through the shared array
        inp = synth.make_inputs(case)
        qw = B.quantize_weight(inp["W"].cuda(), case.fmt)
        X, A, Bm = inp["X"].cuda(), inp["A"].cuda(), inp["B"].cuda()
        Y_ref, T_ref = B.linear_fwd(qw, X, A, Bm, case.alpha)
        Y, T = _static_fwd(qw, X, A, Bm, case.alpha)
        torch.cuda.synchronize()
        assert B.device_status() == B.QL_OK
        _close(Y, Y_ref)
        _close(T, T_ref)


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
