"""GPU: the decode-shaped forward of several linears sharing X in one launch
(qlora_linear_fwd_group). Every output must equal the single-linear call on the same X bit
for bit (the same per-cluster arithmetic and reduction order), and one group is checked
against the fp64 oracle within the forward's tolerance."""
import numpy as np
import pytest
import torch

import oracle.qlora_oracle as o
from quantized_base_rank_b200 import binding as B
from quantized_base_rank_b200 import synth

pytestmark = pytest.mark.gpu


def _linears(specs, K, fmt, seed):
    out = []
    for i, (N, r) in enumerate(specs):
        W = synth.normal_bf16((N, K), 0.02, seed + i, 0).cuda()
        qw = B.quantize_weight(W, fmt)
        A = synth.normal_bf16((r, K), 0.02, seed + i, 1).cuda() if r else None
        Bm = synth.normal_bf16((N, r), 0.02, seed + i, 2).cuda() if r else None
        out.append((qw, A, Bm, 2.0 * r if r else 0.0, W))
    return out


@pytest.mark.parametrize("fmt", ["nf4_dq", "int8"])
@pytest.mark.parametrize("M,K,specs", [
    (1, 4096, [(4096, 16), (1024, 16), (1024, 16)]),    # a 7B-style query, key, value with GQA widths
    (5, 704, [(136, 8), (264, 0), (128, 24)]),          # ragged rows, a base-only member, mixed ranks
    (16, 1024, [(512, 64), (256, 32)]),                 # sixteen tokens, rank tiles of four and two
    (3, 2048, [(384, 16)] * 8),                         # the largest group
])
def test_group_equals_single_calls(M, K, specs, fmt):
    lins = _linears(specs, K, fmt, 11 + M)
    X = synth.normal_bf16((M, K), 1.0, 5, M).cuda()
    Ys = B.linear_fwd_group([(qw, A, Bm, al) for (qw, A, Bm, al, _) in lins], X)
    torch.cuda.synchronize()
    assert B.device_status() == B.QL_OK
    for (qw, A, Bm, al, _), Yg in zip(lins, Ys):
        if A is None:
            ref = B.linear_fwd_group([(qw, None, None, 0.0)], X)[0]
        else:
            ref, _ = B.linear_fwd(qw, X, A, Bm, al, save_T=False)
        torch.cuda.synchronize()
        assert torch.equal(Yg, ref)


def test_group_against_oracle():
    """Query, key and value of a small layer against the fp64 oracle on the same
    dequantised weights: relative Frobenius <= 5e-3, elementwise <= 1e-2 * max|ref|."""
    M, K = 4, 512
    lins = _linears([(256, 16), (128, 8), (128, 0)], K, "nf4_dq", 3)
    X = synth.normal_bf16((M, K), 1.0, 6, 0).cuda()
    Ys = B.linear_fwd_group([(qw, A, Bm, al) for (qw, A, Bm, al, _) in lins], X)
    torch.cuda.synchronize()
    Xn = X.float().cpu().numpy().astype(np.float64)
    for (qw, A, Bm, al, W), Yg in zip(lins, Ys):
        N = W.shape[0]
        wd = o.quantize_weight(W.float().cpu().numpy(), "nf4_dq")["wdeq"].reshape(N, K).astype(np.float64)
        ref = Xn @ wd.T
        if A is not None:
            r = A.shape[0]
            ref = ref + (al / r) * (Xn @ A.float().cpu().numpy().astype(np.float64).T) @ \
                Bm.float().cpu().numpy().astype(np.float64).T
        got = Yg.float().cpu().numpy().astype(np.float64)
        err = got - ref
        assert np.linalg.norm(err) / np.linalg.norm(ref) <= 5e-3
        assert np.max(np.abs(err)) <= 1e-2 * np.max(np.abs(ref))
