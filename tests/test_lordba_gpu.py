"""GPU vs oracle: the quantised linear with a LoRDBA double-binary adapter branch
(LoRDBA page, gist.science/ko/paper/2605.24058, section "2. Methodology"), on the
large-M fused path and the decode-shaped path, both base formats, 1 to 3 envelope
terms. Tolerance as for the dense adapter: relative Frobenius <= 5e-3 and elementwise
<= 1e-2 * max|ref| against the fp64 oracle on the same dequantised weight."""
import numpy as np
import pytest
import torch

import oracle.qlora_oracle as o
from quantized_base_rank_b200 import binding as B
from quantized_base_rank_b200 import synth

pytestmark = pytest.mark.gpu


def _close(got, ref, what):
    got = np.asarray(got, np.float64)
    err = got - ref
    rel = np.linalg.norm(err) / np.linalg.norm(ref)
    elem = np.max(np.abs(err)) / np.max(np.abs(ref))
    assert np.all(np.isfinite(got)) and rel <= 5e-3 and elem <= 1e-2, f"{what}: {rel:.3e} {elem:.3e}"


def _run(M, N, K, R, ell, fmt, zero_w=False, seed=1):
    case = synth.LinearCase(f"lordba-{M}-{N}-{K}", N=N, K=K, M=M, r=8, alpha=8.0, fmt=fmt, seed=seed,
                            backward=False)
    inp = synth.make_inputs(case)
    W = torch.zeros_like(inp["W"]) if zero_w else inp["W"]
    ad = synth.lordba_inputs(N, K, R, ell, seed)
    qw = B.quantize_weight(W.cuda(), fmt)
    Y = B.linear_fwd_lordba(qw, inp["X"].cuda(), B.pack_signs(ad["B1"].cuda()), B.pack_signs(ad["B2"].cuda()),
                            ad["alpha"].cuda(), ad["beta"].cuda(), ad["gamma"].cuda(), R)
    torch.cuda.synchronize()
    assert B.device_status() == B.QL_OK
    wd = o.quantize_weight(W.float().numpy(), fmt)["wdeq"].reshape(N, K)
    ref = o.lordba_linear_fwd(inp["X"].float().numpy(), wd, ad["alpha"].numpy(), ad["beta"].numpy(),
                              ad["gamma"].numpy(), ad["B1"].numpy(), ad["B2"].numpy())
    _close(Y.float().cpu().numpy(), ref, f"Y M={M} R={R} ell={ell} {fmt}")


@pytest.mark.parametrize("fmt", ["nf4_dq", "int8"])
@pytest.mark.parametrize("M,N,K,R,ell", [(64, 256, 256, 16, 1), (300, 392, 512, 20, 2), (130, 256, 1344, 33, 3),
                                         (1, 4096, 4096, 16, 1), (5, 136, 704, 8, 3), (16, 512, 1024, 64, 1)])
def test_lordba_forward(M, N, K, R, ell, fmt):
    _run(M, N, K, R, ell, fmt)


@pytest.mark.parametrize("M", [64, 3])
def test_lordba_branch_alone(M):
    """W = 0: Y is the double-binary branch alone."""
    _run(M, 256, 512, 16, 2, "nf4_dq", zero_w=True)


def test_pack_signs_layout():
    S = torch.tensor([[1.0] * 31 + [-1.0] + [1.0, -1.0, 1.0]], device="cuda")
    w = B.pack_signs(S).cpu().numpy().view(np.uint32)
    assert w.shape == (1, 2)
    assert w[0, 0] == 0x7FFFFFFF and w[0, 1] == 0b101
