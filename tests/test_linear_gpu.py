"""GPU vs oracle for the quantised linear with an unmerged adapter: Y, T, dX, dA, dB.

Tolerance (fp32 accumulation, bf16 outputs): relative Frobenius error <= 5e-3 and
elementwise |err| <= 1e-2 * max|ref| against the fp64 oracle on the same dequantised
weight. The dequantised weight itself is bit-exact (tests/test_quant_gpu.py)."""
import numpy as np
import pytest
import torch

import oracle.qlora_oracle as o
from quantized_base_rank_b200 import binding as B
from quantized_base_rank_b200 import synth

pytestmark = pytest.mark.gpu

REL_FRO = 5e-3
REL_ELEM = 1e-2


def close(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), what
    err = got - ref
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(err) / nref
    elem = np.max(np.abs(err)) / np.max(np.abs(ref))
    assert rel <= REL_FRO and elem <= REL_ELEM, f"{what}: rel_fro={rel:.3e} rel_elem={elem:.3e}"
    return rel, elem


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def run_gpu(case, inp):
    qw = B.quantize_weight(inp["W"].cuda(), case.fmt)
    X, A, Bm = inp["X"].cuda(), inp["A"].cuda(), inp["B"].cuda()
    Y, T = B.linear_fwd(qw, X, A, Bm, case.alpha)
    out = {"Y": Y, "T": T}
    if case.backward:
        dX, dA, dB = B.linear_bwd(qw, X, inp["dY"].cuda(), A, Bm, T, case.alpha)
        out.update(dX=dX, dA=dA, dB=dB)
    torch.cuda.synchronize()
    assert B.device_status() == B.QL_OK
    return out


def run_oracle(case, inp, rows=None):
    wd = o.quantize_weight(inp["W"].float().numpy(), case.fmt)["wdeq"].reshape(case.N, case.K)
    X = f64(inp["X"])
    A, Bm = f64(inp["A"]), f64(inp["B"])
    Y, T = o.linear_fwd(X if rows is None else X[rows], wd, A, Bm, case.alpha, case.r)
    out = {"Y": Y, "T": T}
    if case.backward:
        dY = f64(inp["dY"])
        dXf, dA, dB = o.linear_bwd(X, dY, wd, A, Bm, case.alpha, case.r)
        out.update(dX=dXf if rows is None else dXf[rows], dA=dA, dB=dB)
    return out


def check_case(case, inp=None):
    inp = inp or synth.make_inputs(case)
    g = run_gpu(case, inp)
    r = run_oracle(case, inp)
    close(f64(g["Y"]), r["Y"], "Y")
    close(f64(g["T"]), r["T"], "T")
    if case.backward:
        close(f64(g["dX"]), r["dX"], "dX")
        close(g["dA"].cpu().numpy(), r["dA"], "dA")
        close(g["dB"].cpu().numpy(), r["dB"], "dB")
    return g, r


def test_cfg1_single_linear_full():
    check_case(synth.CFG1)


@pytest.mark.parametrize("fmt", ["nf4_dq", "int8"])
@pytest.mark.parametrize("M,N,K,r", [(200, 320, 320, 8), (130, 256, 512, 100), (64, 512, 256, 256),
                                     (1, 256, 256, 16), (300, 1024, 768, 64)])
def test_ragged_shapes_and_ranks(fmt, M, N, K, r):
    case = synth.LinearCase(f"ragged-{M}-{N}-{K}-{r}", N=N, K=K, M=M, r=r, alpha=2.0 * r,
                            fmt=fmt, seed=M + r)
    check_case(case)


def test_B_zero_gives_base_and_zero_dA():
    case = synth.CFG1
    inp = synth.make_inputs(case)
    inp["B"] = torch.zeros_like(inp["B"])
    g, r = check_case(case, inp) if False else (run_gpu(case, inp), run_oracle(case, inp))
    close(f64(g["Y"]), r["Y"], "Y(B=0)")
    assert torch.count_nonzero(g["dA"]).item() == 0


def test_A_zero_gives_zero_T_and_dB():
    case = synth.CFG1
    inp = synth.make_inputs(case)
    inp["A"] = torch.zeros_like(inp["A"])
    g = run_gpu(case, inp)
    r = run_oracle(case, inp)
    close(f64(g["Y"]), r["Y"], "Y(A=0)")
    assert torch.count_nonzero(g["T"]).item() == 0
    assert torch.count_nonzero(g["dB"]).item() == 0


def test_W_zero_isolates_the_adapter_branch():
    """W = 0: codes 8, W' = +0, so Y is the adapter term alone and dX = s U A alone."""
    case = synth.CFG1
    inp = synth.make_inputs(case)
    inp["W"] = torch.zeros_like(inp["W"])
    g = run_gpu(case, inp)
    r = run_oracle(case, inp)
    close(f64(g["Y"]), r["Y"], "Y(W=0)")
    close(f64(g["dX"]), r["dX"], "dX(W=0)")


def test_cfg3_upproj_full_size_sampled():
    """Fine-tune-shaped up-projection at full size: 256 sampled rows of Y and dX, dA and
    dB in full, against the fp64 oracle."""
    case = synth.CFG3
    inp = synth.make_inputs(case)
    g = run_gpu(case, inp)
    rows = np.sort(np.random.default_rng(0).choice(case.M, 256, replace=False))
    r = run_oracle(case, inp, rows=rows)
    close(f64(g["Y"])[rows], r["Y"], "Y")
    close(f64(g["T"])[rows], r["T"], "T")
    close(f64(g["dX"])[rows], r["dX"], "dX")
    close(g["dA"].cpu().numpy(), r["dA"], "dA")
    close(g["dB"].cpu().numpy(), r["dB"], "dB")


def test_timeout_path_reports_and_recovers():
    """Force every bounded wait to give up almost at once: the kernels must return,
    report QL_ERR_TIMEOUT through the device flag, free their TMEM, and leave the
    context usable for a normal run afterwards.

    With a 1 ns bound, any mbarrier wait that is not satisfied on its first poll gives
    up at the next tick of the global timer. The epilogue warps of the fused GEMM wait
    for the first accumulator during the whole first tile (the TMA loads from HBM, the
    decode and 12 contraction chunks of 64), which spans many timer ticks, so the
    timeout must be reported."""
    case = synth.LinearCase("timeout-300x1024x768", N=1024, K=768, M=300, r=64, alpha=16.0, seed=4)
    inp = synth.make_inputs(case)
    qw = B.quantize_weight(inp["W"].cuda(), case.fmt)
    X, A, Bm = inp["X"].cuda(), inp["A"].cuda(), inp["B"].cuda()
    torch.cuda.synchronize()
    assert B.device_status() == B.QL_OK
    B.lib().ql_set_wait_timeout_ns(1)
    try:
        B.linear_fwd(qw, X, A, Bm, case.alpha)
        st = B.device_status()
    finally:
        B.lib().ql_set_wait_timeout_ns(0)
    assert st == B.QL_ERR_TIMEOUT, B.status_string(st)
    assert B.device_status() == B.QL_OK                     # the flag was read and cleared
    check_case(case, inp)
    check_case(synth.CFG1)


# ---- decode-shaped forward (M <= 16): one cluster-split kernel ------------------------

@pytest.mark.parametrize("case", synth.CFG2, ids=[c.name for c in synth.CFG2])
def test_cfg2_decode_7b_full(case):
    """7B decode-shaped linear, 4096x4096 with 0.1% outliers at 20 sigma, r=16: every
    output of Y and T against the oracle."""
    check_case(case)


@pytest.mark.parametrize("M,N,K,r,fmt", [(1, 256, 256, 8, "nf4_dq"), (3, 200, 320, 20, "int8"),
                                         (16, 1024, 4160, 64, "nf4_dq"), (9, 136, 704, 1, "nf4_dq"),
                                         (16, 512, 11008, 16, "int8"), (5, 4096, 64, 33, "nf4_dq")])
def test_small_m_ragged(M, N, K, r, fmt):
    case = synth.LinearCase(f"small-{M}-{N}-{K}-{r}", N=N, K=K, M=M, r=r, alpha=16.0, fmt=fmt,
                            seed=N + K)
    check_case(case)


# ---- both fused-GEMM variants: single CTAs (default) and CTA pairs -------------------

@pytest.mark.parametrize("pair", [1, 0], ids=["pair", "single"])
@pytest.mark.parametrize("fmt", ["nf4_dq", "int8"])
@pytest.mark.parametrize("M,N,K,r", [(300, 1024, 768, 64), (517, 392, 1344, 24), (257, 640, 512, 130)])
def test_gemm_variants(pair, fmt, M, N, K, r):
    """Ragged weight rows and tokens (pair tiles of 256 x 256 leave an idle half), both
    formats, adapter ranks that need one, one and three extension chunks."""
    B.lib().ql_set_gemm_pair(pair)
    try:
        case = synth.LinearCase(f"variant-{M}-{N}-{K}-{r}", N=N, K=K, M=M, r=r, alpha=2.0 * r,
                                fmt=fmt, seed=M + N)
        check_case(case)
    finally:
        B.lib().ql_set_gemm_pair(0)
