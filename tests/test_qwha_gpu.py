"""GPU vs oracle: the quantised linear with a Walsh-Hadamard adapter (QWHA page,
gist.science/ko/paper/2509.17428, section 2.1), Delta W = F H^{-1}, on the decode-shaped
and the large-M paths, both base formats, power-of-two and blockwise widths, and the
standalone transform.

Y is checked within relative Frobenius <= 5e-3 and elementwise <= 1e-2 * max|ref| of the
fp64 oracle on the same dequantised weight and the same bf16 c. The transform alone is
checked element by element against one bf16 rounding of the exact value."""
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


def _adapter(N, K, r_equiv, seed, dev="cuda"):
    ad = synth.qwha_inputs(N, K, r_equiv, seed)
    return ad, (ad["row_ptr"].to(dev), ad["col"].to(dev), ad["c"].to(dev))


def _run(M, N, K, r_equiv, fmt, zero_w=False, zero_c=False, seed=1, rows=None):
    case = synth.LinearCase(f"qwha-{M}-{N}-{K}", N=N, K=K, M=M, r=8, alpha=8.0, fmt=fmt, seed=seed,
                            backward=False)
    inp = synth.make_inputs(case)
    W = torch.zeros_like(inp["W"]) if zero_w else inp["W"]
    ad, (rp, col, c) = _adapter(N, K, r_equiv, seed)
    if zero_c:
        c = torch.zeros_like(c)
    qw = B.quantize_weight(W.cuda(), fmt)
    Y = B.linear_fwd_qwha(qw, inp["X"].cuda(), rp, col, c)
    torch.cuda.synchronize()
    assert B.device_status() == B.QL_OK
    wd = o.quantize_weight(W.float().numpy(), fmt)["wdeq"].reshape(N, K)
    X = inp["X"].float().numpy()
    cv = c.float().cpu().numpy()
    sel = np.arange(M) if rows is None else rows
    ref = o.qwha_linear_fwd_factored(X[sel], wd, ad["row_ptr"].numpy(), ad["col"].numpy().astype(np.int64), cv)
    _close(Y.float().cpu().numpy()[sel], ref, f"Y M={M} N={N} K={K} r~{r_equiv} {fmt}")
    return Y, qw, inp


@pytest.mark.parametrize("fmt", ["nf4_dq", "int8"])
@pytest.mark.parametrize("M,N,K,r_equiv", [
    (1, 4096, 4096, 16),        # decode-shaped sparse path, one full-width block
    (5, 136, 704, 8),           # decode-shaped, 11 blocks of 64
    (16, 512, 1024, 64),        # decode-shaped, 16 tokens
    (17, 256, 256, 8),          # smallest tensor-core case: dW = F H in blocks of 256
    (300, 392, 512, 20),        # blocks of 512
    (33, 64, 192, 4),           # blocks of 64 (the tile transform is the row transform alone)
    (33, 64, 384, 4),           # blocks of 128
    (24, 128, 1024, 8),         # blocks of 1024
    (24, 128, 2048, 8),         # blocks of 2048
    (200, 512, 4096, 64),       # full 4096-wide blocks
    (70, 264, 11008, 16),       # 43 blocks of 256 over three 4096-column tiles, the last partial
    (40, 128, 8192, 8),         # one block of 8192: dW through the dense F and the row transform
])
def test_qwha_forward(M, N, K, r_equiv, fmt):
    _run(M, N, K, r_equiv, fmt)


@pytest.mark.parametrize("fmt", ["nf4_dq", "int8"])
@pytest.mark.parametrize("M,N,K,r_equiv", [(300, 392, 512, 20), (70, 264, 11008, 16), (257, 128, 4096, 32)])
def test_qwha_forward_pair_gemm(M, N, K, r_equiv, fmt):
    """The update merged into the decoded weight by the CTA-pair GEMM (256 weight rows x
    256 tokens per MMA): ragged rows and tokens leave idle halves of pair tiles."""
    B.lib().ql_set_gemm_pair(1)
    try:
        _run(M, N, K, r_equiv, fmt)
    finally:
        B.lib().ql_set_gemm_pair(0)


@pytest.mark.parametrize("M", [3, 77])
def test_qwha_adapter_alone(M):
    """W = 0: Y is the Walsh-Hadamard branch alone."""
    _run(M, 256, 1024, 32, "nf4_dq", zero_w=True)


@pytest.mark.parametrize("M", [4, 100])
def test_qwha_zero_values_equal_base(M):
    """c = 0: Y equals the quantised base product of the LoRA entry with B = 0."""
    Y, qw, inp = _run(M, 256, 512, 16, "nf4_dq", zero_c=True)
    A = inp["A"].cuda()
    Yl, _ = B.linear_fwd(qw, inp["X"].cuda(), A, torch.zeros_like(inp["B"]).cuda(), 8.0, save_T=False)
    assert torch.equal(Y.float(), Yl.float())


def test_qwha_empty_adapter():
    """nnz = 0: the base product alone."""
    case = synth.LinearCase("qwha-empty", N=128, K=256, M=20, r=8, alpha=8.0, fmt="nf4_dq", seed=4,
                            backward=False)
    inp = synth.make_inputs(case)
    qw = B.quantize_weight(inp["W"].cuda(), "nf4_dq")
    rp = torch.zeros(129, dtype=torch.int32, device="cuda")
    empty_col = torch.zeros(0, dtype=torch.uint16, device="cuda")
    empty_c = torch.zeros(0, dtype=torch.bfloat16, device="cuda")
    Y = B.linear_fwd_qwha(qw, inp["X"].cuda(), rp, empty_col, empty_c)
    torch.cuda.synchronize()
    wd = o.quantize_weight(inp["W"].float().numpy(), "nf4_dq")["wdeq"].reshape(128, 256)
    _close(Y.float().cpu().numpy(), inp["X"].float().numpy() @ wd.T, "Y empty adapter")


def test_qwha_full_size_sampled_rows():
    """The 7B up-projection at 8192 tokens, adapter budget of a rank-64 LoRA (966,656
    values): 64 sampled token rows against the oracle."""
    rows = np.sort(np.random.default_rng(0).choice(8192, 64, replace=False))
    _run(8192, 11008, 4096, 64, "nf4_dq", rows=rows, seed=3)


def test_qwha_bad_index_is_flagged_not_read():
    """A column index >= K and a row offset past nnz are skipped by the kernel's own
    bounds checks and reported as QL_ERR_INVALID_ARG; Y stays finite."""
    case = synth.LinearCase("qwha-bad", N=64, K=256, M=33, r=8, alpha=8.0, fmt="nf4_dq", seed=6,
                            backward=False)
    inp = synth.make_inputs(case)
    qw = B.quantize_weight(inp["W"].cuda(), "nf4_dq")
    ad, (rp, col, c) = _adapter(64, 256, 4, 6)
    col_bad = col.clone()
    col_bad[3] = 300                                  # >= K
    Y = B.linear_fwd_qwha(qw, inp["X"].cuda(), rp, col_bad, c)
    assert B.device_status() == B.QL_ERR_INVALID_ARG
    assert torch.isfinite(Y.float()).all()
    rp_bad = rp.clone()
    rp_bad[-1] = rp_bad[-1] + 5                       # past nnz
    B.linear_fwd_qwha(qw, inp["X"].cuda(), rp_bad, col, c)
    assert B.device_status() == B.QL_ERR_INVALID_ARG
    B.linear_fwd_qwha(qw, inp["X"].cuda(), rp, col, c)
    assert B.device_status() == B.QL_OK


# ---- the transform alone --------------------------------------------------------------

@pytest.mark.parametrize("K", [64, 256, 704, 4096, 8192, 11008])
@pytest.mark.parametrize("M", [1, 21])
def test_wht_against_oracle(M, K):
    """Z = bf16(X H^{-T}): every element within one bf16 rounding of the exact value (half
    an ulp: at most 2^-8 relative, bf16 keeping 8 significant bits), plus fp32 summation
    error."""
    X = synth.normal_bf16((M, K), 1.0, 9, K)
    Z = B.wht(X.cuda()).float().cpu().numpy()
    ref = o.qwha_transform(X.float().numpy())
    tol = 2.0 ** -8 * np.abs(ref) + 1e-5 * np.sqrt(np.mean(ref ** 2))
    assert np.all(np.abs(Z - ref) <= tol), f"K={K}: max excess {np.max(np.abs(Z - ref) - tol):.3e}"


def test_wht_of_unit_vectors_is_exact():
    """e_k -> the Walsh function of index k / 64 (K = 4096): every value is +-2^-6, exact."""
    K = 4096
    ks = [0, 1, 77, 2048, 4095]
    X = torch.zeros((len(ks), K), dtype=torch.bfloat16)
    for t, k in enumerate(ks):
        X[t, k] = 1.0
    Z = B.wht(X.cuda()).float().cpu().numpy()
    j = np.arange(K)
    for t, k in enumerate(ks):
        par = np.array([bin(k & v).count("1") & 1 for v in j])
        assert np.array_equal(Z[t], np.where(par == 1, -1.0, 1.0) / 64.0)


# ---- edge cases ------------------------------------------------------------------------

def _run_custom(M, N, K, row_ptr, col, c, fmt="nf4_dq", seed=12):
    case = synth.LinearCase(f"qwha-edge-{M}-{N}-{K}", N=N, K=K, M=M, r=8, alpha=8.0, fmt=fmt, seed=seed,
                            backward=False)
    inp = synth.make_inputs(case)
    qw = B.quantize_weight(inp["W"].cuda(), fmt)
    Y = B.linear_fwd_qwha(qw, inp["X"].cuda(), torch.tensor(row_ptr, dtype=torch.int32).cuda(),
                          torch.tensor(np.asarray(col, np.uint16)).cuda(),
                          synth.to_bf16(np.asarray(c, np.float32)).cuda())
    torch.cuda.synchronize()
    assert B.device_status() == B.QL_OK
    wd = o.quantize_weight(inp["W"].float().numpy(), fmt)["wdeq"].reshape(N, K)
    cv = synth.to_bf16(np.asarray(c, np.float32)).float().numpy()
    ref = o.qwha_linear_fwd(inp["X"].float().numpy(), wd, row_ptr, np.asarray(col, np.int64), cv)
    _close(Y.float().cpu().numpy(), ref, f"edge M={M} N={N} K={K}")


@pytest.mark.parametrize("M", [1, 16, 17])
def test_qwha_smallest_width(M):
    """K = 64 (one 64-point block), N = 8: the smallest shape the format allows."""
    rng = np.random.default_rng(M)
    cnt = [3, 0, 64, 1, 0, 7, 2, 5]                   # an empty row and a full row
    row_ptr = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int32)
    col = np.concatenate([np.sort(rng.choice(64, k, replace=False)) for k in cnt])
    c = rng.standard_normal(int(row_ptr[-1])) * 0.05
    _run_custom(M, 8, 64, row_ptr, col, c)


@pytest.mark.parametrize("M", [1, 8, 16, 40])
def test_qwha_dense_row_spans_several_batches(M):
    """One row holds all 1024 columns (several gather batches on the decode-shaped path,
    and a full dense row on the tensor-core path); the others hold one value or none."""
    N, K = 24, 1024
    rng = np.random.default_rng(40 + M)
    cnt = [0] * N
    cnt[5] = K
    for i in range(0, N, 3):
        if i != 5:
            cnt[i] = 1
    row_ptr = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int32)
    col = np.concatenate([np.sort(rng.choice(K, k, replace=False)) for k in cnt])
    c = rng.standard_normal(int(row_ptr[-1])) * 0.02
    _run_custom(M, N, K, row_ptr, col, c)
