"""The weight that the hot-path kernels decode, compared bit for bit with the oracle's W'.

The dequantisation rule (QLoRA page, aizip.shop/methodologies/qlora, "1. 4-bit NormalFloat"
and "2. Double Quantization"; blockwise int8 for the 8-bit format) is applied in three
places that never write W' out: the fused forward GEMM's decode warps, the same warps in
the input-backward GEMM (where the weight is used transposed), and the decode-shaped
kernel's lanes. A tolerance on Y or dX cannot see a one-ulp error in W', so these tests
feed inputs that make an output equal to W' exactly:

  forward,  X = I (one unit row per input feature), B = 0:  Y = X W'^T = W'^T;
  backward, dY = I (one unit row per output feature), B = 0:  dX = dY W' = W';
  decode-shaped forward, 16 unit rows per call:  Y holds 16 columns of W'^T.

Each output element is then one product 1 * w' added to exact zeros in fp32 and rounded
to bf16, which is w' itself. The comparison is on bf16 bit patterns; the only freedom is
the sign of a zero (a w' of -0 sums with +0 products to +0), so zeros are compared as
zeros."""
import numpy as np
import pytest
import torch

import oracle.qlora_oracle as o
from quantized_base_rank_b200 import binding as B
from quantized_base_rank_b200 import synth

pytestmark = pytest.mark.gpu

WEIGHTS = {
    # the 7B decode-shaped weight with 0.1% outliers at 20 sigma
    "decode-7b-4096x4096": lambda: synth.weight_with_outliers(4096, 4096, 0.02, 0.001, 20.0, 0),
    # ragged tiles: 640 rows (5 x 128; 2.5 pair tiles of 256), 768 features (3 x 256 tokens)
    "ragged-640x768": lambda: synth.normal_bf16((640, 768), 0.02, 11, 0),
}


def _bits(t: torch.Tensor) -> np.ndarray:
    b = t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16).astype(np.uint32)
    return np.where((b & 0x7FFF) == 0, 0, b)


def _oracle_bits(W: torch.Tensor, fmt: str) -> np.ndarray:
    N, K = W.shape
    wd = o.quantize_weight(W.float().numpy(), fmt)["wdeq"].reshape(N, K).astype(np.float32)
    b = o.f32_to_bf16_bits(wd).astype(np.uint32)
    return np.where((b & 0x7FFF) == 0, 0, b)


_cache = {}


def _weight(name: str, fmt: str):
    key = (name, fmt)
    if key not in _cache:
        W = WEIGHTS[name]()
        _cache[key] = (W, _oracle_bits(W, fmt))
    return _cache[key]


def _eye(n: int, dev) -> torch.Tensor:
    return torch.eye(n, dtype=torch.bfloat16, device=dev)


@pytest.mark.parametrize("pair", [0, 1], ids=["single", "pair"])
@pytest.mark.parametrize("fmt", ["nf4_dq", "int8"])
@pytest.mark.parametrize("name", list(WEIGHTS))
def test_fused_forward_decodes_the_oracle_weight(name, fmt, pair):
    W, want = _weight(name, fmt)
    N, K = W.shape
    r = 8
    qw = B.quantize_weight(W.cuda(), fmt)
    X = _eye(K, "cuda")                                     # M = K unit rows
    A = synth.normal_bf16((r, K), 1.0 / K, 3, 0).cuda()
    Bz = torch.zeros((N, r), dtype=torch.bfloat16, device="cuda")
    B.lib().ql_set_gemm_pair(pair)
    try:
        Y, _ = B.linear_fwd(qw, X, A, Bz, 16.0)
        torch.cuda.synchronize()
    finally:
        B.lib().ql_set_gemm_pair(0)
    assert B.device_status() == B.QL_OK
    got = _bits(Y.t())                                      # Y = W'^T
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} decoded elements differ, first at (n, k) = {tuple(bad[0])}"


@pytest.mark.parametrize("pair", [0, 1], ids=["single", "pair"])
@pytest.mark.parametrize("fmt", ["nf4_dq", "int8"])
@pytest.mark.parametrize("name", list(WEIGHTS))
def test_input_backward_decodes_the_oracle_weight(name, fmt, pair):
    W, want = _weight(name, fmt)
    N, K = W.shape
    r = 8
    qw = B.quantize_weight(W.cuda(), fmt)
    M = N
    dY = _eye(N, "cuda")                                    # M = N unit rows
    X = synth.normal_bf16((M, K), 1.0, 4, 0).cuda()
    A = synth.normal_bf16((r, K), 1.0 / K, 3, 0).cuda()
    Bz = torch.zeros((N, r), dtype=torch.bfloat16, device="cuda")
    T = synth.normal_bf16((M, r), 1.0, 5, 0).cuda()
    B.lib().ql_set_gemm_pair(pair)
    try:
        dX, dA, _ = B.linear_bwd(qw, X, dY, A, Bz, T, 16.0)
        torch.cuda.synchronize()
    finally:
        B.lib().ql_set_gemm_pair(0)
    assert B.device_status() == B.QL_OK
    got = _bits(dX)                                         # dX = W'
    bad = np.argwhere(got != want)
    assert bad.size == 0, f"{len(bad)} decoded elements differ, first at (n, k) = {tuple(bad[0])}"
    assert torch.count_nonzero(dA).item() == 0              # Q = s dY B = 0, so dA = Q^T X = 0


@pytest.mark.parametrize("fmt", ["nf4_dq", "int8"])
@pytest.mark.parametrize("name", list(WEIGHTS))
def test_decode_shaped_forward_decodes_the_oracle_weight(name, fmt):
    W, want = _weight(name, fmt)
    N, K = W.shape
    r = 16
    qw = B.quantize_weight(W.cuda(), fmt)
    A = synth.normal_bf16((r, K), 1.0 / K, 3, 0).cuda()
    Bz = torch.zeros((N, r), dtype=torch.bfloat16, device="cuda")
    eye = _eye(K, "cuda")
    got = torch.empty((K, N), dtype=torch.bfloat16, device="cuda")
    for k0 in range(0, K, 16):                              # 16 unit rows per call
        Y, _ = B.linear_fwd(qw, eye[k0:k0 + 16].contiguous(), A, Bz, 32.0)
        got[k0:k0 + 16] = Y
    torch.cuda.synchronize()
    assert B.device_status() == B.QL_OK
    g = _bits(got.t())
    bad = np.argwhere(g != want)
    assert bad.size == 0, f"{len(bad)} decoded elements differ, first at (n, k) = {tuple(bad[0])}"
