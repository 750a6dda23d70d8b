"""The Python binding refuses mismatched tensors before it calls the library.

The C entry points take bare pointers, so a wrong shape, a short output buffer or a tensor
on another device would make a kernel read or write outside the caller's memory. These
checks run on the CPU: the CUDA-placement test is stubbed to accept CPU tensors and the
library loader is replaced by one that raises `Reached`, so a well-formed call ends there
and a malformed one must raise ValueError first.
"""
import pytest
import torch

import quantized_base_rank_b200.binding as B


class Reached(Exception):
    pass


@pytest.fixture
def cpu_binding(monkeypatch):
    monkeypatch.setattr(B, "_is_cuda", lambda t: True)

    def no_library():
        raise Reached()

    monkeypatch.setattr(B, "lib", no_library)
    return B


bf, f32 = torch.bfloat16, torch.float32
M, N, K, r = 5, 128, 192, 8


def weight():
    n = N * K
    nb = n // 64
    return B.QuantWeight("nf4_dq", N, K, torch.zeros(n // 2, dtype=torch.uint8), None,
                         torch.zeros(nb, dtype=torch.int8), torch.zeros((nb + 255) // 256, dtype=f32),
                         torch.zeros(1, dtype=f32))


def z(*shape, dtype=bf):
    return torch.zeros(shape, dtype=dtype)


def test_linear_forward(cpu_binding):
    qw = weight()
    with pytest.raises(Reached):
        B.linear_fwd(qw, z(M, K), z(r, K), z(N, r), 16.0)
    with pytest.raises(Reached):
        B.linear_fwd(qw, z(M, K), z(r, K), z(N, r), 16.0, Y=z(M, N), T=z(M, r))
    bad = [
        dict(X=z(M, K + 64)),                       # X does not match the weight's K
        dict(A=z(r, K - 64)),
        dict(B=z(N, r + 1)),
        dict(B=z(N - 1, r)),
        dict(Y=z(M, N - 1)),
        dict(Y=z(M, N, dtype=f32)),
        dict(T=z(M + 1, r)),
    ]
    for kw in bad:
        args = dict(X=z(M, K), A=z(r, K), B=z(N, r), Y=None, T=None)
        args.update(kw)
        with pytest.raises(ValueError):
            B.linear_fwd(qw, args["X"], args["A"], args["B"], 16.0, Y=args["Y"], T=args["T"])


def test_linear_backward(cpu_binding):
    qw = weight()
    ok = dict(X=z(M, K), dY=z(M, N), A=z(r, K), B=z(N, r), T=z(M, r), dX=None, dA=None, dB=None)
    with pytest.raises(Reached):
        B.linear_bwd(qw, ok["X"], ok["dY"], ok["A"], ok["B"], ok["T"], 16.0)
    bad = [dict(dY=z(M, N + 1)), dict(T=z(M, r + 1)), dict(A=z(r + 1, K)), dict(dX=z(M, K + 1)),
           dict(dA=z(r, K)), dict(dA=z(r, K - 1, dtype=f32)), dict(dB=z(N, r + 1, dtype=f32))]
    for kw in bad:
        a = dict(ok)
        a.update(kw)
        with pytest.raises(ValueError):
            B.linear_bwd(qw, a["X"], a["dY"], a["A"], a["B"], a["T"], 16.0, dX=a["dX"], dA=a["dA"], dB=a["dB"])


def test_quantise_outputs(cpu_binding):
    n = 64 * 300 + 11                       # odd: the codes need (n + 1) // 2 bytes
    W = z(n)
    nb = (n + 63) // 64
    with pytest.raises(Reached):
        B.nf4_quantize(W)
    with pytest.raises(ValueError):
        B.nf4_quantize(W, codes=z(n // 2, dtype=torch.uint8))             # one byte short
    with pytest.raises(ValueError):
        B.nf4_quantize(W, absmax=z(nb - 1, dtype=f32))
    with pytest.raises(ValueError):
        B.int8_quantize(W, codes=z(n, dtype=torch.uint8))                 # int8 codes, not uint8
    with pytest.raises(ValueError):
        B.nf4_dq_quantize(W, group_scale=z(1, dtype=f32))                 # nb > 256 needs 2 scales
    with pytest.raises(ValueError):
        B.dq_quantize(z(nb, dtype=f32), qabsmax=z(nb - 1, dtype=torch.int8))
    with pytest.raises(ValueError):
        B.dq_quantize(z(nb, dtype=f32), mean=z(2, dtype=f32))
    with pytest.raises(ValueError):
        B.nf4_quantize_shard(W, bins=z(15, dtype=torch.int64))
    with pytest.raises(ValueError):
        B.dq_quantize_shard(z(nb, dtype=f32), z(16, dtype=torch.int32), nb)


def test_adapters(cpu_binding):
    qw = weight()
    R, ell = 40, 2
    lb = dict(B1=z(N, 2, dtype=torch.int32), B2=z(R, K // 32, dtype=torch.int32), alpha=z(ell, N, dtype=torch.float16),
              beta=z(ell, R, dtype=torch.float16), gamma=z(ell, K, dtype=torch.float16))
    with pytest.raises(Reached):
        B.linear_fwd_lordba(qw, z(M, K), lb["B1"], lb["B2"], lb["alpha"], lb["beta"], lb["gamma"], R)
    for k, t in (("B1", z(N, 1, dtype=torch.int32)), ("B2", z(R, K // 32 - 1, dtype=torch.int32)),
                 ("beta", z(ell, R - 1, dtype=torch.float16)), ("gamma", z(ell, K + 1, dtype=torch.float16)),
                 ("alpha", z(ell, N, dtype=bf))):
        a = dict(lb)
        a[k] = t
        with pytest.raises(ValueError):
            B.linear_fwd_lordba(qw, z(M, K), a["B1"], a["B2"], a["alpha"], a["beta"], a["gamma"], R)
    nnz = 37
    rp, col, c = z(N + 1, dtype=torch.int32), z(nnz, dtype=torch.uint16), z(nnz)
    with pytest.raises(Reached):
        B.linear_fwd_qwha(qw, z(M, K), rp, col, c)
    for args in ((z(N, dtype=torch.int32), col, c), (rp, z(nnz - 1, dtype=torch.uint16), c)):
        with pytest.raises(ValueError):
            B.linear_fwd_qwha(qw, z(M, K), *args)
    with pytest.raises(ValueError):
        B.linear_fwd_qwha(qw, z(M, K), rp, col, c, Y=z(N, M))
    with pytest.raises(ValueError):
        B.wht(z(M, K), Z=z(M, K - 64))


def test_optimisers(cpu_binding):
    n = 1000
    v = lambda k=n, dt=f32: z(k, dtype=dt)
    with pytest.raises(Reached):
        B.adamw_step(v(), v(dt=bf), v(), v(), v(), 1, 1e-3)
    with pytest.raises(ValueError):
        B.adamw_step(v(), v(dt=bf), v(), v(n - 1), v(), 1, 1e-3)
    with pytest.raises(Reached):
        B.lion_int8_step(v(), v(dt=bf), v(), v(dt=torch.int8), v((n + 63) // 64), 1e-4)
    with pytest.raises(ValueError):
        B.lion_int8_step(v(), v(dt=bf), v(), v(dt=torch.int8), v(n // 64), 1e-4)
