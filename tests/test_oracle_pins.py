"""Pins for the CPU oracle: each test fixes part of it against something other than
itself (a closed form, an independent high-precision evaluation, exact rational
brute force, finite differences, or a figure printed on the QLoRA page)."""
import json
import math
import os
from fractions import Fraction

import mpmath
import numpy as np
import pytest
import torch

import oracle.qlora_oracle as o

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_f32(x):
    return torch.tensor(np.asarray(x, np.float32)).to(torch.bfloat16).float().numpy()


# ---------------------------------------------------------------- P1 codebook

def _mp_rn32(x: mpmath.mpf):
    """Round an mpmath real to the nearest fp32 directly (no fp64 step); also
    return the distance from the nearest rounding boundary in ulps."""
    if x == 0:
        return np.float32(0), 0.5
    e = int(mpmath.floor(mpmath.log(abs(x), 2)))
    scaled = abs(x) * mpmath.mpf(2) ** (23 - e)
    n = int(mpmath.nint(scaled))
    margin = 0.5 - abs(float(scaled - mpmath.floor(scaled)) - 0.5)
    val = math.copysign(n * 2.0 ** (e - 23), float(x))
    return np.float32(val), margin


def test_codebook_matches_50_digit_evaluation():
    mpmath.mp.dps = 50
    q = o.nf4_codebook()
    scale = mpmath.sqrt(2) * mpmath.erfinv(2 * mpmath.mpf(31) / 32 - 1)
    for i in range(16):
        p = (mpmath.mpf(i) + mpmath.mpf(1) / 2) / 16
        exact = mpmath.sqrt(2) * mpmath.erfinv(2 * p - 1) / scale
        ref, margin = _mp_rn32(exact)
        assert ref.view(np.uint32) == q[i].view(np.uint32), (i, ref, q[i])
        # far from a rounding boundary, so RN32 of the fp64 quantile is unambiguous
        assert margin > 0.02 or i in (0, 15)


def test_codebook_shape_symmetry_endpoints():
    q = o.nf4_codebook()
    assert q.dtype == np.float32 and q.size == 16
    assert q[0] == -1.0 and q[15] == 1.0
    assert np.all(np.diff(q) > 0)
    assert np.array_equal(q[::-1], -q)           # exact antisymmetry
    assert not np.any(q == 0)                    # the centred grid has no zero point


def test_codebook_equal_mass():
    """Phi(q_i * Q(31/32)) = (i + 1/2)/16: every point is the centre of an equal-mass
    bin of N(0, 1) (checked with math.erfc, independent of the quantile routine)."""
    q = o.nf4_codebook().astype(np.float64)
    c = o.normal_quantile(31 / 32)
    for i in range(16):
        z = q[i] * c
        phi = 0.5 * math.erfc(-z / math.sqrt(2))
        assert abs(phi - (i + 0.5) / 16) < 2e-7, i


def test_page_grid_size():
    g = json.load(open(os.path.join(GOLDEN, "qlora_page_figures.json")))
    assert o.nf4_codebook().size == g["grid_points"]["value"] == 2 ** g["grid_bits"]["value"]
    assert o.BLOCK == g["block_size"]["value"]


# ---------------------------------------------------------------- P2 midpoints

def test_midpoints():
    q = o.nf4_codebook().astype(np.float64)
    m = o.nf4_midpoints()
    assert m.size == 15 and m[7] == 0.0
    assert np.all(np.diff(m) > 0)
    assert np.all((q[:-1] < m) & (m < q[1:]))
    assert np.array_equal(2.0 * m - q[:-1], q[1:])     # exact midpoints
    assert np.array_equal(m[::-1], -m)


def test_midpoints_have_many_significant_bits():
    """a * m_j is never a bf16 value for a bf16 a (so no exact ties except at 0):
    the odd part of every nonzero m_j has more than 8 bits."""
    for j, v in enumerate(o.nf4_midpoints()):
        if v == 0:
            continue
        num = Fraction(float(v)).numerator
        while num % 2 == 0:
            num //= 2
        assert abs(num).bit_length() > 8, j


# ---------------------------------------------------------------- P3 encoder brute force

def _brute_code(x: float, a: float, qf):
    if a == 0:
        return 8
    r = Fraction(x) / Fraction(a)
    d = [abs(r - qi) for qi in qf]
    best = min(d)
    return max(i for i in range(16) if d[i] == best)     # ties go to the upper point


def _all_bf16_upto(a: float):
    bits = np.arange(0, 0x7F80, dtype=np.uint32)          # +0 .. largest finite
    vals = (bits << 16).view(np.float32)
    vals = vals[vals <= a]
    return np.concatenate([vals, -vals])


@pytest.mark.parametrize("a_bits", [0x3F80, 0x3CE0, 0x7F7F, 0x0080, 0x0003, 0x4123])
def test_encoder_matches_exact_rational_nearest(a_bits):
    """Every bf16 x with |x| <= a (or a 3000-sample of them), including +-0 and
    subnormals, against the exact-rational nearest grid point with ties upward."""
    a = float(np.array([a_bits << 16], np.uint32).view(np.float32)[0])
    xs = _all_bf16_upto(a)
    rng = np.random.default_rng(a_bits)
    if xs.size > 3000:
        keep = rng.choice(xs.size, 3000, replace=False)
        xs = np.concatenate([xs[keep], np.float32([0.0, -0.0, a, -a])])
    qf = [Fraction(float(v)) for v in o.nf4_codebook()]
    nb = (xs.size + 63) // 64
    codes = o.nf4_encode(xs, np.full(nb, a, np.float32))
    for x, c in zip(xs.tolist(), codes.tolist()):
        assert c == _brute_code(x, a, qf), (x, a, c)


def test_encoder_zero_block_and_signed_zero():
    codes = o.nf4_encode(np.float32([0.0, -0.0] * 32), np.float32([0.0]))
    assert np.all(codes == 8)
    codes = o.nf4_encode(np.float32([0.0, -0.0, 1.0, -1.0] + [0.5] * 60), np.float32([1.0]))
    assert codes[:4].tolist() == [8, 8, 15, 0]


def test_block_absmax_partial_last_block():
    w = bf16_f32(np.random.default_rng(1).standard_normal(64 * 3 + 5))
    a = o.block_absmax(w)
    assert a.size == 4
    for b in range(4):
        assert a[b] == np.max(np.abs(w[b * 64:(b + 1) * 64]))


# ---------------------------------------------------------------- P4 exact codebook dequant

@pytest.mark.parametrize("e", [-20, -3, 0, 7, 100])
def test_codebook_points_roundtrip_exactly(e):
    """A block built from RNbf(q_c * 2^e) with one entry 2^e (so a = 2^e) encodes
    back to c and, without double quantisation, dequantises to itself bit-exactly."""
    rng = np.random.default_rng(e + 50)
    c = rng.integers(0, 16, size=64).astype(np.uint8)
    c[5] = 15
    q = o.nf4_codebook()
    w = bf16_f32(q[c] * np.float32(2.0 ** e))
    packed, a = o.nf4_quantize(w)
    assert a[0] == np.float32(2.0 ** e)
    assert np.array_equal(o.unpack_nibbles(packed, 64), c)
    wd = o.nf4_dequant(packed, a, 64)
    assert np.array_equal(wd.view(np.uint32), w.view(np.uint32))


def test_pack_order():
    c = np.arange(16, dtype=np.uint8)
    p = o.pack_nibbles(c)
    assert p[0] == 0x10 and p[1] == 0x32 and p[7] == 0xFE
    assert np.array_equal(o.unpack_nibbles(o.pack_nibbles(c[:5]), 5), c[:5])
    assert o.pack_nibbles(c[:5])[2] == 0x04                   # odd count: high nibble 0


# ---------------------------------------------------------------- P5 idempotence

def test_requantise_idempotent_without_dq():
    w = bf16_f32(np.random.default_rng(7).standard_normal(64 * 512) * 0.02)
    packed, a = o.nf4_quantize(w)
    wd = o.nf4_dequant(packed, a, w.size)
    packed2, a2 = o.nf4_quantize(wd)
    assert np.array_equal(packed2, packed)
    assert np.array_equal(a2, a)
    wd2 = o.nf4_dequant(packed2, a2, w.size)
    assert np.array_equal(wd2.view(np.uint32), wd.view(np.uint32))


def test_requantise_codes_stable_with_dq():
    w = bf16_f32(np.random.default_rng(8).standard_normal(64 * 1024) * 0.02)
    r = o.quantize_weight(w, "nf4_dq")
    r2 = o.quantize_weight(r["wdeq"], "nf4_dq")
    assert np.array_equal(r2["codes"], r["codes"])
    # the re-derived constants differ by at most half a DQ step, so W'' differs from
    # W' by at most that (|q| <= 1) plus one bf16 rounding on each side
    g = (np.arange(w.size) // 64) // 256
    d = np.abs(r2["wdeq"].astype(np.float64) - r["wdeq"])
    bound = r2["group_scale"][g] * 0.5 + np.abs(r["wdeq"]) * 2.0 ** -7 + 1e-30
    assert np.all(d <= bound)


# ---------------------------------------------------------------- P6 accounting

def test_bits_per_param_accounting():
    g = json.load(open(os.path.join(GOLDEN, "qlora_page_figures.json")))
    for n in (16384, 4096 * 4096, 11008 * 4096):
        sb = o.storage_bytes("nf4_dq", n)
        assert sb["codes"] * 2 == n                         # ~N/2 bytes of NF4 weights
        per_group = (sb["codes"] + sb["qabsmax"] + sb["group_scale"]) * 8 / n
        assert per_group == 4.126953125                     # 4 + 8/64 + 32/(64*256)
        total = sum(sb.values()) * 8 / n
        assert total == 4.126953125 + 32 / n                # plus one fp32 mean
        const_bits = per_group - 4
        assert abs(const_bits - g["const_bits_after_dq"]["value"]) <= g["const_bits_after_dq"]["tol"]
        # the page's 0.37 saving holds against 32-bit constants (32/64 - 0.127)
        assert abs((32 / 64 - const_bits) - g["saving_bits"]["value"]) <= g["saving_bits"]["tol"]
        assert 16 / g["block_size"]["value"] == g["const_bits_16bit"]["value"]
        assert sb["codes"] / n == g["nf4_weight_bytes_per_param"]["value"]
        sb8 = o.storage_bytes("int8", n)
        assert sum(sb8.values()) * 8 / n == 8.5
    # 65B parameters in fp16: the page's ~130 GB
    assert abs(65e9 * 2 / 1e9 - g["fp16_65b_full_gb"]["value"]) <= g["fp16_65b_full_gb"]["tol"]


# ---------------------------------------------------------------- P7 double quantisation

def test_dq_worked_example():
    """absmax [1, 3]: mu = 2, d = [-1, 1], s = RN32(1/127), codes -127/+127, and the
    reconstruction is exact (worked by hand: RN32(127 * RN32(1/127)) = 1)."""
    qa, sc, mu = o.dq_encode(np.float32([1.0, 3.0]))
    assert mu == 2.0
    assert sc.tolist() == [float(np.float32(1.0) / np.float32(127))]
    assert qa.tolist() == [-127, 127]
    assert o.dq_decode(qa, sc, mu).tolist() == [1.0, 3.0]


def test_dq_constant_tensor_is_exact():
    a = np.full(1000, 0.046875, np.float32)
    qa, sc, mu = o.dq_encode(a)
    assert mu == np.float32(0.046875) and np.all(sc == 0) and np.all(qa == 0)
    assert np.array_equal(o.dq_decode(qa, sc, mu), a)


def test_dq_roundtrip_bound_and_mean():
    w = bf16_f32(np.random.default_rng(3).standard_normal(64 * 256 * 9 + 64 * 17) * 0.02)
    a = o.block_absmax(w)
    qa, sc, mu = o.dq_encode(a)
    assert sc.size == (a.size + 255) // 256
    # exact mean, by rational arithmetic
    exact = sum(Fraction(float(v)) for v in a) / a.size
    assert mu == np.float32(float(exact))
    ar = o.dq_decode(qa, sc, mu)
    g = np.arange(a.size) // 256
    ulp = np.spacing(np.maximum(np.abs(a), abs(mu)).astype(np.float32))
    assert np.all(np.abs(ar.astype(np.float64) - a) <= sc[g] * 0.5 + 4 * ulp)
    assert np.all(np.abs(qa.astype(int)) <= 127) and np.max(np.abs(qa.astype(int))) == 127


def _dq_tie_groups():
    """Two groups of 256 constants built so that every DQ quantity is exact: each group is
    symmetric about 1 (so the tensor mean is exactly 1), its largest |a - 1| is 127 * 2^-k
    (so the group scale is exactly 2^-k), and the other offsets are small multiples of
    2^-(k+1), so a - 1 and (a - 1) / 2^-k are exact in fp32. The quotients include the
    half-way cases +-0.5, +-1.5, +-2.5, +-3.5 and +-126.5."""
    groups, want = [], []
    for k in (7, 5):
        s = Fraction(1, 2 ** k)
        qs = [Fraction(127), Fraction(5, 2), Fraction(7, 2), Fraction(1, 2), Fraction(3, 2),
              Fraction(253, 2), Fraction(0), Fraction(3), Fraction(41, 4)]
        offs = []
        for qv in qs:
            offs += [qv, -qv]
        offs += [Fraction(0)] * (256 - len(offs))
        groups.append([1 + qv * s for qv in offs])
        # the code each half-way quotient must take under round-half-to-even (by hand)
        hand = {Fraction(127): 127, Fraction(5, 2): 2, Fraction(7, 2): 4, Fraction(1, 2): 0,
                Fraction(3, 2): 2, Fraction(253, 2): 126, Fraction(0): 0, Fraction(3): 3,
                Fraction(41, 4): 10}
        want.append([hand[abs(qv)] * (1 if qv >= 0 else -1) for qv in offs])
    return groups, want


def test_dq_encode_rounds_half_to_even_on_exact_ties():
    """Double quantisation's code is round-half-to-even of d / s_g (QLoRA page, "2. Double
    Quantization", with the half-even reading): constructed exact ties 2.5 -> 2, 3.5 -> 4,
    0.5 -> 0, 1.5 -> 2, 126.5 -> 126 and their negatives, with the mean and the group
    scales exact. Half-away-from-zero, truncation or a floor would each fail here."""
    groups, want = _dq_tie_groups()
    a = np.array([float(v) for g in groups for v in g], dtype=np.float64)
    assert all(Fraction(float(np.float32(v))) == v for g in groups for v in g)   # exact in fp32
    a = a.astype(np.float32)
    qa, sc, mu = o.dq_encode(a)
    assert mu == np.float32(1.0)
    assert sc.tolist() == [2.0 ** -7, 2.0 ** -5]
    assert qa.astype(int).tolist() == [c for w in want for c in w]


# ---------------------------------------------------------------- int8 format

def test_int8_format():
    w = bf16_f32(np.random.default_rng(4).standard_normal(64 * 300) * 0.02)
    c, a = o.int8_quantize(w)
    assert c.dtype == np.int8 and np.max(np.abs(c.astype(int))) == 127
    sc = a / np.float32(127)
    wd = o.int8_dequant(c, a)
    b = np.arange(w.size) // 64
    assert np.all(np.abs(wd - w) <= sc[b] * 0.5 * (1 + 2 ** -7) + np.abs(w) * 2 ** -8)
    # the element equal to the absmax maps to +-127 and back to itself
    i = np.argmax(np.abs(w[:64]))
    assert abs(int(c[i])) == 127
    # a zero block stays zero
    c0, a0 = o.int8_quantize(np.zeros(64, np.float32))
    assert np.all(c0 == 0) and o.int8_dequant(c0, a0).tolist() == [0.0] * 64


def _rn32_exact(q: Fraction) -> Fraction:
    """q rounded to the nearest fp32 value, ties to even, subnormals included (exact
    rational arithmetic, no floating point)."""
    if q == 0:
        return Fraction(0)
    s, q = (-1 if q < 0 else 1), abs(q)
    e = q.numerator.bit_length() - q.denominator.bit_length()
    if Fraction(2) ** e > q:
        e -= 1                                            # now 2^e <= q < 2^(e+1)
    ulp = Fraction(2) ** (max(e, -126) - 23)
    m = q / ulp
    k = m.numerator // m.denominator
    rem = m - k
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and k % 2 == 1):
        k += 1
    return s * k * ulp


@pytest.mark.parametrize("a_bits", [0x3F80, 0x417E, 0x7F7F, 0x0080, 0x0003, 0x4123])
def test_int8_encoder_matches_exact_rational(a_bits):
    """Every bf16 w with |w| <= a (or a 3000-sample of them) against the definition in
    exact rationals: sc = RN32(a / 127), code = clamp(round_half_even(RN32(w / sc)), +-127),
    0 when sc = 0. a = 15.875 = 127/8 makes sc = 1/8, so w = 2.5/8 and 3.5/8 are exact
    half-way cases: half-even gives 2 and 4 (half away from zero would give 3 and 4)."""
    a = float(np.array([a_bits << 16], np.uint32).view(np.float32)[0])
    xs = _all_bf16_upto(a)
    rng = np.random.default_rng(a_bits + 1)
    if xs.size > 3000:
        keep = rng.choice(xs.size, 3000, replace=False)
        xs = np.concatenate([xs[keep], np.float32([0.0, -0.0, a, -a])])
    if a == 15.875:
        xs = np.concatenate([xs, np.float32([2.5 / 8, 3.5 / 8, -2.5 / 8, 0.5 / 8, 1.5 / 8])])
    nb = (xs.size + 63) // 64
    absmax = np.full(nb, a, np.float32)
    sc = _rn32_exact(Fraction(a) / 127)
    assert Fraction(float(np.float32(a) / np.float32(127))) == sc
    codes = o.int8_encode(xs, absmax)
    for w, c in zip(xs.tolist(), codes.tolist()):
        want = 0 if sc == 0 else max(-127, min(127, round(_rn32_exact(Fraction(w) / sc))))
        assert c == want, (w, a, c, want)
    if a == 15.875:
        got = dict(zip(xs[-5:].tolist(), codes[-5:].tolist()))
        assert got == {2.5 / 8: 2, 3.5 / 8: 4, -2.5 / 8: -2, 0.5 / 8: 0, 1.5 / 8: 2}


# ---------------------------------------------------------------- bf16 rounding

def test_rn_bf16_matches_torch():
    rng = np.random.default_rng(5)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32) * 10.0 ** rng.integers(-40, 38, 20000),
        np.float32([0.0, -0.0, np.inf, -np.inf, 3.4028235e38, 1e-45, -1e-45]),
        (np.arange(0, 1 << 16, dtype=np.uint32) << 16 | 0x8000).view(np.float32)[:0x7F80],
    ]).astype(np.float32)
    x = x[np.isfinite(x) | np.isinf(x)]
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(o.f32_to_bf16_bits(x), ref)
    assert np.isnan(o.rn_bf16(np.float32([np.nan]))[0])


# ---------------------------------------------------------------- P8-P11 linear layer

def _naive_fwd(X, W, A, B, s):
    M, K = X.shape
    N, r = B.shape
    Y = np.zeros((M, N))
    T = np.zeros((M, r))
    for m in range(M):
        for j in range(r):
            T[m, j] = sum(X[m, k] * A[j, k] for k in range(K))
        for n in range(N):
            Y[m, n] = sum(X[m, k] * W[n, k] for k in range(K)) \
                + s * sum(T[m, j] * B[n, j] for j in range(r))
    return Y, T


def _tiny(seed=11, M=3, N=5, K=64, r=2):
    g = np.random.default_rng(seed)
    return (g.standard_normal((M, K)), g.standard_normal((N, K)),
            g.standard_normal((r, K)), g.standard_normal((N, r)), g.standard_normal((M, N)))


def test_forward_against_naive_loops():
    X, W, A, B, _ = _tiny()
    Y, T = o.linear_fwd(X, W, A, B, alpha=6.0, r=2)
    Yn, Tn = _naive_fwd(X, W, A, B, 3.0)
    assert np.allclose(Y, Yn, rtol=1e-12, atol=1e-12)
    assert np.allclose(T, Tn, rtol=1e-12, atol=1e-12)


def test_backward_against_finite_differences():
    """L = sum(Y * G); Y is linear in X, in A (B fixed) and in B (A fixed), so
    central differences are exact up to rounding."""
    X, W, A, B, G = _tiny()
    alpha, r = 6.0, 2
    dX, dA, dB = o.linear_bwd(X, G, W, A, B, alpha, r)

    def L(X_, A_, B_):
        return float(np.sum(o.linear_fwd(X_, W, A_, B_, alpha, r)[0] * G))

    h = 1e-3
    for (arr, grad, which) in ((X, dX, 0), (A, dA, 1), (B, dB, 2)):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            p = arr.copy(); p[idx] += h
            m = arr.copy(); m[idx] -= h
            args_p = [X, A, B]; args_p[which] = p
            args_m = [X, A, B]; args_m[which] = m
            fd[idx] = (L(*args_p) - L(*args_m)) / (2 * h)
        assert np.allclose(grad, fd, rtol=1e-7, atol=1e-7), which


def test_special_cases_B0_A0_W0():
    X, W, A, B, G = _tiny(seed=12)
    base = X @ W.T
    Y, _ = o.linear_fwd(X, W, A, np.zeros_like(B), 4.0, 2)
    assert np.array_equal(Y, base)
    dX, dA, dB = o.linear_bwd(X, G, W, A, np.zeros_like(B), 4.0, 2)
    assert np.all(dA == 0)
    Y, T = o.linear_fwd(X, W, np.zeros_like(A), B, 4.0, 2)
    assert np.array_equal(Y, base) and np.all(T == 0)
    dX, dA, dB = o.linear_bwd(X, G, W, np.zeros_like(A), B, 4.0, 2)
    assert np.all(dB == 0)
    # W = 0: every block has absmax 0, codes are 8 and W' = +0, so Y is the branch alone
    r = o.quantize_weight(np.zeros(5 * 64, np.float32), "nf4_dq")
    assert np.all(o.unpack_nibbles(r["codes"], 320) == 8)
    assert np.all(r["wdeq"].view(np.uint32) == 0)
    Y, T = o.linear_fwd(X, r["wdeq"].reshape(5, 64), A, B, 4.0, 2)
    assert np.allclose(Y, 2.0 * T @ B.T, rtol=0, atol=1e-12)


def test_forward_backward_against_torch_autograd():
    X, W, A, B, G = _tiny(seed=13, M=7, N=9, K=128, r=4)
    tX, tA, tB = (torch.tensor(v, requires_grad=True) for v in (X, A, B))
    Y = tX @ torch.tensor(W).T + 0.5 * (tX @ tA.T) @ tB.T
    (Y * torch.tensor(G)).sum().backward()
    Yo, _ = o.linear_fwd(X, W, A, B, 2.0, 4)
    dX, dA, dB = o.linear_bwd(X, G, W, A, B, 2.0, 4)
    assert np.allclose(Yo, Y.detach().numpy(), rtol=1e-12, atol=1e-12)
    for a, b in ((dX, tX.grad), (dA, tA.grad), (dB, tB.grad)):
        assert np.allclose(a, b.numpy(), rtol=1e-12, atol=1e-12)


# ---- LoRDBA double-binary adapter ----------------------------------------------------

def _lordba_case(N=24, K=40, R=6, ell=2, seed=5):
    rng = np.random.default_rng(seed)
    B1 = np.where(rng.random((N, R)) < 0.5, -1.0, 1.0)
    B2 = np.where(rng.random((R, K)) < 0.5, -1.0, 1.0)
    alpha = rng.uniform(0.1, 1.0, (ell, N))
    beta = rng.uniform(0.1, 1.0, (ell, R))
    gamma = rng.uniform(0.1, 1.0, (ell, K))
    return alpha, beta, gamma, B1, B2


def test_lordba_two_stage_sign_accumulate():
    """The page's inference kernel: gamma-scale x, accumulate with B2's signs (adds and
    subtracts only), beta-scale, accumulate with B1's signs, alpha-scale. Written as
    plain loops over Python floats, it must equal the oracle's Delta W x."""
    alpha, beta, gamma, B1, B2 = _lordba_case()
    ell, N = alpha.shape
    R, K = B2.shape
    x = np.random.default_rng(6).standard_normal(K)
    y = [0.0] * N
    for i in range(ell):
        u = []
        for j in range(R):
            acc = 0.0
            for k in range(K):
                v = gamma[i][k] * x[k]
                acc = acc + v if B2[j][k] > 0 else acc - v
            u.append(beta[i][j] * acc)
        for n in range(N):
            acc = 0.0
            for j in range(R):
                acc = acc + u[j] if B1[n][j] > 0 else acc - u[j]
            y[n] += alpha[i][n] * acc
    ref = o.lordba_delta(alpha, beta, gamma, B1, B2) @ x
    np.testing.assert_allclose(np.array(y), ref, rtol=1e-12, atol=1e-12)


def test_lordba_all_plus_carriers_closed_form():
    """B1 = B2 = all +1: Delta W[n, k] = sum_i alpha_i[n] (sum_j beta_i[j]) gamma_i[k]."""
    alpha, beta, gamma, B1, B2 = _lordba_case()
    B1 = np.ones_like(B1)
    B2 = np.ones_like(B2)
    D = o.lordba_delta(alpha, beta, gamma, B1, B2)
    want = sum(np.outer(alpha[i], gamma[i]) * beta[i].sum() for i in range(alpha.shape[0]))
    np.testing.assert_allclose(D, want, rtol=1e-13)


def test_lordba_terms_add_and_sign_flips():
    """Envelope terms add; flipping every sign of B1 (or of B2) negates Delta W; zero
    alpha (or beta, or gamma) removes the branch."""
    alpha, beta, gamma, B1, B2 = _lordba_case()
    D = o.lordba_delta(alpha, beta, gamma, B1, B2)
    D0 = o.lordba_delta(alpha[:1], beta[:1], gamma[:1], B1, B2)
    D1 = o.lordba_delta(alpha[1:], beta[1:], gamma[1:], B1, B2)
    np.testing.assert_allclose(D, D0 + D1, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(o.lordba_delta(alpha, beta, gamma, -B1, B2), -D, rtol=1e-13)
    np.testing.assert_allclose(o.lordba_delta(alpha, beta, gamma, B1, -B2), -D, rtol=1e-13)
    assert np.all(o.lordba_delta(0 * alpha, beta, gamma, B1, B2) == 0)
    # rank: with one envelope term, Delta W has rank <= R
    assert np.linalg.matrix_rank(D0) <= B1.shape[1]


def test_lordba_linear_is_base_plus_branch():
    alpha, beta, gamma, B1, B2 = _lordba_case()
    rng = np.random.default_rng(7)
    X = rng.standard_normal((5, B2.shape[1]))
    Wd = rng.standard_normal((B1.shape[0], B2.shape[1]))
    Y = o.lordba_linear_fwd(X, Wd, alpha, beta, gamma, B1, B2)
    naive = np.zeros_like(Y)
    D = o.lordba_delta(alpha, beta, gamma, B1, B2)
    for t in range(X.shape[0]):
        for n in range(Wd.shape[0]):
            naive[t, n] = sum(X[t, k] * (Wd[n, k] + D[n, k]) for k in range(X.shape[1]))
    np.testing.assert_allclose(Y, naive, rtol=1e-12)


# ---------------------------------------------------------------- QWHA adapter

def _walsh_butterflies(x, b):
    """The fast recursive Walsh-Hadamard transform of each length-b block of x, written
    as in-place butterflies of adds and subtracts (the page's fast kernel), then scaled
    by 1/sqrt(b). Plain Python floats."""
    x = [float(v) for v in x]
    for s in range(0, len(x), b):
        h = 1
        while h < b:
            for i in range(s, s + b, 2 * h):
                for j in range(i, i + h):
                    u, v = x[j], x[j + h]
                    x[j], x[j + h] = u + v, u - v
            h *= 2
    return [v / math.sqrt(b) for v in x]


def _qwha_case(N=7, K=192, seed=5):
    rng = np.random.default_rng(seed)
    cnt = rng.integers(0, 6, N)
    row_ptr = np.concatenate([[0], np.cumsum(cnt)])
    col = np.concatenate([np.sort(rng.choice(K, k, replace=False)) for k in cnt]).astype(np.int64)
    c = rng.standard_normal(int(row_ptr[-1]))
    return row_ptr, col, c


@pytest.mark.parametrize("b", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_qwha_hadamard_is_sylvester(b):
    """H for a power-of-two width is scipy's Sylvester-construction Hadamard matrix / sqrt(b)."""
    import scipy.linalg
    np.testing.assert_array_equal(o.walsh_hadamard(b) * math.sqrt(b), scipy.linalg.hadamard(b))


def test_qwha_block_structure():
    """Non-power-of-two widths: H = I (x) H_b with b the largest power of two dividing K
    (11008 = 2^8 * 43, 22016 = 2^9 * 43)."""
    import scipy.linalg
    assert [o.wht_block_size(K) for K in (4096, 8192, 11008, 22016, 192)] == [4096, 8192, 256, 512, 64]
    want = np.kron(np.eye(3), scipy.linalg.hadamard(64) / 8.0)
    np.testing.assert_array_equal(o.walsh_hadamard(192), want)


def test_qwha_H_is_orthogonal_and_inverts():
    H = o.walsh_hadamard(96)
    np.testing.assert_allclose(H @ H.T, np.eye(96), atol=1e-14)
    np.testing.assert_allclose(np.linalg.inv(H), H.T, atol=1e-13)


def test_qwha_single_coefficient_is_a_walsh_function():
    """One value c at (n, k): row n of Delta W = F H^{-1} is c times the Walsh function
    j -> (-1)^popcount(k & j) / sqrt(b) on the block holding k, zero elsewhere; every
    other row is zero."""
    N, K, n, k, c = 4, 192, 2, 77, 0.375
    row_ptr = [0, 0, 0, 1, 1]
    D = o.qwha_delta(N, K, row_ptr, [k], [c])
    b = 64
    want = np.zeros((N, K))
    s = (k // b) * b
    for j in range(s, s + b):
        want[n, j] = c * (-1) ** bin((k - s) & (j - s)).count("1") / math.sqrt(b)
    np.testing.assert_allclose(D, want, rtol=0, atol=1e-15)


@pytest.mark.parametrize("K", [64, 128, 192])
def test_qwha_transform_equals_butterflies_and_keeps_norms(K):
    """Z = H^{-1} x per token equals the add/subtract recursion, and the orthonormal
    transform keeps each block's Euclidean norm."""
    rng = np.random.default_rng(K)
    X = rng.standard_normal((3, K))
    Z = o.qwha_transform(X)
    b = o.wht_block_size(K)
    for t in range(3):
        np.testing.assert_allclose(Z[t], _walsh_butterflies(X[t], b), rtol=0, atol=1e-12)
        for s in range(0, K, b):
            assert math.isclose(np.linalg.norm(Z[t, s:s + b]), np.linalg.norm(X[t, s:s + b]), rel_tol=1e-13)


def test_qwha_linear_as_sparse_gather_of_the_transformed_input():
    """Y = X Wd^T + X (F H^{-1})^T equals the page's association Delta W x = F (H^{-1} x):
    the butterfly transform of x, then for every stored value c at (n, k) an add of
    c * z_k into y_n (loops)."""
    N, K = 7, 192
    row_ptr, col, c = _qwha_case(N, K)
    rng = np.random.default_rng(11)
    X = rng.standard_normal((4, K))
    Wd = rng.standard_normal((N, K))
    Y = o.qwha_linear_fwd(X, Wd, row_ptr, col, c)
    for t in range(4):
        z = _walsh_butterflies(X[t], o.wht_block_size(K))
        for n in range(N):
            y = sum(X[t, k] * Wd[n, k] for k in range(K))
            for j in range(row_ptr[n], row_ptr[n + 1]):
                y += c[j] * z[col[j]]
            assert math.isclose(Y[t, n], y, rel_tol=1e-11, abs_tol=1e-11)
    # the factored form (block transform, then the sparse product) is the same Y
    np.testing.assert_allclose(o.qwha_linear_fwd_factored(X, Wd, row_ptr, col, c), Y, rtol=1e-12, atol=1e-12)


def test_qwha_block_transform_equals_full_matrix():
    """The transform taken one diagonal block at a time equals the product with the full
    K x K matrix, for a width with 7 blocks."""
    rng = np.random.default_rng(2)
    X = rng.standard_normal((3, 448))
    np.testing.assert_allclose(o.qwha_transform(X), X @ np.linalg.inv(o.walsh_hadamard(448)).T,
                               rtol=0, atol=1e-12)


def test_qwha_zero_and_linear_in_c():
    N, K = 7, 192
    row_ptr, col, c = _qwha_case(N, K)
    rng = np.random.default_rng(3)
    X = rng.standard_normal((2, K))
    Wd = rng.standard_normal((N, K))
    np.testing.assert_allclose(o.qwha_linear_fwd(X, Wd, row_ptr, col, 0 * c), X @ Wd.T, rtol=1e-13)
    D1 = o.qwha_delta(N, K, row_ptr, col, c)
    D2 = o.qwha_delta(N, K, row_ptr, col, -2.5 * c)
    np.testing.assert_allclose(D2, -2.5 * D1, rtol=1e-13, atol=1e-15)


def _qwha_bwd_case(N=7, K=192, M=5, seed=5):
    row_ptr, col, c = _qwha_case(N, K, seed)
    rng = np.random.default_rng(seed + 100)
    return (rng.standard_normal((M, K)), rng.standard_normal((M, N)), rng.standard_normal((N, K)),
            row_ptr, col, c)


def test_qwha_backward_matches_torch_autograd():
    """dX and dc equal torch's fp64 autograd of sum(dY * Y), with F scattered from c by
    torch, H built from scipy's Sylvester matrix block by block, and its inverse taken by
    torch.linalg.inv."""
    import scipy.linalg
    X, dY, Wd, row_ptr, col, c = _qwha_bwd_case()
    N, K = Wd.shape
    b = 64                                            # 192 = 3 * 64
    H = torch.block_diag(*[torch.tensor(scipy.linalg.hadamard(b) / math.sqrt(b))] * (K // b))
    rows = torch.repeat_interleave(torch.arange(N), torch.tensor(np.diff(row_ptr)))
    Xt = torch.tensor(X, requires_grad=True)
    ct = torch.tensor(c, requires_grad=True)
    F = torch.zeros((N, K), dtype=torch.float64).index_put((rows, torch.tensor(col)), ct)
    Y = Xt @ torch.tensor(Wd).T + Xt @ (F @ torch.linalg.inv(H)).T
    (Y * torch.tensor(dY)).sum().backward()
    dX, dc = o.qwha_linear_bwd(X, dY, Wd, row_ptr, col, c)
    np.testing.assert_allclose(dX, Xt.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dc, ct.grad.numpy(), rtol=1e-12, atol=1e-12)


def test_qwha_backward_central_differences():
    """Y is linear in X and in c, so a central difference of sum(dY * Y) with a unit step
    is the exact derivative up to rounding: checked for every value c_j and a spread of
    entries of X."""
    X, dY, Wd, row_ptr, col, c = _qwha_bwd_case(N=5, K=128, M=3, seed=9)
    dX, dc = o.qwha_linear_bwd(X, dY, Wd, row_ptr, col, c)
    L = lambda Xv, cv: float(np.sum(dY * o.qwha_linear_fwd(Xv, Wd, row_ptr, col, cv)))
    for j in range(c.size):
        e = np.zeros_like(c)
        e[j] = 1.0
        assert math.isclose((L(X, c + e) - L(X, c - e)) / 2, dc[j], rel_tol=1e-9, abs_tol=1e-9)
    for m, k in [(0, 0), (1, 37), (2, 127), (0, 64), (2, 90)]:
        E = np.zeros_like(X)
        E[m, k] = 1.0
        assert math.isclose((L(X + E, c) - L(X - E, c)) / 2, dX[m, k], rel_tol=1e-9, abs_tol=1e-9)


def test_qwha_backward_adjoint_identities():
    """The adapter branch A(X, c) = X Delta W^T is bilinear, so Euler's identity fixes
    both gradients against the forward: <dc, c> = <dY, A> and <dX - dY Wd, X> = <dY, A>."""
    X, dY, Wd, row_ptr, col, c = _qwha_bwd_case(N=9, K=448, M=4, seed=13)
    dX, dc = o.qwha_linear_bwd(X, dY, Wd, row_ptr, col, c)
    A = o.qwha_linear_fwd(X, Wd, row_ptr, col, c) - X @ Wd.T
    pair = float(np.sum(dY * A))
    assert math.isclose(float(dc @ c), pair, rel_tol=1e-11)
    assert math.isclose(float(np.sum((dX - dY @ Wd) * X)), pair, rel_tol=1e-11)


def test_qwha_backward_single_coefficient_is_a_walsh_correlation():
    """One value at (n, k): dc = sum over tokens m and block columns j of
    dY[m, n] X[m, j] (-1)^popcount((k - s) & (j - s)) / sqrt(b), s the start of k's
    block; and the adapter's part of dX is dY[:, n] c times that Walsh function (loops)."""
    N, K, n, k, cv = 4, 192, 2, 77, 0.625
    rng = np.random.default_rng(17)
    X, dY, Wd = rng.standard_normal((3, K)), rng.standard_normal((3, N)), rng.standard_normal((N, K))
    dX, dc = o.qwha_linear_bwd(X, dY, Wd, [0, 0, 0, 1, 1], [k], [cv])
    b, s = 64, 64
    walsh = lambda j: (-1) ** bin((k - s) & (j - s)).count("1") / math.sqrt(b)
    want = sum(dY[m, n] * X[m, j] * walsh(j) for m in range(3) for j in range(s, s + b))
    assert math.isclose(dc[0], want, rel_tol=1e-12)
    for m in range(3):
        for j in range(K):
            ad = dY[m, n] * cv * walsh(j) if s <= j < s + b else 0.0
            assert math.isclose(dX[m, j] - float(dY[m] @ Wd[:, j]), ad, abs_tol=1e-12)


@pytest.mark.parametrize("K", [192, 256, 448])
def test_qwha_backward_factored_equals_dense(K):
    X, dY, Wd, row_ptr, col, c = _qwha_bwd_case(N=11, K=K, M=6, seed=K)
    dX, dc = o.qwha_linear_bwd(X, dY, Wd, row_ptr, col, c)
    fX, fc = o.qwha_linear_bwd_factored(X, dY, Wd, row_ptr, col, c, chunk=7)
    np.testing.assert_allclose(fX, dX, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(fc, dc, rtol=1e-12, atol=1e-12)


def test_qwha_backward_empty_and_zero():
    """No stored values: dc is empty and dX is the base's dY Wd. c = 0: dX is the base's
    and dc is unchanged (it does not depend on c)."""
    X, dY, Wd, row_ptr, col, c = _qwha_bwd_case(seed=21)
    N = Wd.shape[0]
    dX0, dc0 = o.qwha_linear_bwd(X, dY, Wd, np.zeros(N + 1, np.int64), np.zeros(0, np.int64), np.zeros(0))
    assert dc0.shape == (0,)
    np.testing.assert_allclose(dX0, dY @ Wd, rtol=1e-13)
    dX, dc = o.qwha_linear_bwd(X, dY, Wd, row_ptr, col, c)
    dXz, dcz = o.qwha_linear_bwd(X, dY, Wd, row_ptr, col, 0 * c)
    np.testing.assert_allclose(dXz, dY @ Wd, rtol=1e-13)
    np.testing.assert_array_equal(dcz, dc)


# ---------------------------------------------------------------- AdamW step (paged states)

def test_adamw_matches_torch_over_several_steps():
    """The oracle's step equals torch.optim.AdamW (fp64) over six steps with weight decay
    and a gradient scale folded into the gradient."""
    rng = np.random.default_rng(21)
    n = 257
    theta0 = rng.standard_normal(n) * 0.05
    hp = dict(lr=2e-3, beta1=0.9, beta2=0.995, eps=1e-8, weight_decay=0.05)
    p = torch.nn.Parameter(torch.tensor(theta0, dtype=torch.float64))
    opt = torch.optim.AdamW([p], lr=hp["lr"], betas=(hp["beta1"], hp["beta2"]), eps=hp["eps"],
                            weight_decay=hp["weight_decay"])
    theta, m, v = theta0.copy(), np.zeros(n), np.zeros(n)
    for t in range(1, 7):
        g = rng.standard_normal(n)
        p.grad = torch.tensor(g * 0.5, dtype=torch.float64)
        opt.step()
        theta, m, v, bits = o.adamw_step(theta, g, m, v, t, grad_scale=0.5, **hp)
        np.testing.assert_allclose(theta, p.detach().numpy(), rtol=1e-13, atol=1e-15)
        st = opt.state[p]
        np.testing.assert_allclose(m, st["exp_avg"].numpy(), rtol=1e-13, atol=1e-16)
        np.testing.assert_allclose(v, st["exp_avg_sq"].numpy(), rtol=1e-13, atol=1e-18)
    assert np.array_equal(bits, o.f32_to_bf16_bits(theta.astype(np.float32)))


def test_adamw_first_step_closed_form():
    """Step 1 without weight decay: m_hat = g and v_hat = g^2, so the update is
    -lr g / (|g| + eps), a step of lr against the sign of g."""
    g = np.array([3.0, -0.25, 1e-3, -7.5])
    lr, eps = 1e-2, 1e-8
    theta, m, v, _ = o.adamw_step(np.zeros(4), g, np.zeros(4), np.zeros(4), 1, lr, 0.9, 0.999, eps, 0.0)
    np.testing.assert_allclose(theta, -lr * g / (np.abs(g) + eps), rtol=1e-14)
    np.testing.assert_allclose(m, 0.1 * g, rtol=1e-15)
    np.testing.assert_allclose(v, 0.001 * g * g, rtol=1e-14)


def test_adamw_zero_gradient_only_decays():
    """g = 0: the moments decay by beta1 and beta2 and, without weight decay, theta moves by
    the remaining momentum alone; with m = 0 too it stays where it is except for decay."""
    theta0 = np.array([0.5, -1.0])
    theta, m, v, _ = o.adamw_step(theta0, np.zeros(2), np.zeros(2), np.zeros(2), 3, 1e-3, 0.9, 0.99, 1e-8, 0.1)
    np.testing.assert_allclose(theta, theta0 * (1 - 1e-4), rtol=1e-15)
    assert np.all(m == 0) and np.all(v == 0)


# ---------------------------------------------------------------- Lion with INT8 momentum

def _lion_case(n=300, seed=4):
    rng = np.random.default_rng(seed)
    th = (rng.standard_normal(n) * 0.02).astype(np.float32)
    g = (rng.standard_normal(n) * 1e-3).astype(np.float32)
    m_exact = (rng.standard_normal(n) * 1e-4).astype(np.float32)
    codes, am = o.int8_quantize(m_exact)
    return th, g, codes, am


def test_lion_first_step_closed_form():
    """From a zero momentum: c = (1 - beta1) g, so theta' = RN32(theta decay) - lr sign(g),
    and the new momentum is the blockwise INT8 code of RN32((1 - beta2) g)."""
    th, g, _, _ = _lion_case()
    n = th.size
    lr, wd = 1e-4, 0.1
    t2, c2, a2, _ = o.lion_int8_step(th, g, np.zeros(n, np.int8), np.zeros(5, np.float32), lr, 0.9, 0.99, wd)
    decay = np.float32(np.float32(1) - np.float32(np.float32(lr) * np.float32(wd)))
    want = (th * decay).astype(np.float32) - np.float32(lr) * np.sign(g).astype(np.float32)
    assert np.array_equal(t2, want.astype(np.float32))
    m_new = (np.float32(np.float32(1) - np.float32(0.99)) * g).astype(np.float32)
    c_ref, a_ref = o.int8_quantize(m_new)
    assert np.array_equal(c2, c_ref) and np.array_equal(a2, a_ref)


def test_lion_update_size_is_fixed():
    """Without weight decay every element moves by lr (the sign update's fixed size, the
    property the page relies on), up to one fp32 rounding of theta, against the direction
    of c computed independently in fp64."""
    th, g, codes, am = _lion_case()
    lr = 3e-4
    t2, _, _, _ = o.lion_int8_step(th, g, codes, am, lr, 0.9, 0.99, 0.0)
    m = codes.astype(np.float64) * (am.astype(np.float64) / 127.0)[np.arange(th.size) // 64]
    c64 = 0.9 * m + 0.1 * g.astype(np.float64)
    sure = np.abs(c64) > 1e-9
    step = t2.astype(np.float64) - th.astype(np.float64)
    # one rounding of theta' (at the larger of |theta|, |theta'|), against lr as an fp32
    ulp = np.spacing(np.maximum(np.abs(th), np.abs(t2))).astype(np.float64)
    lr32 = float(np.float32(lr))
    assert np.all(np.abs(np.abs(step[sure]) - lr32) <= ulp[sure])
    assert np.all(np.sign(step[sure]) == -np.sign(c64[sure]))


def test_lion_momentum_round_trip_bound():
    """The stored momentum is within half a code step of the exact new momentum, and each
    block's largest element is stored as +-127."""
    th, g, codes, am = _lion_case(n=640)
    b1, b2 = 0.9, 0.95
    _, c2, a2, _ = o.lion_int8_step(th, g, codes, am, 1e-4, b1, b2, 0.0)
    blk = np.arange(th.size) // 64
    m = codes.astype(np.float64) * (am.astype(np.float64) / 127.0)[blk]
    m_new = b2 * m + (1 - b2) * g.astype(np.float64)
    step = (a2.astype(np.float64) / 127.0)[blk]
    got = c2.astype(np.float64) * step
    assert np.all(np.abs(got - m_new) <= 0.5 * step * (1 + 1e-5) + 1e-12)
    for b in range(a2.size):
        assert np.max(np.abs(c2[blk == b])) == 127
