"""CPU oracle for the QLoRA-style quantised linear layer.

TEST INFRASTRUCTURE ONLY. Only the test suite, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this module.
The product path (the CUDA library and its Python binding) never imports it, and this
module imports nothing from the product package.

It is a plain, slow, obviously correct restatement of what the method computes:

* NF4 blockwise quantisation of a bf16 weight
  (QLoRA page, aizip.shop/methodologies/qlora, section "1. 4-bit NormalFloat (NF4)").
* Double quantisation of the absmax constants
  (same page, section "2. Double Quantization").
* Blockwise int8, the 8-bit alternative format of the per-layer bit-width choice
  (AutoQRA page, gist.science/ko/paper/2602.22268, section 3.1; QFT page,
  gist.science/ko/paper/2310.07147, section 2.2 "dense INT8 part").
* The unmerged adapter linear Y = X deq(W)^T + (alpha/r) (X A^T) B^T and its
  gradients, computed in fp64 (QLoRA page, section "memory decomposition": frozen
  4-bit base plus bf16 LoRA adapters; LoRDBA page, gist.science/ko/paper/2605.24058,
  "adapter mode", for the unmerged branch).
* The low-rank double-binary adapter of the LoRDBA page (section "2. Methodology",
  core architecture): Delta W = sum_i diag(alpha_i) B1 diag(beta_i) B2 diag(gamma_i)
  with sign carriers B1, B2 in {+-1}, in fp64.
* The Walsh-Hadamard adapter of the QWHA page (gist.science/ko/paper/2509.17428,
  section 2.1): Delta W = F H^{-1} with a sparse coefficient matrix F and the
  Walsh-Hadamard matrix H, in fp64.
* The adapter optimiser step whose states the QLoRA page pages to host memory (section
  "3. Paged Optimizer"): AdamW on the flat adapter vector, in fp64.
* The Lion step with INT8 momentum of the QFT page (section 2.1), in fp32 one operation
  at a time, since the new momentum codes are integer decisions.

Where the pages are silent the reading taken is stated in the docstring of the
function that takes it. Floating-point steps are written with numpy float32 scalars
/ arrays, whose +, -, *, / are single IEEE operations rounded to nearest even (numpy
never contracts them into FMAs), so ``RN32(a op b)`` below is literally ``a op b``
on float32 operands. Matrix products use numpy float64 matmul.

Notation: RN32 = round to nearest-even fp32, RNbf = round to nearest-even bf16,
n = number of weight elements, block = 64 consecutive elements of the row-major
flattening, group = 256 consecutive blocks.
"""
from __future__ import annotations

import functools
import math
import statistics

import numpy as np

BLOCK = 64          # QLoRA page, "2. Double Quantization": block size 64
DQ_GROUP = 256      # blocks per double-quantisation group
NF4_BITS = 4        # QLoRA page, "1. NF4": b = 4 gives 16 grid points
INT8_QMAX = 127     # symmetric int8 range used for every 8-bit code here


# --------------------------------------------------------------------------------------
# bf16 helpers (storage conversions, written out bit by bit)
# --------------------------------------------------------------------------------------

def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to the fp32 values they denote (exact)."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """RNbf: round fp32 to the nearest bf16, ties to even; NaN stays a quiet NaN.

    Written from the definition: keep the top 16 bits, and add one unit in the last
    kept place when the dropped 16 bits exceed half a unit, or equal it and the kept
    part is odd. A carry into the exponent is the correct rounding up (it also turns
    the largest values into infinity, as round-to-nearest requires).
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    keep = u >> np.uint64(16)
    drop = u & np.uint64(0xFFFF)
    half = np.uint64(0x8000)
    round_up = (drop > half) | ((drop == half) & ((keep & np.uint64(1)) == np.uint64(1)))
    out = (keep + round_up.astype(np.uint64)).astype(np.uint32)
    nan = np.isnan(x)
    out = np.where(nan, (keep | np.uint64(0x40)).astype(np.uint32), out)
    return out.astype(np.uint16)


def rn_bf16(x: np.ndarray) -> np.ndarray:
    """RNbf as fp32 values (the bf16 result widened back, exactly)."""
    return bf16_bits_to_f32(f32_to_bf16_bits(x))


# --------------------------------------------------------------------------------------
# NF4 codebook (QLoRA page, section "1. 4-bit NormalFloat (NF4)")
# --------------------------------------------------------------------------------------

def normal_quantile(p: float) -> float:
    """Q_N(p): inverse CDF of the standard normal, in fp64.

    Python's ``statistics.NormalDist.inv_cdf`` implements Wichura's algorithm AS241
    (Applied Statistics 37(3), 1988), accurate to about 1e-16 relative.
    """
    return statistics.NormalDist().inv_cdf(p)


def nf4_codebook() -> np.ndarray:
    """The 16 NF4 grid points q_0 < ... < q_15 as fp32.

    The page defines the grid by quantiles of N(0, 1) at equal-probability points,
    q_i = Q_N(p_i), i = 0..2^b - 1, with b = 4. The printed p_i = (i - 1/2)/2^b is
    undefined at i = 0 (Q_N of a negative probability); the reading taken is the
    centred form p_i = (i + 1/2)/16, the midpoints of 16 equal-mass bins. The grid
    is then normalised so that max |q| = 1 (the block absmax maps to +-1), and each
    point is rounded once to fp32: q_i = RN32(Q_N((i + 1/2)/16) / Q_N(31/32)).
    """
    scale = normal_quantile(31.0 / 32.0)
    pts = [normal_quantile((i + 0.5) / 16.0) / scale for i in range(2 ** NF4_BITS)]
    return np.array(pts, dtype=np.float64).astype(np.float32)


def nf4_midpoints() -> np.ndarray:
    """m_j = (q_j + q_{j+1}) / 2 for j = 0..14, exact, as fp64.

    Two fp32 values with exponents this close add exactly in fp64, and halving is
    exact, so these are the exact decision points of "nearest grid point".
    """
    q = nf4_codebook().astype(np.float64)
    return (q[:-1] + q[1:]) / 2.0


# --------------------------------------------------------------------------------------
# Blockwise absmax + NF4 encode (QLoRA page, sections "1. NF4" and "2. Double
# Quantization": quantisation constants per block of 64)
# --------------------------------------------------------------------------------------

def num_blocks(n: int) -> int:
    return (n + BLOCK - 1) // BLOCK


def _blocks(x: np.ndarray, fill=0) -> np.ndarray:
    """View a flat array as [nblocks, 64], padding a partial last block with ``fill``."""
    nb = num_blocks(x.size)
    if x.size == nb * BLOCK:
        return x.reshape(nb, BLOCK)
    pad = np.full(nb * BLOCK - x.size, fill, dtype=x.dtype)
    return np.concatenate([x, pad]).reshape(nb, BLOCK)


def block_absmax(w: np.ndarray) -> np.ndarray:
    """a_b = max_{j in block b} |w_j| over blocks of 64 consecutive elements, fp32.

    ``w`` holds bf16 values as fp32 (flattened row-major). A partial last block takes
    the max over the elements it has (padding with 0 does not change a max of |w|).
    The max of exact values is exact.
    """
    w = np.asarray(w, dtype=np.float32).ravel()
    if w.size == 0:
        return np.zeros(0, np.float32)
    return np.max(np.abs(_blocks(w)), axis=1).astype(np.float32)


def nf4_encode(w: np.ndarray, absmax: np.ndarray) -> np.ndarray:
    """NF4 code of every element: the index of the grid point nearest to w / a_b.

    Reading taken (the pages say "nearest quantile point" without a precision):
    the decision is exact. For a_b > 0 the nearest point to the real number w/a_b
    is found with the grid's exact midpoints, code = #{ j : w/a_b >= m_j }, so a
    value exactly halfway between two points takes the upper one. The test
    w/a_b >= m_j is evaluated as w >= a_b * m_j in fp64, which is exact: a_b has at
    most 8 significant bits (a bf16 value), m_j at most 26, so the product fits in
    fp64's 53 bits and cannot underflow or overflow. For a_b = 0 the block is all
    zeros, w/a_b is taken as 0, and 0 sits exactly between q_7 and q_8, so code 8.
    Returns one uint8 code (0..15) per element, not yet packed.
    """
    w = np.asarray(w, dtype=np.float32).ravel()
    absmax = np.asarray(absmax, dtype=np.float32)
    n = w.size
    m = nf4_midpoints()
    wb = _blocks(w)
    codes = np.empty(wb.shape, dtype=np.uint8)
    step = 1 << 16                                     # blocks per chunk (memory bound)
    for b0 in range(0, wb.shape[0], step):
        seg = wb[b0:b0 + step].astype(np.float64)
        a = absmax[b0:b0 + step].astype(np.float64)[:, None]
        cnt = np.zeros(seg.shape, dtype=np.uint8)
        for j in range(m.size):
            cnt += seg >= a * m[j]                      # exact, see docstring
        cnt[a[:, 0] == 0.0, :] = 8
        codes[b0:b0 + step] = cnt
    return codes.ravel()[:n]


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Two 4-bit codes per byte: element 2j in the low nibble of byte j, element
    2j+1 in the high nibble (the pages fix no nibble order; this is the reading).
    An odd count leaves the last high nibble 0."""
    codes = np.asarray(codes, dtype=np.uint8).ravel()
    if codes.size % 2:
        codes = np.concatenate([codes, np.zeros(1, np.uint8)])
    lo = codes[0::2] & np.uint8(0xF)
    hi = codes[1::2] & np.uint8(0xF)
    return (lo | (hi << np.uint8(4))).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray, n: int) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8).ravel()
    out = np.empty(packed.size * 2, dtype=np.uint8)
    out[0::2] = packed & np.uint8(0xF)
    out[1::2] = packed >> np.uint8(4)
    return out[:n]


def nf4_quantize(w: np.ndarray):
    """Blockwise NF4 of a bf16 weight (values as fp32): (packed codes, fp32 absmax)."""
    a = block_absmax(w)
    return pack_nibbles(nf4_encode(w, a)), a


# --------------------------------------------------------------------------------------
# Double quantisation (QLoRA page, section "2. Double Quantization")
# --------------------------------------------------------------------------------------

def dq_mean(absmax: np.ndarray) -> np.float32:
    """mu = mean of all absmax constants of the tensor, fp32.

    Readings taken: one mean per tensor (storing one fp32 per group of 256 is what
    gives 4 + 8/64 + 32/(64*256) ~= 4.127 bits per parameter); the sum is the exact
    sum rounded once to fp64 (``math.fsum``), divided by the count in fp64, then
    rounded to fp32. An exact sum makes the result independent of summation order.
    """
    absmax = np.asarray(absmax, dtype=np.float32)
    s = math.fsum(float(v) for v in absmax)
    return np.float32(s / absmax.size)


def dq_encode(absmax: np.ndarray):
    """Re-quantise the fp32 absmax constants to int8 in groups of 256.

    Per group g: d_b = RN32(a_b - mu); s_g = RN32(max_b |d_b| / 127);
    c_b = clamp(round_half_even(RN32(d_b / s_g)), -127, 127), and c_b = 0 when
    s_g = 0. Readings taken: symmetric int8 range +-127 and round-half-even.
    Returns (int8 codes [nblocks], fp32 group scales [ceil(nblocks/256)], fp32 mu).
    """
    absmax = np.asarray(absmax, dtype=np.float32)
    nb = absmax.size
    mu = dq_mean(absmax)
    ng = (nb + DQ_GROUP - 1) // DQ_GROUP
    d = absmax - mu                                          # fp32, RN, per block
    dpad = np.concatenate([d, np.zeros(ng * DQ_GROUP - nb, np.float32)])
    scales = (np.max(np.abs(dpad.reshape(ng, DQ_GROUP)), axis=1)
              / np.float32(INT8_QMAX)).astype(np.float32)    # fp32, RN, per group
    s_b = scales[np.arange(nb) // DQ_GROUP]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.rint(d / s_b)                                 # fp32 divide, half-even
    q = np.where(s_b == 0, 0, np.clip(t, -INT8_QMAX, INT8_QMAX)).astype(np.int8)
    return q, scales, mu


def dq_decode(qabsmax: np.ndarray, scales: np.ndarray, mu) -> np.ndarray:
    """a'_b = RN32(RN32(c_b * s_g) + mu), two separately rounded steps."""
    qabsmax = np.asarray(qabsmax, dtype=np.int8)
    g = np.arange(qabsmax.size) // DQ_GROUP
    prod = qabsmax.astype(np.float32) * np.asarray(scales, np.float32)[g]
    return (prod + np.float32(mu)).astype(np.float32)


def nf4_dequant(packed: np.ndarray, absmax_rec: np.ndarray, n: int) -> np.ndarray:
    """w'_j = RNbf(RN32(q[code_j] * a'_b)), returned as fp32 holding bf16 values."""
    codes = unpack_nibbles(packed, n)
    q = nf4_codebook()
    b = np.arange(n) // BLOCK
    prod = q[codes] * np.asarray(absmax_rec, np.float32)[b]
    return rn_bf16(prod)


# --------------------------------------------------------------------------------------
# Blockwise int8 (AutoQRA page, section 3.1: the per-layer bit-width q_l; QFT page,
# section 2.2: a dense INT8 weight with per-block scale)
# --------------------------------------------------------------------------------------

def int8_encode(w: np.ndarray, absmax: np.ndarray) -> np.ndarray:
    """c_j = clamp(round_half_even(RN32(w_j / sc_b)), -127, 127), sc_b = RN32(a_b/127);
    c_j = 0 when sc_b = 0. Reading taken: the plainest absmax-linear 8-bit code, shaped
    like NF4 (code times a per-block scale); the stored constant is a_b itself (fp32)."""
    w = np.asarray(w, dtype=np.float32).ravel()
    absmax = np.asarray(absmax, dtype=np.float32)
    sc = (absmax / np.float32(INT8_QMAX)).astype(np.float32)       # fp32, RN
    s_j = sc[np.arange(w.size) // BLOCK]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.rint(w / s_j)                                       # fp32 divide, half-even
    return np.where(s_j == 0, 0, np.clip(t, -INT8_QMAX, INT8_QMAX)).astype(np.int8)


def int8_quantize(w: np.ndarray):
    a = block_absmax(w)
    return int8_encode(w, a), a


def int8_dequant(codes: np.ndarray, absmax: np.ndarray) -> np.ndarray:
    """w'_j = RNbf(RN32(c_j * RN32(a_b / 127)))."""
    codes = np.asarray(codes, dtype=np.int8).ravel()
    sc = np.asarray(absmax, np.float32) / np.float32(INT8_QMAX)
    b = np.arange(codes.size) // BLOCK
    return rn_bf16(codes.astype(np.float32) * sc[b])


# --------------------------------------------------------------------------------------
# Storage accounting (QLoRA page, "2. Double Quantization" and "memory decomposition")
# --------------------------------------------------------------------------------------

def storage_bytes(fmt: str, n: int) -> dict:
    """Bytes of every stored array for n parameters."""
    nb = num_blocks(n)
    if fmt == "nf4_dq":
        return {"codes": (n + 1) // 2, "qabsmax": nb,
                "group_scale": 4 * ((nb + DQ_GROUP - 1) // DQ_GROUP), "mean": 4}
    if fmt == "int8":
        return {"codes": n, "absmax": 4 * nb}
    raise ValueError(fmt)


# --------------------------------------------------------------------------------------
# The linear layer with an unmerged LoRA branch, fp64 (QLoRA page, "memory
# decomposition": NF4 base + bf16 adapters; AutoQRA page section 1: frozen quantised
# backbone, adapters trained)
# --------------------------------------------------------------------------------------

def linear_fwd(X, Wd, A, B, alpha: float, r: int):
    """T = X A^T;  Y = X Wd^T + s T B^T,  s = alpha / r.  All in fp64.

    X [M,K], Wd [N,K] (the dequantised weight), A [r,K], B [N,r]. Returns (Y, T).
    """
    X = np.asarray(X, np.float64)
    Wd = np.asarray(Wd, np.float64)
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    s = alpha / r
    T = X @ A.T
    Y = X @ Wd.T + s * (T @ B.T)
    return Y, T


def adapter_grads(X, dY, A, B, alpha: float, r: int):
    """The adapter gradients alone, fp64: dA = s U^T X and dB = s dY^T T, with
    U = dY B and T = X A^T. They need no weight, so large layers can be checked in full
    without the dX product."""
    X = np.asarray(X, np.float64)
    dY = np.asarray(dY, np.float64)
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    s = alpha / r
    T = X @ A.T
    U = dY @ B
    return s * (U.T @ X), s * (dY.T @ T)


def linear_bwd(X, dY, Wd, A, B, alpha: float, r: int):
    """Gradients of Y = X Wd^T + s (X A^T) B^T with Wd frozen, fp64.

    U = dY B;  dX = dY Wd + s U A;  dA = s U^T X;  dB = s dY^T T  (T = X A^T).
    Returns (dX, dA, dB). dX of a subset of rows needs only those rows of dY.
    """
    dY = np.asarray(dY, np.float64)
    Wd = np.asarray(Wd, np.float64)
    A = np.asarray(A, np.float64)
    B = np.asarray(B, np.float64)
    s = alpha / r
    U = dY @ B
    dX = dY @ Wd + s * (U @ A)
    dA, dB = adapter_grads(X, dY, A, B, alpha, r)
    return dX, dA, dB


def quantize_weight(w: np.ndarray, fmt: str):
    """Full quantise of one weight in format ``fmt`` ('nf4_dq' or 'int8'), returning a
    dict of the stored arrays and the dequantised weight W' (fp32 holding bf16)."""
    w = np.asarray(w, dtype=np.float32).ravel()
    n = w.size
    if fmt == "nf4_dq":
        packed, a = nf4_quantize(w)
        qa, sc, mu = dq_encode(a)
        wd = nf4_dequant(packed, dq_decode(qa, sc, mu), n)
        return {"codes": packed, "absmax": a, "qabsmax": qa, "group_scale": sc,
                "mean": mu, "wdeq": wd}
    if fmt == "int8":
        c, a = int8_quantize(w)
        return {"codes": c, "absmax": a, "wdeq": int8_dequant(c, a)}
    raise ValueError(fmt)


# --------------------------------------------------------------------------------------
# LoRDBA: low-rank double-binary adapter (LoRDBA page, gist.science/ko/paper/2605.24058,
# section "2. Methodology", core architecture: the parameterisation, 1-bit carriers and
# fp16 channel scales, and the two-stage sign-accumulate inference kernel)
# --------------------------------------------------------------------------------------

def lordba_delta(alpha, beta, gamma, B1, B2):
    """Delta W = sum_{i < l} diag(alpha[i]) B1 diag(beta[i]) B2 diag(gamma[i]), fp64.

    B1 [N, R] and B2 [R, K] hold +-1 (the carriers are shared by the l envelope terms;
    only the scale vectors carry the index i). alpha [l, N], beta [l, R], gamma [l, K]
    are the channel scales. Returns Delta W [N, K], the update to the frozen weight
    [out, in]."""
    B1 = np.asarray(B1, np.float64)
    B2 = np.asarray(B2, np.float64)
    alpha = np.atleast_2d(np.asarray(alpha, np.float64))
    beta = np.atleast_2d(np.asarray(beta, np.float64))
    gamma = np.atleast_2d(np.asarray(gamma, np.float64))
    assert set(np.unique(B1)) <= {-1.0, 1.0} and set(np.unique(B2)) <= {-1.0, 1.0}
    D = np.zeros((B1.shape[0], B2.shape[1]))
    for i in range(alpha.shape[0]):
        D += (alpha[i][:, None] * B1 * beta[i][None, :]) @ (B2 * gamma[i][None, :])
    return D


def lordba_linear_fwd(X, Wd, alpha, beta, gamma, B1, B2):
    """Y = X Wd^T + X Delta W^T in fp64: the frozen (dequantised) base plus the unmerged
    double-binary adapter branch (the page's "adapter mode")."""
    X = np.asarray(X, np.float64)
    Wd = np.asarray(Wd, np.float64)
    return X @ Wd.T + X @ lordba_delta(alpha, beta, gamma, B1, B2).T


# --------------------------------------------------------------------------------------
# QWHA: Walsh-Hadamard adapter (QWHA page, gist.science/ko/paper/2509.17428, section
# "2.1 Adapter design: Walsh-Hadamard adaptation"): Delta W = F H^{-1} with a sparse
# coefficient matrix F (values c at the positions of an index list E) and the
# predefined Walsh-Hadamard transform H
# --------------------------------------------------------------------------------------

def wht_block_size(K: int) -> int:
    """Order of the Walsh-Hadamard blocks of H for an input width K.

    Reading: a Walsh-Hadamard matrix exists only for power-of-two orders and the page
    does not say what H is when K is not one (LLaMA's 11008 and 22016 are 2^8 * 43 and
    2^9 * 43). H is taken as the block-diagonal matrix whose blocks are the Walsh-Hadamard
    matrix of the largest power of two dividing K, which keeps Delta W = F H^{-1} a K x K
    product; for a power-of-two K it is the single full-width transform."""
    assert K >= 1
    return K & (-K)


@functools.lru_cache(maxsize=4)
def walsh_hadamard_block(b: int) -> np.ndarray:
    """One Walsh-Hadamard block [b, b] in fp64: entry (i, j) = (-1)^popcount(i & j) / sqrt(b).

    Reading: the page names H only as the predefined WHT matrix. Sylvester's (natural)
    ordering is taken, the one the recursion H_2n = [[H_n, H_n], [H_n, -H_n]] produces,
    and the orthonormal scaling 1/sqrt(b), so that H is symmetric and orthogonal. Another
    ordering of the same Walsh functions only relabels the columns of F (the positions
    E), and another scale only rescales c."""
    assert b >= 1 and b & (b - 1) == 0
    i = np.arange(b)
    par = np.zeros((b, b), dtype=np.int64)
    ij = i[:, None] & i[None, :]
    while np.any(ij):
        par ^= ij & 1
        ij = ij >> 1
    H = np.where(par == 1, -1.0, 1.0) / math.sqrt(b)
    H.flags.writeable = False                       # shared by the cache
    return H


def walsh_hadamard(K: int) -> np.ndarray:
    """H [K, K] in fp64: block-diagonal with blocks walsh_hadamard_block(wht_block_size(K))."""
    b = wht_block_size(K)
    blk = walsh_hadamard_block(b)
    H = np.zeros((K, K))
    for s in range(0, K, b):
        H[s:s + b, s:s + b] = blk
    return H


def qwha_dense_F(N: int, K: int, row_ptr, col, c) -> np.ndarray:
    """The sparse coefficient matrix F [N, K] written out densely: row n holds the values
    c[j] at columns col[j] for j in [row_ptr[n], row_ptr[n+1]).

    Reading: the page gives F as a value vector c and an index list E. E is taken in
    compressed-row form (row offsets plus column indices), the position (n, col[j]) of
    each value; every position appears at most once."""
    row_ptr = np.asarray(row_ptr, np.int64)
    col = np.asarray(col, np.int64)
    c = np.asarray(c, np.float64)
    assert row_ptr.shape == (N + 1,) and row_ptr[0] == 0 and np.all(np.diff(row_ptr) >= 0)
    assert col.shape == c.shape == (row_ptr[-1],)
    F = np.zeros((N, K))
    for n in range(N):
        for j in range(row_ptr[n], row_ptr[n + 1]):
            assert 0 <= col[j] < K and F[n, col[j]] == 0.0
            F[n, col[j]] = c[j]
    return F


def qwha_delta(N: int, K: int, row_ptr, col, c) -> np.ndarray:
    """Delta W = F H^{-1} [N, K] in fp64 (the page's single-transform formula). H is
    orthogonal, so H^{-1} is its transpose."""
    H_inv = walsh_hadamard(K).T
    return qwha_dense_F(N, K, row_ptr, col, c) @ H_inv


def qwha_transform(X) -> np.ndarray:
    """Z = X H^{-T} in fp64: each token row x becomes H^{-1} x, the transformed input that
    F multiplies in Delta W x = F (H^{-1} x). H is block-diagonal, so the product is taken
    one diagonal block at a time (the same numbers as the full K x K product without
    forming it); each block is orthogonal, so its inverse is its transpose."""
    X = np.asarray(X, np.float64)
    K = X.shape[1]
    b = wht_block_size(K)
    H_inv = walsh_hadamard_block(b).T
    Z = np.empty_like(X)
    for s in range(0, K, b):
        Z[:, s:s + b] = X[:, s:s + b] @ H_inv.T
    return Z


def qwha_adapter_out(Z, N: int, row_ptr, col, c) -> np.ndarray:
    """Z F^T [M, N] in fp64: for each token, F applied to its transformed input, i.e. the
    page's F (H^{-1} x), with F given by its compressed rows (a scipy sparse product)."""
    import scipy.sparse
    Z = np.asarray(Z, np.float64)
    row_ptr = np.asarray(row_ptr, np.int64)
    col = np.asarray(col, np.int64)
    c = np.asarray(c, np.float64)
    K = Z.shape[1]
    assert row_ptr.shape == (N + 1,) and row_ptr[0] == 0 and np.all(np.diff(row_ptr) >= 0)
    assert col.shape == c.shape == (row_ptr[-1],) and np.all((col >= 0) & (col < K))
    for n in range(N):                              # positions within a row are distinct
        seg = col[row_ptr[n]:row_ptr[n + 1]]
        assert np.unique(seg).size == seg.size
    F = scipy.sparse.csr_matrix((c, col, row_ptr), shape=(N, K))
    return np.asarray((F @ Z.T).T)


def qwha_linear_fwd_factored(X, Wd, row_ptr, col, c) -> np.ndarray:
    """The same Y as qwha_linear_fwd in the page's order Delta W x = F (H^{-1} x): the
    transform of each token, then the sparse product. For widths where forming
    Delta W [N, K] or H [K, K] would be too large."""
    X = np.asarray(X, np.float64)
    Wd = np.asarray(Wd, np.float64)
    return X @ Wd.T + qwha_adapter_out(qwha_transform(X), Wd.shape[0], row_ptr, col, c)


def qwha_linear_fwd(X, Wd, row_ptr, col, c) -> np.ndarray:
    """Y = X Wd^T + X Delta W^T in fp64: the frozen (dequantised) base plus the unmerged
    Walsh-Hadamard adapter, with Delta W = F H^{-1} [N, K]."""
    X = np.asarray(X, np.float64)
    Wd = np.asarray(Wd, np.float64)
    N, K = Wd.shape
    return X @ Wd.T + X @ qwha_delta(N, K, row_ptr, col, c).T


def _qwha_value_rows(N: int, row_ptr) -> np.ndarray:
    """The row n of every stored value, in storage order."""
    row_ptr = np.asarray(row_ptr, np.int64)
    assert row_ptr.shape == (N + 1,) and row_ptr[0] == 0 and np.all(np.diff(row_ptr) >= 0)
    return np.repeat(np.arange(N), np.diff(row_ptr))


def qwha_linear_bwd(X, dY, Wd, row_ptr, col, c):
    """Gradients of the QWHA linear Y = X Wd^T + X Delta W^T, Delta W = F H^{-1}, in fp64,
    for an upstream gradient dY [M, N]:
        dX  = dY (Wd + Delta W)                          [M, K]
        dc_j = (dY^T Z)[n_j, col_j],  Z = X H^{-T}        [nnz]
    where value j sits at (n_j, col_j). Returns (dX, dc).

    Reading: the page trains the values c of F at positions E chosen once at
    initialisation (AdaAlloc, then the refinement of c), and the frozen quantised base
    gets no gradient. So the trainable gradient is that of c alone: the gradient of F,
    dY^T X H^{-T}, read at the positions E and nowhere else."""
    X = np.asarray(X, np.float64)
    dY = np.asarray(dY, np.float64)
    Wd = np.asarray(Wd, np.float64)
    N, K = Wd.shape
    dX = dY @ (Wd + qwha_delta(N, K, row_ptr, col, c))
    G = dY.T @ qwha_transform(X)                    # gradient of the dense F [N, K]
    rows = _qwha_value_rows(N, row_ptr)
    dc = G[rows, np.asarray(col, np.int64)]
    return dX, dc


def qwha_inverse_transform_rows(U) -> np.ndarray:
    """U H^{-1} in fp64 for rows U [M, K], one diagonal block of H at a time (the same
    numbers as the full K x K product without forming it)."""
    U = np.asarray(U, np.float64)
    K = U.shape[1]
    b = wht_block_size(K)
    H_inv = walsh_hadamard_block(b).T
    out = np.empty_like(U)
    for s in range(0, K, b):
        out[:, s:s + b] = U[:, s:s + b] @ H_inv
    return out


def qwha_linear_bwd_factored(X, dY, Wd, row_ptr, col, c, chunk: int = 4096):
    """The same (dX, dc) as qwha_linear_bwd without forming Delta W or the dense gradient of
    F, for widths where those [N, K] matrices are too large:
        dX   = dY Wd + (dY F) H^{-1}     (the sparse product, then the blockwise inverse
                                          transform of each token row)
        dc_j = sum_m dY[m, n_j] Z[m, col_j]   with Z = X H^{-T} (taken in chunks of values)."""
    import scipy.sparse
    X = np.asarray(X, np.float64)
    dY = np.asarray(dY, np.float64)
    Wd = np.asarray(Wd, np.float64)
    N, K = Wd.shape
    row_ptr = np.asarray(row_ptr, np.int64)
    col = np.asarray(col, np.int64)
    c = np.asarray(c, np.float64)
    assert col.shape == c.shape == (row_ptr[-1],) and np.all((col >= 0) & (col < K))
    F = scipy.sparse.csr_matrix((c, col, row_ptr), shape=(N, K))
    dX = dY @ Wd + qwha_inverse_transform_rows(np.asarray((F.T @ dY.T).T))
    Z = qwha_transform(X)
    rows = _qwha_value_rows(N, row_ptr)
    dc = np.empty(c.shape[0])
    for s in range(0, c.shape[0], chunk):
        e = min(s + chunk, c.shape[0])
        dc[s:e] = np.einsum("mj,mj->j", dY[:, rows[s:e]], Z[:, col[s:e]])
    return dX, dc


# --------------------------------------------------------------------------------------
# The adapter optimiser step with paged states (QLoRA page, aizip.shop/methodologies/qlora,
# section "3. Paged Optimizer": optimiser states held in unified memory, paged to host RAM
# when device memory runs short, with the memory decomposition listing the optimiser
# states as the pageable part)
# --------------------------------------------------------------------------------------

def adamw_step(master, grad, m, v, step: int, lr: float, beta1: float, beta2: float, eps: float,
               weight_decay: float, grad_scale: float = 1.0):
    """One AdamW step on a flat adapter parameter vector, fp64.

    Reading: the page names no optimiser, only that its states are pageable. AdamW is
    taken: Adam's bias-corrected first and second moments with weight decay decoupled from
    the gradient. With g = grad_scale * grad and t = step (1 for the first step):
        m <- beta1 m + (1 - beta1) g
        v <- beta2 v + (1 - beta2) g^2
        theta <- theta (1 - lr weight_decay) - lr (m / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + eps)
    The trained copy theta (`master`) is kept in full precision; the bf16 copy the linear
    layer reads is RNbf(theta). grad_scale folds a data-parallel average (1/world) into
    the step. Returns (master, m, v, param_bf16_bits)."""
    assert step >= 1
    theta = np.asarray(master, np.float64).copy()
    g = np.asarray(grad, np.float64) * grad_scale
    m = beta1 * np.asarray(m, np.float64) + (1.0 - beta1) * g
    v = beta2 * np.asarray(v, np.float64) + (1.0 - beta2) * g * g
    m_hat = m / (1.0 - beta1 ** step)
    v_hat = v / (1.0 - beta2 ** step)
    theta = theta * (1.0 - lr * weight_decay) - lr * m_hat / (np.sqrt(v_hat) + eps)
    return theta, m, v, f32_to_bf16_bits(theta.astype(np.float32))


# --------------------------------------------------------------------------------------
# Lion with INT8 momentum (QFT page, gist.science/ko/paper/2310.07147, section 2.1:
# the Lion optimiser tracks only a momentum, its update is a sign so the update size is
# fixed, and the momentum is stored in INT8)
# --------------------------------------------------------------------------------------

def lion_int8_step(theta, grad, m_codes, m_absmax, lr: float, beta1: float, beta2: float,
                   weight_decay: float):
    """One Lion step with the momentum held as blockwise INT8, in fp32, one IEEE operation
    at a time (the new momentum codes are integer decisions, so the arithmetic is fixed).

    Lion (the published update): c = beta1 m + (1 - beta1) g, theta <- theta (1 - lr
    weight_decay) - lr sign(c), m <- beta2 m + (1 - beta2) g. Reading: the page gives no
    INT8 scheme for the momentum; the blockwise absmax code of the int8 weight format is
    taken (blocks of 64, fp32 absmax per block, codes in [-127, 127]): before the step
    m_j = RN32(code_j * RN32(a_b / 127)); after it the blocks are re-encoded with their new
    absmax. With f32 values: omb = RN32(1 - beta), decay = RN32(1 - RN32(lr wd)),
        c      = RN32(RN32(beta1 m) + RN32(omb1 g))
        theta' = RN32(RN32(theta decay) - lr sign(c))        (sign(0) = 0)
        m'     = RN32(RN32(beta2 m) + RN32(omb2 g))
    The trained copy theta is fp32; the bf16 copy is RNbf(theta'). The last block may be
    partial. Returns (theta', m_codes', m_absmax', param_bf16_bits)."""
    f = np.float32
    theta = np.asarray(theta, np.float32).ravel()
    g = np.asarray(grad, np.float32).ravel()
    n = theta.size
    codes = np.asarray(m_codes, np.int8).ravel()[:n]
    absmax = np.asarray(m_absmax, np.float32).ravel()
    b1, b2 = f(beta1), f(beta2)
    omb1, omb2 = f(f(1.0) - b1), f(f(1.0) - b2)
    decay = f(f(1.0) - f(f(lr) * f(weight_decay)))
    blk = np.arange(n) // BLOCK
    sc = (absmax / f(INT8_QMAX)).astype(np.float32)
    m = (codes.astype(np.float32) * sc[blk]).astype(np.float32)
    c = (b1 * m).astype(np.float32) + (omb1 * g).astype(np.float32)
    u = np.where(c > 0, f(1.0), np.where(c < 0, f(-1.0), f(0.0))).astype(np.float32)
    theta_new = (theta * decay).astype(np.float32) - (f(lr) * u).astype(np.float32)
    m_new = ((b2 * m).astype(np.float32) + (omb2 * g).astype(np.float32)).astype(np.float32)
    nb = (n + BLOCK - 1) // BLOCK
    a_new = np.zeros(nb, np.float32)
    np.maximum.at(a_new, blk, np.abs(m_new))
    codes_new = int8_encode(m_new, a_new)
    return theta_new.astype(np.float32), codes_new, a_new, f32_to_bf16_bits(theta_new)
