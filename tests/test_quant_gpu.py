"""GPU vs oracle, bit-exact: NF4 codes, absmax, double-quantised constants, int8
codes and dequantised weights, on the workloads' weights and on edge cases."""
import numpy as np
import pytest
import torch

import oracle.qlora_oracle as o
from quantized_base_rank_b200 import binding as B
from quantized_base_rank_b200 import synth

pytestmark = pytest.mark.gpu


def _u32(x):
    return np.asarray(x, np.float32).view(np.uint32)


def _weights():
    yield "cfg1-256x256", synth.make_inputs(synth.CFG1)["W"]
    yield "cfg2-4096x4096-outliers", synth.weight_with_outliers(4096, 4096, 0.02, 0.001, 20.0, 0)
    yield "ragged-odd", synth.normal_bf16((64 * 1000 + 37,), 0.02, 5, 0)
    rng = np.random.default_rng(9)
    special = np.zeros(64 * 64, np.float32)
    special[64:128] = 0.0                                            # zero block
    special[128:192] = -0.0
    special[192:256] = rng.standard_normal(64) * 1e-39               # subnormal block
    special[256:320] = rng.standard_normal(64) * 3e38 / 4            # huge block
    special[320:384] = np.float32([1.0, -1.0] * 32)                  # +-absmax only
    vals = (np.arange(0, 0x7F80, 7, dtype=np.uint32) << 16).view(np.float32)
    special[384:384 + 2048] = np.resize(vals, 2048) * np.resize([1, -1], 2048)
    special[2432:] = rng.standard_normal(special.size - 2432) * 0.05
    yield "special-values", synth.to_bf16(special)
    yield "boundary-sweep", _boundary_sweep()


def _ceil_bf16_bits(d):
    """Bits of the smallest bf16 >= d, elementwise (d > 0, fp64): round up to fp32, then
    round the fp32 bit pattern up to bf16."""
    f = d.astype(np.float32)
    f = np.where(f.astype(np.float64) < d, np.nextafter(f, np.float32(np.inf)), f)
    return ((f.view(np.uint32).astype(np.uint64) + 0xFFFF) >> 16).astype(np.uint32)


def _boundary_sweep():
    """One block for every positive finite bf16 absmax a (all exponents, all mantissas,
    subnormals included). Each block holds +a, then, for each positive midpoint m of the
    grid, the bf16 values at and just below ceil_bf16(a*m), each with both signs; the
    rest of the block is uniform in [-a, a]. Every element sits on or next to a decision
    point, so a wrong boundary for any absmax changes a code."""
    mids = o.nf4_midpoints()[8:]                     # the 7 positive midpoints (fp64, exact)
    assert len(mids) == 7 and min(mids) > 0
    rng = np.random.default_rng(11)
    abits = np.arange(1, 0x7F80, dtype=np.uint32)
    a = (abits << 16).view(np.float32).astype(np.float64)
    blocks = np.zeros((abits.size, 64), np.uint32)
    blocks[:, 0] = abits
    for k, m in enumerate(mids):
        c = _ceil_bf16_bits(a * m)
        below = np.where(c > 0, c - 1, 0)
        blocks[:, 1 + 4 * k] = c
        blocks[:, 2 + 4 * k] = c | 0x8000
        blocks[:, 3 + 4 * k] = below
        blocks[:, 4 + 4 * k] = below | 0x8000
    rest = (rng.uniform(-1.0, 1.0, (abits.size, 64 - 29)) * a[:, None]).astype(np.float32)
    blocks[:, 29:] = synth.to_bf16(rest).view(torch.int16).numpy().astype(np.uint32) & 0xFFFF
    return torch.from_numpy(blocks.astype(np.uint16).view(np.int16).ravel()).view(torch.bfloat16)


WEIGHTS = list(_weights())


@pytest.mark.parametrize("name,W", WEIGHTS, ids=[w[0] for w in WEIGHTS])
def test_nf4_dq_bitexact(name, W):
    w = W.float().numpy().ravel()
    n = w.size
    codes, absmax = B.nf4_quantize(W.cuda().contiguous().view(-1))
    qa, gs, mu = B.dq_quantize(absmax)
    ref_codes, ref_a = o.nf4_quantize(w)
    ref_qa, ref_gs, ref_mu = o.dq_encode(ref_a)
    assert np.array_equal(codes.cpu().numpy(), ref_codes)
    assert np.array_equal(_u32(absmax.cpu().numpy()), _u32(ref_a))
    assert np.array_equal(qa.cpu().numpy(), ref_qa)
    assert np.array_equal(_u32(gs.cpu().numpy()), _u32(ref_gs))
    assert _u32(mu.cpu().numpy())[0] == _u32(np.float32(ref_mu))
    if n % 64 == 0:
        Wr = W.reshape(-1, 64)
        qw = B.QuantWeight("nf4_dq", Wr.shape[0], 64, codes, None, qa, gs, mu)
        wd = B.dequantize(qw).float().cpu().numpy().ravel()
        ref_wd = o.nf4_dequant(ref_codes, o.dq_decode(ref_qa, ref_gs, ref_mu), n)
        assert np.array_equal(_u32(wd), _u32(ref_wd))
    assert B.device_status() == B.QL_OK


@pytest.mark.parametrize("name,W", WEIGHTS, ids=[w[0] for w in WEIGHTS])
def test_nf4_dq_fused_matches_two_step(name, W):
    """The one-call NF4 + double quantisation gives the same bits as the two calls, and
    the oracle's."""
    Wd = W.cuda().contiguous().view(-1)
    codes, absmax, qa, gs, mu = B.nf4_dq_quantize(Wd)
    c2, a2 = B.nf4_quantize(Wd)
    qa2, gs2, mu2 = B.dq_quantize(a2)
    for x, y in ((codes, c2), (absmax, a2), (qa, qa2), (gs, gs2), (mu, mu2)):
        assert torch.equal(x.view(torch.uint8), y.view(torch.uint8))
    ref_codes, ref_a = o.nf4_quantize(W.float().numpy().ravel())
    ref_qa, ref_gs, ref_mu = o.dq_encode(ref_a)
    assert np.array_equal(codes.cpu().numpy(), ref_codes)
    assert np.array_equal(qa.cpu().numpy(), ref_qa)
    assert np.array_equal(_u32(gs.cpu().numpy()), _u32(ref_gs))
    assert _u32(mu.cpu().numpy())[0] == _u32(np.float32(ref_mu))
    assert B.device_status() == B.QL_OK


@pytest.mark.parametrize("name,W", WEIGHTS, ids=[w[0] for w in WEIGHTS])
def test_int8_bitexact(name, W):
    w = W.float().numpy().ravel()
    codes, absmax = B.int8_quantize(W.cuda().contiguous().view(-1))
    ref_c, ref_a = o.int8_quantize(w)
    assert np.array_equal(codes.cpu().numpy(), ref_c)
    assert np.array_equal(_u32(absmax.cpu().numpy()), _u32(ref_a))
    if w.size % 64 == 0:
        qw = B.QuantWeight("int8", w.size // 64, 64, codes, absmax)
        wd = B.dequantize(qw).float().cpu().numpy().ravel()
        assert np.array_equal(_u32(wd), _u32(o.int8_dequant(ref_c, ref_a)))
    assert B.device_status() == B.QL_OK


def _int8_exhaustive_blocks():
    """For each of 473 absmax values a (43 mantissas at each of 11 exponents, the
    subnormal range, the smallest normals and the largest finite included), every bf16
    magnitude <= a in both signs, 63 to a block with +a first so that each block's absmax
    is a. Every quotient x / (a/127) an element of such a block can produce is covered."""
    rows = []
    for e in (0, 1, 2, 20, 60, 100, 120, 127, 140, 200, 254):
        for m in range(0, 128, 3):
            ab = (e << 7) | m
            if ab == 0:
                continue
            mags = np.arange(0, ab + 1, dtype=np.uint32)
            vals = np.concatenate([mags, mags | 0x8000])
            pad = (-vals.size) % 63
            vals = np.concatenate([vals, np.zeros(pad, np.uint32)]).reshape(-1, 63)
            blk = np.empty((vals.shape[0], 64), np.uint32)
            blk[:, 0] = ab
            blk[:, 1:] = vals
            rows.append(blk)
    bits = np.concatenate(rows).ravel().astype(np.uint16)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)


def test_int8_every_bf16_below_many_absmax():
    """The fast quotient (reciprocal plus one residual correction) and the add-based
    half-even rounding give the oracle's codes, bit for bit, on every element value."""
    W = _int8_exhaustive_blocks()
    w = W.float().numpy()
    codes, absmax = B.int8_quantize(W.cuda())
    ref_c, ref_a = o.int8_quantize(w)
    got = codes.cpu().numpy()
    bad = np.flatnonzero(got != ref_c)
    assert bad.size == 0, (f"{bad.size} codes differ; first at {bad[0]}: x={w[bad[0]]!r} "
                           f"a={ref_a[bad[0] // 64]!r} got {got[bad[0]]} want {ref_c[bad[0]]}")
    assert np.array_equal(_u32(absmax.cpu().numpy()), _u32(ref_a))
    assert B.device_status() == B.QL_OK


def test_unaligned_input_takes_scalar_path():
    W = synth.normal_bf16((64 * 300 + 3,), 0.02, 6, 0).cuda()
    Wu = W[1:]                                   # 2-byte aligned, not 16
    codes, absmax = B.nf4_quantize(Wu)
    ref_codes, ref_a = o.nf4_quantize(Wu.float().cpu().numpy())
    assert np.array_equal(codes.cpu().numpy(), ref_codes)
    assert np.array_equal(_u32(absmax.cpu().numpy()), _u32(ref_a))


def test_dq_exact_mean_on_wide_exponent_range():
    """Arbitrary fp32 constants spanning ~240 binades: the mean comes from the exact
    sum, so GPU and oracle (math.fsum) agree bit for bit."""
    rng = np.random.default_rng(21)
    a = (rng.random(300_000) * 2.0 ** rng.integers(-148, 100, 300_000)).astype(np.float32)
    a[:5] = np.float32([0.0, 1e-45, 3.0e38, 1.0, 2.0 ** -126])
    qa, gs, mu = B.dq_quantize(torch.from_numpy(a).cuda())
    rqa, rgs, rmu = o.dq_encode(a)
    assert _u32(mu.cpu().numpy())[0] == _u32(np.float32(rmu))
    assert np.array_equal(_u32(gs.cpu().numpy()), _u32(rgs))
    assert np.array_equal(qa.cpu().numpy(), rqa)


def test_nonfinite_input_sets_device_flag():
    assert B.device_status() == B.QL_OK
    W = synth.normal_bf16((64 * 8,), 0.02, 7, 0)
    W[100] = float("nan")
    B.nf4_quantize(W.cuda())
    assert B.device_status() == B.QL_ERR_NONFINITE
    assert B.device_status() == B.QL_OK            # cleared on read
    W[100] = float("inf")
    B.int8_quantize(W.cuda())
    assert B.device_status() == B.QL_ERR_NONFINITE


@pytest.mark.parametrize("N,K", [(8192, 8192), (22016, 8192)])
def test_full_size_65b_shapes(N, K):
    W = synth.normal_bf16((N, K), 0.02, 3, N % 7).cuda()
    codes, absmax = B.nf4_quantize(W.view(-1))
    qa, gs, mu = B.dq_quantize(absmax)
    w = W.float().cpu().numpy().ravel()
    ref_codes, ref_a = o.nf4_quantize(w)
    ref_qa, ref_gs, ref_mu = o.dq_encode(ref_a)
    assert np.array_equal(codes.cpu().numpy(), ref_codes)
    assert np.array_equal(qa.cpu().numpy(), ref_qa)
    assert _u32(mu.cpu().numpy())[0] == _u32(np.float32(ref_mu))
    c8, a8 = B.int8_quantize(W.view(-1))
    rc8, ra8 = o.int8_quantize(w)
    assert np.array_equal(c8.cpu().numpy(), rc8)


# ---- quantisation sharded across ranks (run here as shards in sequence) -------------

@pytest.mark.parametrize("shards", [2, 3])
@pytest.mark.parametrize("name,W", [w for w in WEIGHTS if w[0] in ("cfg2-4096x4096-outliers", "ragged-odd",
                                                                 "boundary-sweep")],
                         ids=lambda v: v if isinstance(v, str) else "")
def test_sharded_nf4_dq_matches_whole(shards, name, W):
    """Each shard quantised on its own with its exact DQ bins, the bins summed as integers
    (the all-reduce), the double quantisation finished per shard: every array is the
    whole-weight nf4_dq_quantize result, bit for bit."""
    from quantized_base_rank_b200 import dp
    flat = W.cuda().contiguous().view(-1)
    n = flat.numel()
    codes, absmax, qa, gs, mu = B.nf4_dq_quantize(flat)
    spans = [dp.shard_elems(n, shards, r) for r in range(shards)]
    parts = [B.nf4_quantize_shard(flat[a:b]) for a, b in spans]
    total = sum(p[2] for p in parts)                       # integer sum of the bins
    nb_total = (n + 63) // 64
    for (a, b), (c, am, _) in zip(spans, parts):
        q, g, m = B.dq_quantize_shard(am, total, nb_total)
        assert a % 2 == 0 and a % 64 == 0
        assert torch.equal(c[: (b - a + 1) // 2], codes[a // 2: a // 2 + (b - a + 1) // 2])
        assert torch.equal(am.view(torch.int32), absmax[a // 64: a // 64 + am.numel()].view(torch.int32))
        assert torch.equal(q, qa[a // 64: a // 64 + q.numel()])
        assert torch.equal(g.view(torch.int32), gs[a // 16384: a // 16384 + g.numel()].view(torch.int32))
        assert torch.equal(m.view(torch.int32), mu.view(torch.int32))
    assert B.device_status() == B.QL_OK


def test_nf4_dq_batch_matches_single_weight_calls():
    """The batched entry equals nf4_dq_quantize of each weight bit for bit: every output
    (codes, absmax, DQ codes, group scales, mean). The mix spans the batch kernel (whole
    blocks, aligned), the single-weight path inside the batch (a ragged block count, an
    unaligned source), weights of one to thousands of groups, the outlier weight, the
    special values, and more than 128 weights so that the batch runs in two launches."""
    specials = dict(_weights())
    Ws = [specials["cfg1-256x256"], specials["cfg2-4096x4096-outliers"], specials["special-values"],
          specials["ragged-odd"], synth.normal_bf16((11008 * 64,), 0.02, 21, 0)]
    Ws += [synth.normal_bf16((64 * (1 + (i * 37) % 300),), 0.01 * (1 + i % 5), 30 + i, 0) for i in range(127)]
    dev_Ws = [W.cuda().contiguous().view(-1) for W in Ws]
    base = torch.empty(64 * 500 + 1, dtype=torch.bfloat16, device="cuda")
    base[1:].copy_(synth.normal_bf16((64 * 500,), 0.02, 99, 0).cuda())
    dev_Ws.append(base[1:])                                  # 2-byte aligned only
    got = B.nf4_dq_quantize_batch(dev_Ws)
    torch.cuda.synchronize()
    assert B.device_status() == B.QL_OK
    for i, (W, g) in enumerate(zip(dev_Ws, got)):
        ref = B.nf4_dq_quantize(W)
        for name, a, b in zip(("codes", "absmax", "qabsmax", "group_scale", "mean"), g, ref):
            assert torch.equal(a.view(torch.uint8) if a.dtype != torch.uint8 else a,
                               b.view(torch.uint8) if b.dtype != torch.uint8 else b), (i, name)
    # and two of them against the oracle
    for i in (0, 1):
        w = Ws[i].float().numpy().ravel()
        ref = o.quantize_weight(w, "nf4_dq")
        assert np.array_equal(got[i][0].cpu().numpy(), ref["codes"])
        assert np.array_equal(got[i][2].cpu().numpy(), ref["qabsmax"])
