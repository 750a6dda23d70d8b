"""The multi-layer stacks: per-layer format/rank dispatch and memory accounting (CPU), and
GPU parity on sampled linears of the 7B stack and of the 65B per-layer mix.

Parity follows the single-linear tests: the quantised weight bit-exact against the
oracle's, and Y, T, dX on sampled rows plus dA, dB in full within relative Frobenius
<= 5e-3 and elementwise <= 1e-2 * max|ref| of the fp64 oracle."""
import json
import os

import numpy as np
import pytest
import torch

import oracle.qlora_oracle as o
from quantized_base_rank_b200 import stack, synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "qlora_page_figures.json")


# ---- CPU: the stacks and their accounting ----------------------------------------------

def test_7b_stack_shapes_params_and_bits():
    specs = stack.stack_7b()
    assert len(specs) == 32 * 7
    assert all(s.fmt == "nf4_dq" and s.r == 64 and s.alpha == 16.0 for s in specs)
    acc = stack.accounting(specs)
    assert acc["params"] == 32 * (4 * 4096 * 4096 + 3 * 11008 * 4096) == 6_476_005_376
    # 4 + 8/64 + 32/16384 bits per parameter, plus one fp32 mean per matrix
    n_mats = len(specs)
    assert acc["weight_bytes"] * 8 == acc["params"] * 4.126953125 + 32 * n_mats


@pytest.mark.parametrize("fmt", stack.FORMATS)
@pytest.mark.parametrize("n", [64, 65, 64 * 256, 64 * 256 + 1, 4096 * 4096, 22016 * 8192, 1000003])
def test_weight_bytes_match_the_oracle_layout(fmt, n):
    assert stack.weight_bytes(fmt, n) == sum(o.storage_bytes(fmt, n).values())


def test_page_figures_for_the_formats():
    """The NF4 + DQ layout gives the QLoRA page's bits per parameter for the constants
    (0.127) and the codes (4), and int8 gives 8.5."""
    g = json.load(open(GOLDEN))
    n = 4096 * 4096
    bits_nf4 = 8.0 * (stack.weight_bytes("nf4_dq", n) - 4) / n   # without the one fp32 mean
    const = g["const_bits_after_dq"]
    assert abs((bits_nf4 - g["grid_bits"]["value"]) - const["value"]) <= const["tol"]
    codes_per_param = (n // 2) / n
    assert codes_per_param == g["nf4_weight_bytes_per_param"]["value"]
    assert 8.0 * stack.weight_bytes("int8", n) / n == 8.5


def test_65b_mix_dispatch_is_per_decoder_layer():
    specs = stack.stack_65b_mix()
    assert len(specs) == 80 * 7
    by_layer = {}
    for s in specs:
        by_layer.setdefault(s.layer, set()).add((s.fmt, s.r))
    assert all(len(v) == 1 for v in by_layer.values())          # the layer's 7 share one choice
    choices = [next(iter(v)) for _, v in sorted(by_layer.items())]
    assert choices == synth.layer_mix_65b(80, 0)
    assert {f for f, _ in choices} == set(stack.FORMATS)
    assert {r for _, r in choices} <= {8, 16, 32, 64}
    acc = stack.accounting(specs)
    params = acc["params"]
    assert params == 80 * (4 * 8192 * 8192 + 3 * 22016 * 8192)
    all_nf4 = sum(stack.weight_bytes("nf4_dq", s.params) for s in specs)
    all_int8 = sum(stack.weight_bytes("int8", s.params) for s in specs)
    assert all_nf4 < acc["weight_bytes"] < all_int8
    assert abs(all_nf4 / 1e9 - 33.4) < 0.05 and abs(all_int8 / 1e9 - 68.8) < 0.05
    assert acc["weight_bytes"] == sum(acc["weight_bytes_by_format"].values())


def test_linear_flops_of_the_up_projection():
    spec = stack.LinearSpec(0, 5, "up", 11008, 4096, "nf4_dq", 64, 16.0)
    fwd, bwd = stack.linear_flops(spec, 8192)
    assert fwd == 2 * 8192 * 11008 * (4096 + 64) + 2 * 8192 * 4096 * 64
    assert round((fwd + bwd) / 1e9) == 1525                       # fwd + bwd + dA/dB of config 3


# ---- GPU: sampled linears against the oracle ------------------------------------------

REL_FRO, REL_ELEM = 5e-3, 1e-2


def _close(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape and np.all(np.isfinite(got)), what
    err = got - ref
    rel = np.linalg.norm(err) / np.linalg.norm(ref)
    elem = np.max(np.abs(err)) / np.max(np.abs(ref))
    assert rel <= REL_FRO and elem <= REL_ELEM, f"{what}: rel_fro={rel:.3e} rel_elem={elem:.3e}"


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _check_linear(spec, M, n_rows=128):
    from quantized_base_rank_b200 import binding as bd
    inp = synth.stack_linear_inputs(spec.layer, spec.which, spec.N, spec.K, M, spec.r)
    lin = stack.QuantizedLinear(spec, inp["W"], inp["A"], inp["B"])
    assert lin.stored_bytes() == stack.weight_bytes(spec.fmt, spec.params)
    Y, T = lin.forward(inp["X"])
    dX, dA, dB = lin.backward(inp["X"], inp["dY"], T)
    torch.cuda.synchronize()
    assert bd.device_status() == bd.QL_OK

    ref = o.quantize_weight(inp["W"].float().cpu().numpy(), spec.fmt)
    wd_gpu = bd.dequantize(lin.qw).float().cpu().numpy().ravel()
    assert np.array_equal(wd_gpu.view(np.uint32), ref["wdeq"].view(np.uint32))
    wd = ref["wdeq"].reshape(spec.N, spec.K)
    X, A, B, dY = (_f64(inp[k]) for k in ("X", "A", "B", "dY"))
    rows = np.sort(np.random.default_rng(spec.layer * 8 + spec.which).choice(M, n_rows, replace=False))
    Yr, Tr = o.linear_fwd(X[rows], wd, A, B, spec.alpha, spec.r)
    dXr = o.linear_bwd(X[rows], dY[rows], wd, A, B, spec.alpha, spec.r)[0]
    dAr, dBr = o.adapter_grads(X, dY, A, B, spec.alpha, spec.r)
    _close(_f64(Y)[rows], Yr, f"{spec.name}{spec.layer} Y")
    _close(_f64(T)[rows], Tr, f"{spec.name}{spec.layer} T")
    _close(_f64(dX)[rows], dXr, f"{spec.name}{spec.layer} dX")
    _close(dA.cpu().numpy(), dAr, f"{spec.name}{spec.layer} dA")
    _close(dB.cpu().numpy(), dBr, f"{spec.name}{spec.layer} dB")


SAMPLE_7B = [(0, "q"), (31, "down"), (17, "gate")]


@pytest.mark.gpu
@pytest.mark.parametrize("layer,name", SAMPLE_7B, ids=[f"L{l}-{n}" for l, n in SAMPLE_7B])
def test_7b_stack_sampled_linear(layer, name):
    """7B stack, 4096 tokens per linear."""
    spec = next(s for s in stack.stack_7b() if s.layer == layer and s.name == name)
    _check_linear(spec, 4096)


def _sample_65b():
    specs = stack.stack_65b_mix()
    first_int8 = next(s.layer for s in specs if s.fmt == "int8")
    first_nf4 = next(s.layer for s in specs if s.fmt == "nf4_dq")
    last = specs[-1].layer
    pick = [(first_int8, "gate"), (first_nf4, "down"), (last, "q")]
    return [next(s for s in specs if s.layer == l and s.name == n) for l, n in pick]


SAMPLE_65B = _sample_65b()


@pytest.mark.gpu
@pytest.mark.parametrize("spec", SAMPLE_65B, ids=[f"L{s.layer}-{s.name}-{s.fmt}-r{s.r}" for s in SAMPLE_65B])
def test_65b_mix_sampled_linear(spec):
    """65B per-layer mix, 2048 tokens per linear, the layer's own format and rank."""
    _check_linear(spec, 2048)
