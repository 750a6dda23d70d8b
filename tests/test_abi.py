"""CPU checks of the C-ABI library: it builds, loads, exports every declared symbol,
and its host-only entry points behave (no kernel is launched here)."""
import ctypes
import os

import numpy as np
import pytest

import oracle.qlora_oracle as o
from quantized_base_rank_b200 import binding as B
from quantized_base_rank_b200 import build as build_mod


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(B.LIB_PATH):
        build_mod.build()
    return B.lib()


def test_header_declares_the_boundary():
    names = set(B.header_functions())
    for required in ("nf4_quantize", "dq_quantize", "nf4_dq_quantize", "int8_quantize", "ql_dequantize",
                     "qlora_linear_fwd", "qlora_linear_bwd", "ql_workspace_bytes",
                     "ql_get_device_status", "ql_status_string", "ql_nf4_codebook"):
        assert required in names, required


def test_library_exports_every_declared_symbol(lib):
    for name in B.header_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for s in range(7):
        assert B.status_string(s)
    assert B.status_string(0) == "ok"


def test_library_codebook_equals_oracle(lib):
    """The library computes its grid independently (bisection on erfc, in C); it must
    land on the same fp32 points as the oracle."""
    q = np.float32(B.nf4_codebook())
    assert np.array_equal(q.view(np.uint32), o.nf4_codebook().view(np.uint32))


def test_argument_validation_without_a_device(lib):
    # rejected before any CUDA call
    assert lib.nf4_quantize(None, 64, None, None, None) == B.QL_ERR_INVALID_ARG
    assert lib.nf4_quantize(None, -1, None, None, None) == B.QL_ERR_INVALID_ARG
    assert lib.nf4_quantize(None, 0, None, None, None) == B.QL_OK
    assert lib.int8_quantize(None, 64, None, None, None) == B.QL_ERR_INVALID_ARG
    assert lib.dq_quantize(None, 4, None, None, None, None, 0, None) == B.QL_ERR_INVALID_ARG
    assert lib.nf4_dq_quantize(None, 64, None, None, None, None, None, None, 0, None) == B.QL_ERR_INVALID_ARG
    assert lib.nf4_dq_quantize(16, 0, 16, 16, 16, 16, 16, 16, 256, None) == B.QL_ERR_INVALID_ARG
    # more than 2^24 blocks
    assert lib.nf4_dq_quantize(16, 64 * (1 << 24) + 1, 16, 16, 16, 16, 16, 16, 256, None) == B.QL_ERR_UNSUPPORTED
    # workspace too small
    assert lib.nf4_dq_quantize(16, 64, 16, 16, 16, 16, 16, 16, 8, None) == B.QL_ERR_WORKSPACE
    # LoRDBA forward: missing adapter, empty rank, rank beyond 256
    w = B.QLWeight(0, 0, 64, 64, 16, 0, 16, 16, 16)
    assert lib.qlora_linear_fwd_lordba(ctypes.byref(w), 16, 1, None, 16, 16, 1 << 20, None) == B.QL_ERR_INVALID_ARG
    ad = B.QLLordba(0, 1, 16, 16, 16, 16, 16)
    assert lib.qlora_linear_fwd_lordba(ctypes.byref(w), 16, 1, ctypes.addressof(ad), 16, 256, 1 << 20,
                                       None) == B.QL_ERR_INVALID_ARG
    ad = B.QLLordba(100, 3, 16, 16, 16, 16, 16)
    assert lib.qlora_linear_fwd_lordba(ctypes.byref(w), 16, 1, ctypes.addressof(ad), 16, 256, 1 << 20,
                                       None) == B.QL_ERR_UNSUPPORTED
    # Walsh-Hadamard adapter: missing or inconsistent index arrays, oversize K
    assert lib.qlora_linear_fwd_qwha(ctypes.byref(w), 16, 1, None, 16, 256, 1 << 20, None) == B.QL_ERR_INVALID_ARG
    for ad in (B.QLQwha(None, 16, 16, 4), B.QLQwha(16, None, 16, 4), B.QLQwha(16, 16, 16, -1),
               B.QLQwha(18, 16, 16, 4), B.QLQwha(16, 17, 16, 4)):
        assert lib.qlora_linear_fwd_qwha(ctypes.byref(w), 16, 1, ctypes.addressof(ad), 16, 256, 1 << 20,
                                         None) == B.QL_ERR_INVALID_ARG
    ad = B.QLQwha(16, 16, 16, 4)
    assert lib.qlora_linear_fwd_qwha(ctypes.byref(w), 16, 1, ctypes.addressof(ad), 16, None, 1 << 20,
                                     None) == B.QL_ERR_INVALID_ARG
    assert lib.qlora_linear_fwd_qwha(ctypes.byref(w), 16, 1, ctypes.addressof(ad), 16, 256, 16,
                                     None) == B.QL_ERR_WORKSPACE
    wk = B.QLWeight(0, 0, 64, 65600, 16, 0, 16, 16, 16)
    assert lib.qlora_linear_fwd_qwha(ctypes.byref(wk), 16, 1, ctypes.addressof(ad), 16, 256, 1 << 30,
                                     None) == B.QL_ERR_UNSUPPORTED
    assert lib.ql_wht(None, 1, 64, 16, None) == B.QL_ERR_INVALID_ARG
    assert lib.ql_wht(16, 1, 100, 16, None) == B.QL_ERR_UNSUPPORTED
    assert lib.ql_wht(24, 1, 64, 16, None) == B.QL_ERR_INVALID_ARG
    # optimiser step and paged memory: argument checks happen before any CUDA call
    h = B.QLAdamw(1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0, 1)
    assert lib.ql_adamw_step(16, 16, 16, 16, 16, 0, ctypes.addressof(h), None) == B.QL_OK
    assert lib.ql_adamw_step(16, 16, 16, 16, 16, -1, ctypes.addressof(h), None) == B.QL_ERR_INVALID_ARG
    assert lib.ql_adamw_step(None, 16, 16, 16, 16, 8, ctypes.addressof(h), None) == B.QL_ERR_INVALID_ARG
    assert lib.ql_adamw_step(18, 16, 16, 16, 16, 8, ctypes.addressof(h), None) == B.QL_ERR_INVALID_ARG
    for bad in (B.QLAdamw(1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0, 0), B.QLAdamw(1e-3, 1.0, 0.999, 1e-8, 0.0, 1.0, 1),
                B.QLAdamw(1e-3, 0.9, 0.999, 0.0, 0.0, 1.0, 1), B.QLAdamw(-1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0, 1),
                B.QLAdamw(1e-3, 0.9, 0.999, 1e-8, -0.1, 1.0, 1),
                B.QLAdamw(1e-3, 0.9, 0.999, 1e-8, 0.0, float("nan"), 1)):
        assert lib.ql_adamw_step(16, 16, 16, 16, 16, 8, ctypes.addressof(bad), None) == B.QL_ERR_INVALID_ARG
    hl = B.QLLion(1e-4, 0.9, 0.99, 0.0)
    assert lib.ql_lion_int8_step(16, 16, 16, 16, 16, 0, ctypes.addressof(hl), None) == B.QL_OK
    assert lib.ql_lion_int8_step(16, 16, 16, None, 16, 8, ctypes.addressof(hl), None) == B.QL_ERR_INVALID_ARG
    for bad in (B.QLLion(-1e-4, 0.9, 0.99, 0.0), B.QLLion(1e-4, 1.5, 0.99, 0.0), B.QLLion(1e-4, 0.9, -0.1, 0.0),
                B.QLLion(1e-4, 0.9, 0.99, float("inf"))):
        assert lib.ql_lion_int8_step(16, 16, 16, 16, 16, 8, ctypes.addressof(bad), None) == B.QL_ERR_INVALID_ARG
    out = ctypes.c_void_p(1)
    assert lib.ql_paged_alloc(0, ctypes.byref(out)) == B.QL_OK and not out.value
    assert lib.ql_paged_alloc(16, None) == B.QL_ERR_INVALID_ARG
    assert lib.ql_paged_free(None) == B.QL_OK
    assert lib.ql_paged_prefetch(None, 0, 1, None) == B.QL_OK
    assert lib.ql_paged_prefetch(None, 64, 1, None) == B.QL_ERR_INVALID_ARG
    assert lib.ql_dequantize(None, None, None) == B.QL_ERR_INVALID_ARG
    # dequantise: a bad format, a missing constant, an odd output address or an oversize
    # shape is refused before anything is launched or counted
    c0 = lib.ql_launch_count()
    for bad in (B.QLWeight(7, 0, 64, 64, 16, 16, 16, 16, 16), B.QLWeight(0, 0, 64, 64, 16, 0, None, 16, 16),
                B.QLWeight(1, 0, 64, 64, 16, None, 16, 16, 16), B.QLWeight(1, 0, 64, 64, 16, 18, 16, 16, 16)):
        assert lib.ql_dequantize(ctypes.byref(bad), 16, None) == B.QL_ERR_INVALID_ARG
    w = B.QLWeight(0, 0, 64, 64, 16, 0, 16, 16, 16)
    assert lib.ql_dequantize(ctypes.byref(w), 17, None) == B.QL_ERR_INVALID_ARG
    big = B.QLWeight(1, 0, 1 << 21, 1 << 21, 16, 16, 16, 16, 16)
    assert lib.ql_dequantize(ctypes.byref(big), 16, None) == B.QL_ERR_UNSUPPORTED
    assert lib.ql_launch_count() == c0
    # batched NF4 + DQ: nothing to do, a null table, a bad item, a short workspace
    assert lib.nf4_dq_quantize_batch(None, 0, None, 0, None) == B.QL_OK
    assert lib.nf4_dq_quantize_batch(None, 2, 16, 1 << 20, None) == B.QL_ERR_INVALID_ARG
    items = (B.QLNf4DqItem * 2)(B.QLNf4DqItem(16, 64, 16, 16, 16, 16, 16),
                                B.QLNf4DqItem(16, 64, 16, None, 16, 16, 16))
    c0 = lib.ql_launch_count()
    assert lib.nf4_dq_quantize_batch(items, 2, 16, 1 << 20, None) == B.QL_ERR_INVALID_ARG
    items[1] = B.QLNf4DqItem(16, 64 * (1 << 24) + 64, 16, 16, 16, 16, 16)
    assert lib.nf4_dq_quantize_batch(items, 2, 16, 1 << 20, None) == B.QL_ERR_UNSUPPORTED
    assert lib.nf4_dq_quantize_batch(items, 2, 16, 8, None) == B.QL_ERR_WORKSPACE
    assert lib.ql_launch_count() == c0
    assert B.workspace_bytes(B.QL_OP_DQ_BATCH, 224, 0, 0, 0) == 128 * 16 * 8
    assert B.workspace_bytes(B.QL_OP_DQ_BATCH, 1, 0, 0, 0) == 256
    # misaligned or null pointers, bad shapes: all rejected synchronously
    assert lib.qlora_linear_fwd(ctypes.byref(w), None, 1, None, None, 8, 16.0, None, None,
                                None, 0, None) == B.QL_ERR_INVALID_ARG


def test_adapter_entries_refuse_what_the_linear_refuses_before_any_launch(lib):
    """The LoRDBA and Walsh-Hadamard forwards launch a preparation kernel before the fused
    linear, so they must make every refusal of the linear first: a bad weight descriptor,
    misaligned tokens or output, too many tokens. Each must return the linear's own status
    and launch nothing (on a machine without a GPU a launch would fail with a CUDA error
    instead)."""
    P = 16                                                       # any 16-byte-aligned address
    good = B.QLWeight(0, 0, 64, 64, P, 0, P, P, P)
    bad_weights = {
        "null descriptor": None,
        "no codes": B.QLWeight(0, 0, 64, 64, 0, 0, P, P, P),
        "misaligned codes": B.QLWeight(0, 0, 64, 64, 24, 0, P, P, P),
        "N = 0": B.QLWeight(0, 0, 0, 64, P, 0, P, P, P),
        "K below 64": B.QLWeight(0, 0, 64, 32, P, 0, P, P, P),
        "K not a multiple of 64": B.QLWeight(0, 0, 64, 96, P, 0, P, P, P),
        "N not a multiple of 8": B.QLWeight(0, 0, 60, 64, P, 0, P, P, P),
        "NF4 without the DQ codes": B.QLWeight(0, 0, 64, 64, P, 0, 0, P, P),
        "NF4 without the group scales": B.QLWeight(0, 0, 64, 64, P, 0, P, 0, P),
        "NF4 without the mean": B.QLWeight(0, 0, 64, 64, P, 0, P, P, 0),
        "int8 without absmax": B.QLWeight(1, 0, 64, 64, P, 0, 0, 0, 0),
        "int8 with misaligned absmax": B.QLWeight(1, 0, 64, 64, P, 18, 0, 0, 0),
        "unknown format": B.QLWeight(7, 0, 64, 64, P, P, P, P, P),
    }
    ad_l = B.QLLordba(4, 1, P, P, P, P, P)
    ad_q = B.QLQwha(P, P, P, 4)
    big = 1 << 40
    c0 = lib.ql_launch_count()
    for name, w in bad_weights.items():
        wp = ctypes.byref(w) if w is not None else None
        for M in (1, 40):
            want = lib.qlora_linear_fwd(wp, P, M, P, P, 4, 4.0, P, None, 256, big, None)
            assert want in (B.QL_ERR_INVALID_ARG, B.QL_ERR_UNSUPPORTED), name
            assert lib.qlora_linear_fwd_lordba(wp, P, M, ctypes.addressof(ad_l), P, 256, big, None) == want, name
            assert lib.qlora_linear_fwd_qwha(wp, P, M, ctypes.addressof(ad_q), P, 256, big, None) == want, name
    for X, Y, M, want in ((24, P, 1, B.QL_ERR_INVALID_ARG), (P, 24, 40, B.QL_ERR_INVALID_ARG),
                          (P, P, (1 << 31) + 1, B.QL_ERR_UNSUPPORTED)):
        assert lib.qlora_linear_fwd(ctypes.byref(good), X, M, P, P, 4, 4.0, Y, None, 256, big, None) == want
        assert lib.qlora_linear_fwd_lordba(ctypes.byref(good), X, M, ctypes.addressof(ad_l), Y, 256, big,
                                           None) == want
        assert lib.qlora_linear_fwd_qwha(ctypes.byref(good), X, M, ctypes.addressof(ad_q), Y, 256, big,
                                         None) == want
    assert lib.ql_launch_count() == c0


def test_every_entry_refuses_documented_invalid_arguments(lib):
    """One argument at a time made invalid by the header's own rules (a NULL pointer, an
    address below the stated alignment, a size outside the stated range, a workspace too
    small): every entry must return an argument status and launch nothing."""
    P = 1 << 20                                               # a 16-byte-aligned address
    big = 1 << 40
    w = B.QLWeight(0, 0, 64, 64, P, 0, P, P, P)
    hp_a = B.QLAdamw(1e-3, 0.9, 0.999, 1e-8, 0.0, 1.0, 1)
    hp_l = B.QLLion(1e-4, 0.9, 0.99, 0.0)
    items = (B.QLNf4DqItem * 1)(B.QLNf4DqItem(P, 128, P, P, P, P, P))
    bad_items = (B.QLNf4DqItem * 1)(B.QLNf4DqItem(P + 1, 128, P, P, P, P, P))
    table = [
        ("nf4_quantize", [P, 128, P, P, None], {0: [None, P + 1], 1: [-1], 2: [None, P + 1, P + 2], 3: [None, P + 2]}),
        ("int8_quantize", [P, 128, P, P, None], {0: [None, P + 1], 1: [-1], 2: [None], 3: [None, P + 2]}),
        ("dq_quantize", [P, 4, P, P, P, P, big, None],
         {0: [None, P + 2], 1: [0, (1 << 24) + 1], 2: [None], 3: [None, P + 2], 4: [None, P + 2], 5: [None], 6: [0]}),
        ("nf4_dq_quantize", [P, 128, P, P, P, P, P, P, big, None],
         {0: [None, P + 1], 1: [0, (1 << 30) + 64], 2: [None, P + 2], 3: [None, P + 2], 4: [None], 5: [None, P + 2],
          6: [None, P + 2], 7: [None], 8: [0]}),
        ("nf4_quantize_shard", [P, 16384, P, P, P, P, big, None],
         {0: [None], 1: [-1], 2: [None], 3: [None], 4: [None, P + 4], 5: [None], 6: [0]}),
        ("dq_quantize_shard", [P, 256, P, 512, P, P, P, None],
         {0: [None], 1: [0], 2: [None, P + 4], 3: [255], 4: [None], 5: [None, P + 2], 6: [None, P + 2]}),
        ("ql_wht", [P, 4, 64, P, None], {0: [None, P + 8], 1: [0], 2: [32, 100], 3: [None, P + 8]}),
        ("ql_adamw_step", [P, P, P, P, P, 64, ctypes.addressof(hp_a), None],
         {0: [None, P + 2], 1: [None, P + 1], 2: [None, P + 2], 3: [None, P + 2], 4: [None, P + 2], 5: [-1], 6: [None]}),
        ("ql_lion_int8_step", [P, P, P, P, P, 64, ctypes.addressof(hp_l), None],
         {0: [None, P + 2], 1: [None, P + 1], 2: [None, P + 2], 3: [None], 4: [None, P + 2], 5: [-1], 6: [None]}),
        ("nf4_dq_quantize_batch", [ctypes.addressof(items), 1, P, big, None],
         {0: [None, ctypes.addressof(bad_items)], 1: [-1], 2: [None, P + 8], 3: [0]}),
        ("qlora_linear_fwd", [ctypes.byref(w), P, 40, P, P, 8, 8.0, P, P, P, big, None],
         {0: [None], 1: [None, P + 8], 2: [0, (1 << 31) + 1], 3: [None, P + 8], 4: [None, P + 1], 5: [0, 257],
          7: [None, P + 8], 8: [P + 1], 9: [None, P + 8], 10: [0]}),
        ("qlora_linear_bwd", [ctypes.byref(w), P, P, 40, P, P, P, 8, 8.0, P, P, P, P, big, None],
         {0: [None], 1: [None, P + 8], 2: [None, P + 8], 3: [0, (1 << 31) + 1], 4: [None, P + 1], 5: [None, P + 1],
          6: [None, P + 1], 7: [0, 257], 9: [None, P + 8], 10: [None, P + 2], 11: [None, P + 2], 12: [None], 13: [0]}),
        ("ql_dequantize", [ctypes.byref(w), P, None], {0: [None], 1: [None, P + 1]}),
    ]
    refusals = {B.QL_ERR_INVALID_ARG, B.QL_ERR_UNSUPPORTED, B.QL_ERR_WORKSPACE}
    c0 = lib.ql_launch_count()
    for name, args, bad in table:
        f = getattr(lib, name)
        for i, values in bad.items():
            for v in values:
                a = list(args)
                a[i] = v
                st = f(*a)
                assert st in refusals, (name, i, v, B.status_string(st))
    assert lib.ql_launch_count() == c0


def test_workspace_query(lib):
    assert B.workspace_bytes(B.QL_OP_DQ, 0, 0, 0, 0) >= 128
    # Walsh-Hadamard adapter: decode-shaped, one slab of Z (16 tokens); otherwise the update
    # F H [N, K], the dense F [N, K] too when the transform blocks are wider than 4096, and
    # the fused GEMM's block scales
    assert B.workspace_bytes(B.QL_OP_FWD_QWHA, 1, 4096, 4096, 0) == 4096 * 16 * 2
    assert B.workspace_bytes(B.QL_OP_FWD_QWHA, 8192, 11008, 4096, 0) == 11008 * 4096 * 2 + 64 * 11008 * 4
    assert B.workspace_bytes(B.QL_OP_FWD_QWHA, 17, 64, 192, 0) == 64 * 192 * 2 + 3 * 64 * 4
    assert B.workspace_bytes(B.QL_OP_FWD_QWHA, 40, 128, 8192, 0) == 2 * 128 * 8192 * 2 + 128 * 128 * 4
    assert B.workspace_bytes(B.QL_OP_FWD_QWHA, 1, 64, 100, 0) == 0
