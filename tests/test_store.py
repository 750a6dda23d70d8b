"""Quantised weights on disk (quantized_base_rank_b200/store.py), on CPU: a file written
and read back gives the same arrays bit for bit, its arrays take exactly the bytes of
the oracle's storage accounting (4 + 8/64 + 32/16384 bits per parameter for NF4 + DQ),
and damaged or inconsistent files are refused."""
import json
import os
import struct

import numpy as np
import pytest
import torch

import oracle.qlora_oracle as o
from quantized_base_rank_b200 import store, synth
from quantized_base_rank_b200.binding import QuantWeight


def _weight(fmt, N, K, seed):
    """A QuantWeight in host tensors, its arrays from the oracle's quantise."""
    W = synth.normal_bf16((N, K), 0.02, seed, 0)
    q = o.quantize_weight(W.float().numpy(), fmt)
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(np.asarray(a, dtype=dt)).reshape(-1))
    if fmt == "nf4_dq":
        return QuantWeight(fmt, N, K, t(q["codes"], np.uint8), None, t(q["qabsmax"], np.int8),
                           t(q["group_scale"], np.float32), t([q["mean"]], np.float32))
    return QuantWeight(fmt, N, K, t(q["codes"], np.int8), t(q["absmax"], np.float32))


def _same(a: QuantWeight, b: QuantWeight):
    assert (a.fmt, a.N, a.K) == (b.fmt, b.N, b.K)
    for name, _, _ in store.layout(a.fmt, a.N, a.K):
        x, y = getattr(a, name), getattr(b, name)
        assert x.dtype == y.dtype and torch.equal(x.view(torch.uint8), y.view(torch.uint8)), name


WEIGHTS = [("layers.0.q", "nf4_dq", 64, 256), ("layers.0.up", "int8", 48, 320), ("layers.1.down", "nf4_dq", 40, 1344),
           ("odd", "nf4_dq", 3, 100), ("odd8", "int8", 5, 7)]


@pytest.fixture(scope="module")
def weights():
    return {name: _weight(fmt, N, K, i) for i, (name, fmt, N, K) in enumerate(WEIGHTS)}


def test_round_trip_is_bit_exact_and_keeps_order(tmp_path, weights):
    p = str(tmp_path / "stack.qlb")
    store.save(p, weights)
    back = store.load(p)
    assert list(back) == list(weights)
    for name in weights:
        _same(weights[name], back[name])
        assert back[name].desc.N == weights[name].N and back[name].desc.K == weights[name].K
    assert not [f for f in os.listdir(tmp_path) if ".tmp" in f]


def test_array_bytes_equal_the_oracle_storage_accounting(tmp_path, weights):
    for name, fmt, N, K in WEIGHTS:
        acct = o.storage_bytes(fmt, N * K)
        lay = store.layout(fmt, N, K)
        assert [a for a, _, _ in lay] == list(acct)
        assert {a: c * np.dtype(d).itemsize for a, d, c in lay} == acct
    # 4.127 bits per parameter for NF4 + DQ on a 7B-shaped weight (plus the one fp32
    # mean of the tensor), without writing it
    n = 4096 * 4096
    bits = 8 * sum(c * np.dtype(d).itemsize for _, d, c in store.layout("nf4_dq", 4096, 4096)) / n
    assert bits == 4 + 8 / 64 + 32 / 16384 + 32 / n


def test_arrays_start_on_64_byte_boundaries(tmp_path, weights):
    p = str(tmp_path / "w.qlb")
    store.save(p, weights)
    data = open(p, "rb").read()
    (jlen,) = struct.unpack("<Q", data[-16:-8])
    index = json.loads(data[-16 - jlen:-16].decode())
    offs = [a["offset"] for e in index["weights"] for a in e["arrays"]]
    assert all(off % 64 == 0 for off in offs) and offs == sorted(offs) and offs[0] == 64


def _rewrite_index(p, edit):
    data = open(p, "rb").read()
    (jlen,) = struct.unpack("<Q", data[-16:-8])
    index = json.loads(data[-16 - jlen:-16].decode())
    edit(index)
    new = json.dumps(index).encode()
    with open(p, "wb") as f:
        f.write(data[:-16 - jlen] + new + struct.pack("<Q", len(new)) + data[-8:])


def test_empty_file_round_trip(tmp_path):
    p = str(tmp_path / "empty.qlb")
    store.save(p, {})
    assert store.load(p) == {}


@pytest.mark.parametrize("damage", ["flip", "truncate", "magic", "count", "dtype", "offset", "format", "dup"])
def test_damaged_files_are_refused(tmp_path, weights, damage):
    p = str(tmp_path / "w.qlb")
    store.save(p, weights)
    if damage == "flip":                                   # one bit inside the first array
        data = bytearray(open(p, "rb").read())
        data[64 + 5] ^= 0x10
        open(p, "wb").write(bytes(data))
    elif damage == "truncate":
        data = open(p, "rb").read()
        open(p, "wb").write(data[:len(data) // 2])
    elif damage == "magic":
        data = bytearray(open(p, "rb").read())
        data[0] ^= 1
        open(p, "wb").write(bytes(data))
    elif damage == "count":
        _rewrite_index(p, lambda ix: ix["weights"][0]["arrays"][0].update(count=1))
    elif damage == "dtype":
        _rewrite_index(p, lambda ix: ix["weights"][1]["arrays"][0].update(dtype="uint8"))
    elif damage == "offset":
        _rewrite_index(p, lambda ix: ix["weights"][0]["arrays"][1].update(offset=65))
    elif damage == "format":
        _rewrite_index(p, lambda ix: ix["weights"][0].update(format="nf3"))
    elif damage == "dup":
        _rewrite_index(p, lambda ix: ix["weights"][1].update(name=ix["weights"][0]["name"]))
    with pytest.raises(ValueError):
        store.load(p)


def test_save_refuses_inconsistent_weights(tmp_path, weights):
    q = weights["layers.0.q"]
    p = str(tmp_path / "w.qlb")
    with pytest.raises(ValueError):
        store.save(p, [("a", q), ("a", q)])
    with pytest.raises(ValueError):
        store.save(p, [(3, q)])
    short = QuantWeight("nf4_dq", q.N, q.K, q.codes[:-1].clone(), None, q.qabsmax, q.group_scale, q.mean)
    with pytest.raises(ValueError):
        store.save(p, {"short": short})
    wrong = QuantWeight("nf4_dq", q.N, q.K, q.codes, None, q.qabsmax.view(torch.uint8), q.group_scale, q.mean)
    with pytest.raises(ValueError):
        store.save(p, {"wrong": wrong})
    missing = QuantWeight("nf4_dq", q.N, q.K, q.codes, None, None, q.group_scale, q.mean)
    with pytest.raises(ValueError):
        store.save(p, {"missing": missing})
    assert not os.path.exists(p) and not os.listdir(tmp_path)
