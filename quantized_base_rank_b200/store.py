"""Quantised weights on disk: the frozen base kept in its stored form, so a model is
quantised once and loaded straight into the layout the kernels read (QLoRA page,
"memory decomposition": the frozen model is held in 4-bit NF4 with double-quantised
constants; AutoQRA page, section 3.1: each layer in its own format).

One file holds any number of named weights. Layout (all integers little-endian):

    8 bytes   magic b"QLBWGT01"
    the arrays' raw bytes, each at a file offset that is a multiple of 64 (zero padding
    between them)
    J bytes   UTF-8 JSON index: {"weights": [{"name", "format", "N", "K",
                  "arrays": [{"name", "dtype", "count", "offset", "crc32"}, ...]}, ...]}
    8 bytes   J, uint64
    8 bytes   magic b"QLBWGT01"

The index sits at the end so that a writer streams one array at a time (a 65B-shaped
stack is tens of GB) and a reader seeks to each array.

A weight keeps exactly the arrays its format stores, with n = N*K parameters and
nb = ceil(n/64) blocks:

    nf4_dq: codes uint8 [ceil(n/2)], qabsmax int8 [nb], group_scale fp32 [ceil(nb/256)],
            mean fp32 [1]
    int8:   codes int8 [n], absmax fp32 [nb]

(the same arrays, byte for byte, that the quantise calls write; the fp32 absmax of an
NF4 weight is a pre-quantisation intermediate and is not stored). Loading checks both
magics, the index, every array's dtype, count, offset and CRC-32 against the format's
layout, and raises ValueError on any mismatch, so a truncated or corrupted file is never
handed to the kernels. Saving writes a temporary file beside the target and renames it,
so a reader never sees a partly written file.
"""
from __future__ import annotations

import json
import os
import struct
import zlib

import numpy as np
import torch

from .binding import FORMATS, QuantWeight

MAGIC = b"QLBWGT01"
ALIGN = 64
_DTYPES = {"uint8": (np.uint8, torch.uint8), "int8": (np.int8, torch.int8), "float32": (np.float32, torch.float32)}


def layout(fmt: str, N: int, K: int) -> list[tuple[str, str, int]]:
    """(array name, dtype, element count) of every array a weight of this format stores."""
    if N < 1 or K < 1:
        raise ValueError("N and K must be positive")
    n = N * K
    nb = (n + 63) // 64
    if fmt == "nf4_dq":
        return [("codes", "uint8", (n + 1) // 2), ("qabsmax", "int8", nb), ("group_scale", "float32", (nb + 255) // 256),
                ("mean", "float32", 1)]
    if fmt == "int8":
        return [("codes", "int8", n), ("absmax", "float32", nb)]
    raise ValueError(f"unknown format {fmt!r}")


def _align(x: int) -> int:
    return -(-x // ALIGN) * ALIGN


def save(path: str, weights) -> None:
    """Write named weights (a dict name -> QuantWeight, or a sequence of (name, weight)
    pairs) to `path`, one array at a time. Device tensors are copied to the host; nothing
    is changed on the device."""
    items = list(weights.items()) if isinstance(weights, dict) else list(weights)
    names = [nm for nm, _ in items]
    if not all(isinstance(nm, str) for nm in names) or len(set(names)) != len(names):
        raise ValueError("weight names must be distinct strings")
    for name, qw in items:                       # every check before the first byte
        if qw.fmt not in FORMATS:
            raise ValueError(f"{name}: unknown format {qw.fmt!r}")
        for aname, dtype, count in layout(qw.fmt, qw.N, qw.K):
            t = getattr(qw, aname)
            if t is None:
                raise ValueError(f"{name}: the {aname} array is missing")
            if t.dtype != _DTYPES[dtype][1] or t.numel() != count:
                raise ValueError(f"{name}: {aname} must be {dtype} [{count}], got {t.dtype} [{t.numel()}]")
    tmp = f"{path}.tmp{os.getpid()}"
    try:
        with open(tmp, "wb") as f:
            f.write(MAGIC)
            entries = []
            for name, qw in items:
                arrs = []
                for aname, dtype, count in layout(qw.fmt, qw.N, qw.K):
                    host = getattr(qw, aname).detach().contiguous().reshape(-1).cpu().numpy()
                    buf = memoryview(host).cast("B")
                    off = _align(f.tell())
                    f.write(b"\0" * (off - f.tell()))
                    f.write(buf)
                    arrs.append({"name": aname, "dtype": dtype, "count": count, "offset": off,
                                 "crc32": zlib.crc32(buf)})
                entries.append({"name": name, "format": qw.fmt, "N": qw.N, "K": qw.K, "arrays": arrs})
            index = json.dumps({"weights": entries}, separators=(",", ":")).encode()
            f.write(index + struct.pack("<Q", len(index)) + MAGIC)
        os.replace(tmp, path)
    except BaseException:
        if os.path.exists(tmp):
            os.remove(tmp)
        raise


def load(path: str, device="cpu") -> dict[str, QuantWeight]:
    """Read every weight of a file written by save(), in file order, onto `device`."""
    size = os.path.getsize(path)
    with open(path, "rb") as f:
        if size < 2 * len(MAGIC) + 8 or f.read(len(MAGIC)) != MAGIC:
            raise ValueError(f"{path}: not a quantised-weight file")
        f.seek(size - 16)
        tail = f.read(16)
        (jlen,) = struct.unpack("<Q", tail[:8])
        if tail[8:] != MAGIC or jlen > size - 24:
            raise ValueError(f"{path}: truncated or damaged index")
        data_end = size - 16 - jlen
        f.seek(data_end)
        try:
            entries = json.loads(f.read(jlen).decode())["weights"]
            if not isinstance(entries, list) or not all(isinstance(e, dict) for e in entries):
                raise ValueError("weights is not a list of objects")
        except (ValueError, KeyError, TypeError, UnicodeDecodeError) as e:
            raise ValueError(f"{path}: unreadable index ({e})") from None
        out = {}
        for e in entries:
            name, fmt, N, K = e.get("name"), e.get("format"), e.get("N"), e.get("K")
            if not isinstance(name, str) or name in out:
                raise ValueError(f"{path}: missing or repeated weight name {name!r}")
            if fmt not in FORMATS or type(N) is not int or type(K) is not int or N < 1 or K < 1:
                raise ValueError(f"{path}: {name}: bad format or shape")
            got = e.get("arrays")
            if not isinstance(got, list) or not all(isinstance(a, dict) for a in got) or \
                    [(a.get("name"), a.get("dtype"), a.get("count")) for a in got] != layout(fmt, N, K):
                raise ValueError(f"{path}: {name}: arrays do not match the {fmt} layout of [{N}, {K}]")
            tensors = {}
            for a in got:
                off, count = a.get("offset"), a["count"]
                npdt = _DTYPES[a["dtype"]][0]
                nbytes = count * np.dtype(npdt).itemsize
                if type(off) is not int or off < len(MAGIC) or off % ALIGN or off + nbytes > data_end:
                    raise ValueError(f"{path}: {name}.{a['name']}: bad offset")
                host = np.empty(count, dtype=npdt)
                f.seek(off)
                if f.readinto(memoryview(host).cast("B")) != nbytes:
                    raise ValueError(f"{path}: {name}.{a['name']}: short read")
                if zlib.crc32(memoryview(host).cast("B")) != a.get("crc32"):
                    raise ValueError(f"{path}: {name}.{a['name']}: checksum mismatch")
                tensors[a["name"]] = torch.from_numpy(host).to(device)
            out[name] = QuantWeight(fmt, N, K, **tensors)
    return out
