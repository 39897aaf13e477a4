"""WOQC: a file container for packed weights, read by memory map.

The packed tensors of a model live in one file with a table of contents, and every tensor's
data starts on a 64-byte boundary, so that a reader can map the file and use (or copy) each
array in place ("TinyMOSS-Diarize", "How we built it": an mmap container with a
64-byte-aligned tensor table holds the packed tensors). That page names its format MQF1 but
does not give its bytes, so this is a format of this library's own, with its own name.

Layout (all integers little-endian):

  header, 64 bytes
    0   4   magic b"WOQC"
    4   4   u32 version (1)
    8   4   u32 tensor count T
    12  4   u32 entry size (128)
    16  8   u64 offset of the table (64)
    24  8   u64 offset of the first data byte
    32  32  zero
  table, T entries of 128 bytes
    0   64  name, UTF-8, zero-padded (at most 63 bytes)
    64  4   u32 bits (4, 5 or 8)
    68  4   u32 block (32)
    72  8   u64 n (rows, out features)
    80  8   u64 k (columns, in features)
    88  8   u64 offset of the packed codes   (a multiple of 64)
    96  8   u64 offset of the scales         (a multiple of 64)
    104 4   u32 CRC-32 of the packed codes
    108 4   u32 CRC-32 of the scales
    112 16  zero
  data: for each tensor, its codes (n * k * bits / 8 bytes, the layout of include/woq.h) and
  its scales (n * k / 32 binary16 bit patterns, row-major), each at a 64-byte-aligned offset.

Everything here runs on the host; the device sees only the PackedWeight tensors it returns.
"""

from __future__ import annotations

import os
import struct
import zlib

import numpy as np
import torch

MAGIC = b"WOQC"
VERSION = 1
HEADER_BYTES = 64
ENTRY_BYTES = 128
ALIGN = 64
_HEADER = struct.Struct("<4sIIIQQ32x")
_ENTRY = struct.Struct("<64sIIQQQQII16x")


class ContainerError(ValueError):
    """The file is not a well-formed WOQC container, or a checksum does not match."""


def _align(x: int) -> int:
    return (x + ALIGN - 1) // ALIGN * ALIGN


def _host_arrays(w) -> tuple[np.ndarray, np.ndarray]:
    packed = w.packed.detach().to("cpu").contiguous().numpy().view(np.uint8)
    scales = w.scales.detach().to("cpu").contiguous().numpy().view(np.uint16)
    return packed, scales


def save(path: str, weights: dict) -> None:
    """Writes ``weights`` (name -> PackedWeight, on any device) to ``path``."""
    names = list(weights)
    for name in names:
        if len(name.encode()) > 63:
            raise ValueError(f"tensor name longer than 63 bytes: {name!r}")
    table_end = HEADER_BYTES + ENTRY_BYTES * len(names)
    offset = _align(table_end)
    data_start = offset
    entries, blobs = [], []
    for name in names:
        w = weights[name]
        if w.bits not in (4, 5, 8):
            raise ValueError(f"{name}: bits must be 4, 5 or 8")
        packed, scales = _host_arrays(w)
        if packed.size != w.n * w.k * w.bits // 8 or scales.size != w.n * (w.k // 32):
            raise ValueError(f"{name}: array sizes do not match n = {w.n}, k = {w.k}")
        off_p = offset
        off_s = _align(off_p + packed.nbytes)
        offset = _align(off_s + scales.nbytes)
        entries.append(_ENTRY.pack(name.encode(), w.bits, 32, w.n, w.k, off_p, off_s,
                                   zlib.crc32(packed.tobytes()), zlib.crc32(scales.tobytes())))
        blobs.append((off_p, packed.tobytes()))
        blobs.append((off_s, scales.tobytes()))
    with open(path, "wb") as f:
        f.write(_HEADER.pack(MAGIC, VERSION, len(names), ENTRY_BYTES, HEADER_BYTES, data_start))
        for e in entries:
            f.write(e)
        for off, blob in blobs:
            f.write(b"\0" * (off - f.tell()))
            f.write(blob)
        f.write(b"\0" * (offset - f.tell()))


def read_table(path: str) -> list[dict]:
    """The table of contents of ``path``, checked against the file's size."""
    size = os.path.getsize(path)
    with open(path, "rb") as f:
        head = f.read(HEADER_BYTES)
        if len(head) != HEADER_BYTES:
            raise ContainerError("file shorter than the header")
        magic, version, count, entry_bytes, table_off, data_off = _HEADER.unpack(head)
        if magic != MAGIC:
            raise ContainerError("not a WOQC container (bad magic)")
        if version != VERSION or entry_bytes != ENTRY_BYTES or table_off != HEADER_BYTES:
            raise ContainerError(f"unsupported container version {version}")
        f.seek(table_off)
        raw = f.read(ENTRY_BYTES * count)
    if len(raw) != ENTRY_BYTES * count:
        raise ContainerError("table runs past the end of the file")
    table = []
    for i in range(count):
        name, bits, block, n, k, off_p, off_s, crc_p, crc_s = _ENTRY.unpack_from(raw, i * ENTRY_BYTES)
        e = {"name": name.rstrip(b"\0").decode(), "bits": bits, "block": block, "n": n, "k": k,
             "off_packed": off_p, "off_scales": off_s, "crc_packed": crc_p, "crc_scales": crc_s,
             "bytes_packed": n * k * bits // 8, "bytes_scales": n * (k // 32) * 2}
        if bits not in (4, 5, 8) or block != 32 or k % 32 or n < 1:
            raise ContainerError(f"{e['name']}: bad shape or format")
        if off_p % ALIGN or off_s % ALIGN or off_p < data_off or off_s < data_off:
            raise ContainerError(f"{e['name']}: data not 64-byte aligned or inside the table")
        if off_p + e["bytes_packed"] > size or off_s + e["bytes_scales"] > size:
            raise ContainerError(f"{e['name']}: data runs past the end of the file")
        table.append(e)
    return table


def load(path: str, device="cuda", verify: bool = True) -> dict:
    """Maps ``path`` and copies every tensor to ``device`` once: name -> PackedWeight. With
    ``verify`` the CRC-32 of each array is checked first."""
    from . import PackedWeight

    table = read_table(path)
    mm = np.memmap(path, dtype=np.uint8, mode="r")
    out = {}
    for e in table:
        packed = mm[e["off_packed"]:e["off_packed"] + e["bytes_packed"]]
        scales = mm[e["off_scales"]:e["off_scales"] + e["bytes_scales"]]
        if verify and (zlib.crc32(packed) != e["crc_packed"] or zlib.crc32(scales) != e["crc_scales"]):
            raise ContainerError(f"{e['name']}: checksum mismatch")
        n, k, bits = e["n"], e["k"], e["bits"]
        p = torch.from_numpy(np.array(packed).reshape(n, k * bits // 8)).to(device)
        s = torch.from_numpy(np.array(scales).view(np.int16).reshape(n, k // 32)).to(device)
        out[e["name"]] = PackedWeight(p, s, bits, n, k)
    del mm
    return out
