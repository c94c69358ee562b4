"""TRDC container, written and read from its definition (test infrastructure).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: the tests and the
benchmark's checks use it to say what bytes a container must hold; the
library never imports it.  It shares no code with the library's container
writer and reader (``outlier_split_bit_b200/csrc/trdc.cpp``).

Source: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
Architecture" (Dev.to abstract), abstract paragraph: weights, scales and
offsets live in one self-contained binary container (TRDC) that is streamed
into GPU memory with a bounded memory spike.  The pages give no byte
format; this is the repository's, field by field (little-endian):

  header, 64 bytes: b"TRDC", u32 version = 1, u32 layer count L,
      u32 header bytes 64 + 256 L, u64 file bytes, u32 CRC-32 of the layer
      records, then zeros up to byte 64;
  L records of 256 bytes: name (96 bytes, NUL-padded, < 96 characters),
      i32 n, k, n_outliers, k_bulk (0 for a masked bulk), f64 tau, u32 flags
      (bit 0: compacted bulk), u32 0, six (u64 offset, u64 bytes) pairs for
      codes, scales, zeros, outlier_idx, outlier_w, bulk_idx, six u32 CRC-32
      of those buffers, u64 0;
  buffers, each at the first multiple of 4096 at or after the end of the
      previous one (the first after the records), zero bytes between them;
      absent buffers have offset, bytes and CRC 0; the file ends with the
      last buffer.

CRC-32 is zlib's (IEEE polynomial, reflected, initial and final XOR
0xFFFFFFFF).
"""
from __future__ import annotations

import struct
import zlib
from dataclasses import dataclass, field

BUFFERS = ("codes", "scales", "zeros", "outlier_idx", "outlier_w", "bulk_idx")
ALIGN = 4096
HEADER_BYTES = 64
RECORD_BYTES = 256
VERSION = 1


class FormatError(ValueError):
    pass


def _align(x: int) -> int:
    return (x + ALIGN - 1) // ALIGN * ALIGN


def crc32(data: bytes) -> int:
    return zlib.crc32(data) & 0xFFFFFFFF


@dataclass
class Entry:
    name: str
    n: int
    k: int
    n_outliers: int
    k_bulk: int          # 0 for a masked bulk
    tau: float
    flags: int           # bit 0: compacted bulk
    buffers: dict = field(default_factory=dict)  # buffer name -> bytes (absent: missing or empty)


def entry_from_packed(name, packed, tau, k_bulk=0, bulk_idx=None) -> Entry:
    """An Entry from the oracle's packed arrays (``oracle.Packed``)."""
    bufs = {"codes": packed.codes.tobytes(), "scales": packed.scales.tobytes(),
            "zeros": packed.zeros.tobytes()}
    if packed.idx.size:
        bufs["outlier_idx"] = packed.idx.astype("<i4").tobytes()
        bufs["outlier_w"] = packed.outliers.tobytes()
    if bulk_idx is not None:
        bufs["bulk_idx"] = bulk_idx.astype("<i4").tobytes()
    return Entry(name, packed.n, packed.k, int(packed.idx.size), k_bulk, float(tau),
                 1 if bulk_idx is not None else 0, bufs)


def write_bytes(entries) -> bytes:
    """The container of `entries`, as bytes."""
    L = len(entries)
    header_bytes = HEADER_BYTES + RECORD_BYTES * L
    pos = header_bytes
    placed = []
    for e in entries:
        slots = []
        for b in BUFFERS:
            data = e.buffers.get(b, b"")
            if len(data) == 0:
                slots.append((0, 0, 0))
                continue
            off = _align(pos)
            slots.append((off, len(data), crc32(data)))
            pos = off + len(data)
        placed.append(slots)
    file_bytes = pos
    records = b""
    for e, slots in zip(entries, placed):
        name = e.name.encode()
        if len(name) >= 96:
            raise FormatError("name too long")
        rec = struct.pack("<96s4idII", name, e.n, e.k, e.n_outliers, e.k_bulk, e.tau, e.flags, 0)
        for off, size, _ in slots:
            rec += struct.pack("<QQ", off, size)
        for _, _, c in slots:
            rec += struct.pack("<I", c)
        rec += struct.pack("<Q", 0)
        assert len(rec) == RECORD_BYTES
        records += rec
    head = struct.pack("<4sIIIQII", b"TRDC", VERSION, L, header_bytes, file_bytes, crc32(records), 0)
    head += b"\0" * (HEADER_BYTES - len(head))
    out = bytearray(file_bytes)
    out[:HEADER_BYTES] = head
    out[HEADER_BYTES:header_bytes] = records
    for e, slots in zip(entries, placed):
        for b, (off, size, _) in zip(BUFFERS, slots):
            if size:
                out[off:off + size] = e.buffers[b]
    return bytes(out)


def read_bytes(data: bytes, verify: bool = True):
    """Parse a container; returns the list of Entry with their buffers."""
    if len(data) < HEADER_BYTES:
        raise FormatError("short header")
    magic, ver, L, header_bytes, file_bytes, rcrc, _ = struct.unpack_from("<4sIIIQII", data, 0)
    if magic != b"TRDC" or ver != VERSION:
        raise FormatError("not a TRDC version 1 container")
    if header_bytes != HEADER_BYTES + RECORD_BYTES * L or file_bytes != len(data):
        raise FormatError("header sizes")
    records = data[HEADER_BYTES:header_bytes]
    if crc32(records) != rcrc:
        raise FormatError("record checksum")
    out = []
    for i in range(L):
        base = HEADER_BYTES + RECORD_BYTES * i
        name, n, k, n_o, kb, tau, flags, _ = struct.unpack_from("<96s4idII", data, base)
        slots = [struct.unpack_from("<QQ", data, base + 128 + 16 * j) for j in range(6)]
        crcs = struct.unpack_from("<6I", data, base + 224)
        bufs = {}
        for b, (off, size), c in zip(BUFFERS, slots, crcs):
            if size == 0:
                continue
            if off % ALIGN or off + size > len(data):
                raise FormatError("buffer placement")
            chunk = data[off:off + size]
            if verify and crc32(chunk) != c:
                raise FormatError(f"checksum of {b} in layer {i}")
            bufs[b] = chunk
        out.append(Entry(name.rstrip(b"\0").decode(), n, k, n_o, kb, tau, flags, bufs))
    return out
