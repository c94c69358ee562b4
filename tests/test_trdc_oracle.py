"""Pins of the oracle's TRDC container writer and reader (no GPU).

Source: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
Architecture" (Dev.to abstract), abstract paragraph: one self-contained
binary container holds every weight, scale and offset.  The byte format is
the repository's; these tests pin the oracle's writer to hand-derived field
offsets (tests/golden/trdc_layout.txt), its checksum to the standard CRC-32
check value, and its reader to its writer.
"""
import os
import struct

import numpy as np
import pytest

from oracle import trdc


def _entry(name, n, k, n_o, compact, seed=0):
    from oracle import layout_sizes
    rng = np.random.default_rng(seed)
    kb = max(32, -(-(k - n_o) // 32) * 32) if compact else k
    sz = layout_sizes(n, kb, n_o)
    bufs = {"codes": rng.integers(0, 256, sz["codes"], dtype=np.uint8).tobytes(),
            "scales": rng.integers(0, 1 << 16, sz["scales"], dtype=np.uint16).tobytes(),
            "zeros": rng.integers(0, 1 << 32, sz["zeros"], dtype=np.uint32).tobytes()}
    if n_o:
        bufs["outlier_idx"] = np.sort(rng.choice(k, n_o, replace=False)).astype("<i4").tobytes()
        O8 = -(-n_o // 8)
        bufs["outlier_w"] = rng.integers(0, 1 << 16, sz["n_pad"] * O8 * 8, dtype=np.uint16).tobytes()
    if compact:
        bufs["bulk_idx"] = rng.integers(-1, k, kb).astype("<i4").tobytes()
    return trdc.Entry(name, n, k, n_o, kb if compact else 0, 3.0, 1 if compact else 0, bufs)


def test_crc32_check_value():
    assert trdc.crc32(b"123456789") == 0xCBF43926  # the CRC-32 catalogue's check value
    assert trdc.crc32(b"") == 0


def test_layout_matches_hand_derivation(golden_dir):
    files = {"A": trdc.write_bytes([_entry("t", 1, 32, 0, False)]),
             "C": trdc.write_bytes([_entry("c", 33, 64, 3, True)])}
    fmt = {"u8": "<B", "u32": "<I", "i32": "<i", "u64": "<Q"}
    checked = 0
    for line in open(os.path.join(golden_dir, "trdc_layout.txt")):
        if line.startswith("#") or not line.strip():
            continue
        case, off, typ, val = line.split()[:4]
        data, off = files[case], int(off)
        if typ == "magic":
            assert data[off:off + 4] == val.encode()
        else:
            assert struct.unpack_from(fmt[typ], data, off)[0] == int(val), line
        checked += 1
    assert checked >= 30
    assert len(files["A"]) == 12416 and len(files["C"]) == 24832


def test_round_trip_and_alignment():
    entries = [_entry("layers.0.q", 64, 256, 5, False, 1), _entry("layers.0.k", 33, 96, 0, True, 2),
               _entry("lm_head", 100, 2080, 40, True, 3)]
    data = trdc.write_bytes(entries)
    back = trdc.read_bytes(data)
    assert [e.name for e in back] == [e.name for e in entries]
    for a, b in zip(entries, back):
        assert (a.n, a.k, a.n_outliers, a.k_bulk, a.tau, a.flags) == \
            (b.n, b.k, b.n_outliers, b.k_bulk, b.tau, b.flags)
        assert {k: v for k, v in a.buffers.items() if v} == b.buffers
    for i in range(3):
        for j in range(6):
            off, size = struct.unpack_from("<QQ", data, 64 + 256 * i + 128 + 16 * j)
            assert off % 4096 == 0 and (size == 0) == (off == 0)


def test_reader_rejects_damage():
    data = bytearray(trdc.write_bytes([_entry("x", 40, 96, 3, False)]))
    bad = bytearray(data)
    bad[5000] ^= 1  # inside the codes buffer
    with pytest.raises(trdc.FormatError):
        trdc.read_bytes(bytes(bad))
    trdc.read_bytes(bytes(bad), verify=False)  # checksums are the only guard there
    bad = bytearray(data)
    bad[100] ^= 1  # inside the layer record
    with pytest.raises(trdc.FormatError):
        trdc.read_bytes(bytes(bad))
    with pytest.raises(trdc.FormatError):
        trdc.read_bytes(bytes(data[:-1]))
    with pytest.raises(trdc.FormatError):
        trdc.read_bytes(b"TRDX" + bytes(data[4:]))
