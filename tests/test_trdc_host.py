"""The library's TRDC writer and loader on host memory, against the oracle (no GPU).

Source: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
Architecture" (Dev.to abstract), abstract paragraph: one self-contained
binary container holds every weight, scale and offset and is streamed into
memory with a bounded spike.  With host memory the library makes no CUDA
call, so the byte format, the checksums and the chunked staging path are
checked here: files written by the library must equal the oracle's byte for
byte, and the library must load the oracle's files exactly.
"""
import ctypes
import zlib

import numpy as np
import pytest

import oracle
from oracle import trdc
from outlier_split_bit_b200 import _lib
from outlier_split_bit_b200 import build as libbuild
from outlier_split_bit_b200 import workload as wl

BUFS = trdc.BUFFERS


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return _lib.load()


def _layers():
    """Oracle-packed layers: masked and compacted, with and without outliers."""
    out = []
    for name, n, k, n_t, tau, compact in [("layers.0.q", 64, 256, 5, 3.0, False),
                                          ("layers.0.k", 33, 96, 2, 6.0, True),
                                          ("lm_head", 100, 2080, 31, 3.0, True),
                                          ("embed", 40, 64, 0, np.inf, False)]:
        spec = wl.MatrixSpec("single", n, k, n_t)
        wb = wl.bits(wl.weight(spec, seed=n))
        g = wl.gain(spec, seed=n).numpy()
        if compact:
            c = oracle.pack_compact(wb, g, tau)
            e = trdc.entry_from_packed(name, c.packed, tau, c.k_bulk, c.bulk_idx)
        else:
            p = oracle.pack(wb, g, tau)
            e = trdc.entry_from_packed(name, p.packed, tau)
        out.append(e)
    return out


def _arrays(e):
    """Writable numpy copies of an entry's buffers (None where absent)."""
    return {b: (np.frombuffer(e.buffers[b], dtype=np.uint8).copy() if e.buffers.get(b) else None)
            for b in BUFS}


def _view(e, arrs):
    p = {b: (arrs[b].ctypes.data if arrs[b] is not None else None) for b in BUFS}
    return _lib.Layer(e.n, e.k, e.n_outliers, p["codes"], p["scales"], p["zeros"],
                      p["outlier_idx"], p["outlier_w"], e.k_bulk, p["bulk_idx"])


def _write(L, path, entries, staging_bytes):
    keep = [_arrays(e) for e in entries]
    n = len(entries)
    views = (_lib.Layer * n)(*[_view(e, a) for e, a in zip(entries, keep)])
    names = (ctypes.c_char_p * n)(*[e.name.encode() for e in entries])
    taus = (ctypes.c_double * n)(*[e.tau for e in entries])
    stg = np.zeros(max(staging_bytes, 1), dtype=np.uint8)
    return L.spectra_trdc_write(str(path).encode(), n, names, views, taus, _lib.MEM_HOST,
                                stg.ctypes.data if staging_bytes else None, staging_bytes, None)


def _open(L, path):
    h = ctypes.c_void_p()
    st = L.spectra_trdc_open(str(path).encode(), ctypes.byref(h))
    return st, h


def _load(L, h, i, info, staging_bytes, verify=1):
    nb = list(info.bytes)
    dst = {b: (np.zeros(max(int(s), 1), dtype=np.uint8) if s else None) for b, s in zip(BUFS, nb)}
    stg = np.zeros(max(staging_bytes, 1), dtype=np.uint8)
    view = _lib.Layer()
    st = L.spectra_trdc_load(h, i, *[dst[b].ctypes.data if dst[b] is not None else None for b in BUFS],
                             _lib.MEM_HOST, stg.ctypes.data if staging_bytes else None, staging_bytes,
                             verify, ctypes.byref(view), None)
    return st, dst, view


def test_crc32_matches_zlib(L):
    rng = np.random.default_rng(5)
    for n in [0, 1, 7, 8, 9, 63, 64, 4095, 4096, 1 << 20]:
        data = rng.integers(0, 256, n, dtype=np.uint8).tobytes()
        assert L.spectra_crc32(0, data, n) == zlib.crc32(data)
        prev = zlib.crc32(b"prefix")
        assert L.spectra_crc32(prev, data, n) == zlib.crc32(data, prev)


@pytest.mark.parametrize("staging_bytes", [0, 8192, 8192 + 48, 1 << 20])
def test_writer_matches_oracle_bytes(L, tmp_path, staging_bytes):
    entries = _layers()
    path = tmp_path / "model.trdc"
    assert _write(L, path, entries, staging_bytes) == _lib.OK
    assert path.read_bytes() == trdc.write_bytes(entries)


@pytest.mark.parametrize("staging_bytes", [0, 8192, 12288 + 16, 1 << 20])
def test_loader_reads_oracle_file(L, tmp_path, staging_bytes):
    entries = _layers()
    path = tmp_path / "oracle.trdc"
    path.write_bytes(trdc.write_bytes(entries))
    st, h = _open(L, path)
    assert st == _lib.OK
    try:
        assert L.spectra_trdc_count(h) == len(entries)
        for i, e in enumerate(entries):
            info = _lib.TrdcLayer()
            assert L.spectra_trdc_info(h, i, ctypes.byref(info)) == _lib.OK
            assert info.name.decode() == e.name and (info.n, info.k, info.n_outliers) == (e.n, e.k, e.n_outliers)
            assert info.k_bulk == e.k_bulk and info.flags == e.flags and info.tau == e.tau
            st, dst, view = _load(L, h, i, info, staging_bytes)
            assert st == _lib.OK
            for b in BUFS:
                want = e.buffers.get(b, b"")
                got = b"" if dst[b] is None else dst[b][:len(want)].tobytes()
                assert got == want, (e.name, b)
            assert view.n == e.n and view.k_bulk == (e.k_bulk if e.flags else e.k)
            assert (view.bulk_idx is not None) == bool(e.flags)
        info = _lib.TrdcLayer()
        assert L.spectra_trdc_info(h, len(entries), ctypes.byref(info)) == _lib.ERR_INVALID_ARG
    finally:
        L.spectra_trdc_close(h)


def test_damage_is_reported(L, tmp_path):
    entries = _layers()
    data = trdc.write_bytes(entries)
    path = tmp_path / "d.trdc"
    # a flipped byte inside layer 2's codes: the load with verification fails
    off = int(np.frombuffer(data, dtype="<u8", count=1, offset=64 + 256 * 2 + 128)[0])
    bad = bytearray(data)
    bad[off + 100] ^= 0x10
    path.write_bytes(bytes(bad))
    st, h = _open(L, path)
    assert st == _lib.OK
    info = _lib.TrdcLayer()
    L.spectra_trdc_info(h, 2, ctypes.byref(info))
    assert _load(L, h, 2, info, 8192, verify=1)[0] == _lib.ERR_FORMAT
    assert _load(L, h, 2, info, 8192, verify=0)[0] == _lib.OK
    assert _load(L, h, 1, _info(L, h, 1), 0, verify=1)[0] == _lib.OK  # other layers intact
    L.spectra_trdc_close(h)
    # a flipped byte in a layer record, a truncated file, a wrong magic, no file
    for damaged in (data[:70] + bytes([data[70] ^ 1]) + data[71:], data[:-1], b"TRDX" + data[4:]):
        path.write_bytes(damaged)
        assert _open(L, path)[0] == _lib.ERR_FORMAT
    assert _open(L, tmp_path / "missing.trdc")[0] == _lib.ERR_IO


def _info(L, h, i):
    info = _lib.TrdcLayer()
    assert L.spectra_trdc_info(h, i, ctypes.byref(info)) == _lib.OK
    return info


def test_argument_checks(L, tmp_path):
    entries = _layers()[:1]
    path = tmp_path / "a.trdc"
    assert _write(L, path, entries, 4096) == _lib.ERR_BUFFER_TOO_SMALL
    long_name = [trdc.Entry("x" * 96, *[getattr(entries[0], f) for f in
                                        ("n", "k", "n_outliers", "k_bulk", "tau", "flags")],
                            entries[0].buffers)]
    assert _write(L, path, long_name, 0) == _lib.ERR_INVALID_ARG
    views = (_lib.Layer * 1)()
    names = (ctypes.c_char_p * 1)(b"x")
    # device memory needs a staging buffer (checked before any CUDA call)
    assert L.spectra_trdc_write(str(path).encode(), 1, names, views, None, _lib.MEM_DEVICE, None, 0,
                                None) == _lib.ERR_INVALID_ARG
    assert L.spectra_trdc_write(str(path).encode(), 0, names, views, None, _lib.MEM_HOST, None, 0,
                                None) == _lib.ERR_INVALID_ARG
    assert _write(L, path, entries, 0) == _lib.OK
    st, h = _open(L, path)
    info = _info(L, h, 0)
    assert _load(L, h, 0, info, 100)[0] == _lib.ERR_BUFFER_TOO_SMALL
    assert L.spectra_trdc_load(h, 0, None, None, None, None, None, None, _lib.MEM_HOST, None, 0, 1,
                               None, None) == _lib.ERR_INVALID_ARG
    L.spectra_trdc_close(h)
    assert L.spectra_trdc_count(None) == 0
    L.spectra_trdc_close(None)


def test_crc32_of_large_buffers_matches_zlib(L):
    # 4 MB and more are checksummed in slices on several threads and combined
    rng = np.random.default_rng(6)
    for n in [4 << 20, (4 << 20) + 13, (17 << 20) + 5]:
        data = rng.integers(0, 256, n, dtype=np.uint8).tobytes()
        for prev in (0, 0xDEADBEEF):
            assert L.spectra_crc32(prev, data, n) == zlib.crc32(data, prev)


def test_large_buffer_container_round_trip(L, tmp_path):
    # one 8.4 MB code buffer moving through 16 MB staging halves (threaded CRC)
    spec = wl.MatrixSpec("single", 8192, 2080, 31)
    wb = wl.bits(wl.weight(spec, seed=9))
    p = oracle.pack(wb, wl.gain(spec, seed=9).numpy(), 6.0)
    entries = [trdc.entry_from_packed("big", p.packed, 6.0)]
    assert len(entries[0].buffers["codes"]) > 8 << 20
    path = tmp_path / "big.trdc"
    assert _write(L, path, entries, 32 << 20) == _lib.OK
    assert path.read_bytes() == trdc.write_bytes(entries)
    st, h = _open(L, path)
    assert st == _lib.OK
    st, dst, _ = _load(L, h, 0, _info(L, h, 0), 32 << 20)
    L.spectra_trdc_close(h)
    assert st == _lib.OK
    assert dst["codes"].tobytes() == entries[0].buffers["codes"]
