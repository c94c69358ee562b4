"""The C-ABI library loads and exports every symbol that include/spectra.h
declares; host-side argument checks return their status without a GPU.

No test here launches work: every call below fails validation before the
library touches CUDA, so these run on machines without a GPU as well.
"""
import ctypes
import os
import re

import pytest

from outlier_split_bit_b200 import _lib
from outlier_split_bit_b200 import build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "spectra.h")


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return _lib.load()


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SPECTRA_API\s+[^;(]*?\b(spectra_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for must in ["spectra_pack_plan", "spectra_pack", "spectra_unpack", "spectra_gemv",
                 "spectra_gemm_small", "spectra_packed_sizes", "spectra_status_string"]:
        assert must in names


def test_library_exports_every_declared_symbol(L):
    names = _declared()
    assert names
    for name in names:
        assert hasattr(L, name), name
    assert set(names) <= set(_lib.SIGNATURES)


def test_status_strings(L):
    for s in range(10):
        assert L.spectra_status_string(s)
    assert L.spectra_status_string(99) == b"unknown status"
    assert L.spectra_version() >= 100


def test_packed_sizes(L):
    s = _lib.Sizes()
    assert L.spectra_packed_sizes(512, 512, 10, ctypes.byref(s)) == _lib.OK
    assert s.n_pad == 512 and s.codes_bytes == 512 * 256 and s.scales_bytes == 512 * 2 * 2 * 8
    assert s.zeros_bytes == 512 * 2 * 4 and s.outlier_w_bytes == 512 * 16 * 2
    assert s.outlier_idx_bytes == 40
    assert L.spectra_packed_sizes(40, 96, 0, ctypes.byref(s)) == _lib.OK
    assert s.n_pad == 64 and s.scales_bytes == 64 * 8 * 2 and s.outlier_w_bytes == 0
    assert L.spectra_packed_sizes(0, 512, 0, ctypes.byref(s)) == _lib.ERR_SHAPE
    assert L.spectra_packed_sizes(8, 48, 0, ctypes.byref(s)) == _lib.ERR_SHAPE
    assert L.spectra_packed_sizes(8, 64, 65, ctypes.byref(s)) == _lib.ERR_INVALID_ARG
    assert L.spectra_packed_sizes(8, 64, 1, None) == _lib.ERR_INVALID_ARG


def test_workspace_sizes(L):
    assert L.spectra_pack_plan_workspace_size(3072) >= 3072 * 8 + 8
    assert L.spectra_pack_workspace_size() >= 4


FAKE = 0x10000  # never dereferenced: every call below fails its checks first


def _layer(n=64, k=128, n_o=0, off=0):
    return _lib.Layer(n, k, n_o, FAKE + off, FAKE, FAKE, FAKE if n_o else None,
                      FAKE if n_o else None)


def test_gemv_argument_checks(L):
    y = FAKE
    assert L.spectra_gemv(None, FAKE, y, 0, None) == _lib.ERR_INVALID_ARG
    assert L.spectra_gemv(ctypes.byref(_layer(k=100)), FAKE, y, 0, None) == _lib.ERR_SHAPE
    assert L.spectra_gemv(ctypes.byref(_layer(n=0)), FAKE, y, 0, None) == _lib.ERR_SHAPE
    assert L.spectra_gemv(ctypes.byref(_layer(off=8)), FAKE, y, 0, None) == _lib.ERR_ALIGN
    assert L.spectra_gemv(ctypes.byref(_layer()), FAKE + 2, y, 0, None) == _lib.ERR_ALIGN
    assert L.spectra_gemv(ctypes.byref(_layer()), FAKE, FAKE + 2, 0, None) == _lib.ERR_ALIGN
    assert L.spectra_gemv(ctypes.byref(_layer()), None, y, 0, None) == _lib.ERR_INVALID_ARG
    assert L.spectra_gemv(ctypes.byref(_layer()), FAKE, y, 7, None) == _lib.ERR_INVALID_ARG
    bad = _lib.Layer(64, 128, 3, FAKE, FAKE, FAKE, None, None)
    assert L.spectra_gemv(ctypes.byref(bad), FAKE, y, 0, None) == _lib.ERR_INVALID_ARG
    bad = _lib.Layer(64, 128, 200, FAKE, FAKE, FAKE, FAKE, FAKE)
    assert L.spectra_gemv(ctypes.byref(bad), FAKE, y, 0, None) == _lib.ERR_INVALID_ARG


def test_gemm_small_argument_checks(L):
    lay = ctypes.byref(_layer())
    assert L.spectra_gemm_small(lay, FAKE, 0, FAKE, 0, None) == _lib.ERR_SHAPE
    assert L.spectra_gemm_small(lay, FAKE, 33, FAKE, 0, None) == _lib.ERR_SHAPE
    assert L.spectra_gemm_small(lay, FAKE + 4, 4, FAKE, 0, None) == _lib.ERR_ALIGN


def test_pack_argument_checks(L):
    n_o = ctypes.c_int32(-1)
    ws = L.spectra_pack_plan_workspace_size(128)
    assert L.spectra_pack_plan(None, None, 8, 128, 3.0, None, FAKE, ctypes.byref(n_o), FAKE, ws,
                               None) == _lib.ERR_INVALID_ARG
    assert L.spectra_pack_plan(FAKE, None, 8, 120, 3.0, None, FAKE, ctypes.byref(n_o), FAKE, ws,
                               None) == _lib.ERR_SHAPE
    assert L.spectra_pack_plan(FAKE, None, 8, 128, float("nan"), None, FAKE, ctypes.byref(n_o),
                               FAKE, ws, None) == _lib.ERR_INVALID_ARG
    assert L.spectra_pack_plan(FAKE + 2, None, 8, 128, 3.0, None, FAKE, ctypes.byref(n_o), FAKE,
                               ws, None) == _lib.ERR_ALIGN
    assert L.spectra_pack_plan(FAKE, None, 8, 128, 3.0, None, FAKE, ctypes.byref(n_o), FAKE,
                               ws - 1, None) == _lib.ERR_BUFFER_TOO_SMALL
    assert n_o.value == -1  # outputs untouched
    wsb = L.spectra_pack_workspace_size()
    assert L.spectra_pack(FAKE, 8, 128, None, 2, FAKE, FAKE, FAKE, FAKE, FAKE, wsb, None,
                          None) == _lib.ERR_INVALID_ARG
    assert L.spectra_pack(FAKE, 8, 128, None, 0, FAKE, FAKE + 4, FAKE, None, FAKE, wsb, None,
                          None) == _lib.ERR_ALIGN
    assert L.spectra_pack(FAKE, 8, 128, None, 0, FAKE, FAKE, FAKE, None, FAKE, 0, None,
                          None) == _lib.ERR_BUFFER_TOO_SMALL
    assert L.spectra_unpack(None, FAKE, FAKE, FAKE, None) == _lib.ERR_INVALID_ARG


def test_binding_mirrors_the_abi_names():
    import outlier_split_bit_b200 as sp
    for name in ["spectra_pack_plan", "spectra_pack", "spectra_unpack", "spectra_gemv",
                 "spectra_gemm_small", "spectra_packed_sizes", "spectra_status_string"]:
        assert callable(getattr(sp, name))


def test_product_path_does_not_reference_the_oracle():
    pkg = os.path.join(ROOT, "outlier_split_bit_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f
                assert "spectra_ref" not in text, f


def test_embed_argument_checks(L):
    lay = ctypes.byref(_layer())
    assert L.spectra_embed(None, FAKE, 1, FAKE, 0, None) == _lib.ERR_INVALID_ARG
    assert L.spectra_embed(ctypes.byref(_layer(k=100)), FAKE, 1, FAKE, 0, None) == _lib.ERR_SHAPE
    assert L.spectra_embed(lay, FAKE, -1, FAKE, 0, None) == _lib.ERR_SHAPE
    assert L.spectra_embed(lay, FAKE, 1, FAKE, 5, None) == _lib.ERR_INVALID_ARG
    assert L.spectra_embed(lay, None, 1, FAKE, 0, None) == _lib.ERR_INVALID_ARG
    assert L.spectra_embed(lay, FAKE, 1, None, 1, None) == _lib.ERR_INVALID_ARG
    assert L.spectra_embed(lay, FAKE + 2, 1, FAKE, 0, None) == _lib.ERR_ALIGN
    assert L.spectra_embed(lay, FAKE, 1, FAKE + 4, 1, None) == _lib.ERR_ALIGN
    # no rows: nothing to do, and CUDA is never touched (this machine may have no GPU)
    assert L.spectra_embed(lay, None, 0, None, 1, None) == _lib.OK


def test_packed_sizes_compact(L):
    s = _lib.Sizes()
    assert L.spectra_packed_sizes_compact(512, 512, 100, ctypes.byref(s)) == _lib.OK
    assert s.k_bulk == 416 and s.bulk_idx_bytes == 416 * 4
    assert s.codes_bytes == 512 * 416 // 2 and s.scales_bytes == 512 * 2 * 8 * 2
    assert s.zeros_bytes == 512 * 2 * 4 and s.outlier_w_bytes == 512 * 13 * 8 * 2
    assert L.spectra_packed_sizes_compact(40, 96, 96, ctypes.byref(s)) == _lib.OK
    assert s.k_bulk == 32 and s.n_pad == 64  # every column BF16: one all-zero group
    assert L.spectra_packed_sizes_compact(40, 96, 70, ctypes.byref(s)) == _lib.OK
    assert s.k_bulk == 32
    assert L.spectra_packed_sizes_compact(40, 96, 0, ctypes.byref(s)) == _lib.OK
    assert s.k_bulk == 96
    assert L.spectra_packed_sizes(40, 96, 3, ctypes.byref(s)) == _lib.OK
    assert s.k_bulk == 96 and s.bulk_idx_bytes == 0
    assert L.spectra_packed_sizes_compact(40, 96, 97, ctypes.byref(s)) == _lib.ERR_INVALID_ARG


def test_compacted_layer_checks(L):
    y = FAKE
    # a compacted view's k_bulk must be max(32, ceil32(k - n_outliers)): 128 here
    bad = _lib.Layer(64, 128, 3, FAKE, FAKE, FAKE, FAKE, FAKE, 96, FAKE)
    assert L.spectra_gemv(ctypes.byref(bad), FAKE, y, 0, None) == _lib.ERR_INVALID_ARG
    bad = _lib.Layer(64, 128, 40, FAKE, FAKE, FAKE, FAKE, FAKE, 96, FAKE + 4)
    assert L.spectra_gemv(ctypes.byref(bad), FAKE, y, 0, None) == _lib.ERR_ALIGN
    bad = _lib.Layer(64, 128, 3, FAKE, FAKE, FAKE, FAKE, FAKE, 7, None)  # masked: 0 or k
    assert L.spectra_gemv(ctypes.byref(bad), FAKE, y, 0, None) == _lib.ERR_INVALID_ARG
    assert L.spectra_embed(ctypes.byref(bad), FAKE, 1, FAKE, 0, None) == _lib.ERR_INVALID_ARG
    wsb = L.spectra_pack_workspace_size()
    assert L.spectra_pack_compact(FAKE, 8, 128, FAKE, 2, FAKE, FAKE, FAKE, FAKE, None, FAKE, wsb,
                                  None, None) == _lib.ERR_INVALID_ARG
    assert L.spectra_pack_compact(FAKE, 8, 128, FAKE, 2, FAKE, FAKE, FAKE, FAKE, FAKE + 4, FAKE,
                                  wsb, None, None) == _lib.ERR_ALIGN
    assert L.spectra_pack_compact(FAKE, 8, 120, FAKE, 2, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, wsb,
                                  None, None) == _lib.ERR_SHAPE


def test_kv_argument_checks(L):
    cb, sb, zb = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
    assert L.spectra_kv_sizes(2, 128, 100, ctypes.byref(cb), ctypes.byref(sb), ctypes.byref(zb)) == _lib.OK
    assert (cb.value, sb.value, zb.value) == (2 * 100 * 64, 2 * 100 * 4 * 2, 2 * 100 * 4)
    assert L.spectra_kv_sizes(2, 96, 10, ctypes.byref(cb), ctypes.byref(sb), ctypes.byref(zb)) == _lib.OK
    assert L.spectra_kv_sizes(2, 100, 10, ctypes.byref(cb), ctypes.byref(sb), ctypes.byref(zb)) == _lib.ERR_SHAPE
    assert L.spectra_kv_sizes(2, 288, 10, ctypes.byref(cb), ctypes.byref(sb), ctypes.byref(zb)) == _lib.ERR_SHAPE
    kv = _lib.KV(2, 128, 100, FAKE, FAKE, FAKE)
    k = ctypes.byref(kv)
    assert L.spectra_kv_append(k, None, 0, 5, None) == _lib.OK  # nothing to do: no CUDA call
    assert L.spectra_kv_append(k, FAKE, 10, 95, None) == _lib.ERR_SHAPE
    assert L.spectra_kv_append(k, FAKE, 1, -1, None) == _lib.ERR_INVALID_ARG
    assert L.spectra_kv_append(k, FAKE + 1, 1, 0, None) == _lib.ERR_ALIGN
    assert L.spectra_kv_append(ctypes.byref(_lib.KV(2, 128, 100, FAKE + 8, FAKE, FAKE)), FAKE, 1, 0,
                               None) == _lib.ERR_ALIGN
    ws = L.spectra_attention_workspace_size(12, 128, 100)
    assert ws >= 12 * 130 * 4
    att = L.spectra_attention_decode
    other = ctypes.byref(_lib.KV(2, 128, 99, FAKE, FAKE, FAKE))
    assert att(k, other, FAKE, 12, 50, 0.1, FAKE, FAKE, ws, None) == _lib.ERR_SHAPE
    assert att(k, k, FAKE, 13, 50, 0.1, FAKE, FAKE, ws, None) == _lib.ERR_SHAPE  # not a multiple
    assert att(k, k, FAKE, 18, 50, 0.1, FAKE, FAKE, ws, None) == _lib.ERR_SHAPE  # 9 per KV head
    assert att(k, k, FAKE, 12, 0, 0.1, FAKE, FAKE, ws, None) == _lib.ERR_SHAPE
    assert att(k, k, FAKE, 12, 101, 0.1, FAKE, FAKE, ws, None) == _lib.ERR_SHAPE
    assert att(k, k, FAKE, 12, 100, float("nan"), FAKE, FAKE, ws, None) == _lib.ERR_INVALID_ARG
    assert att(k, k, FAKE, 12, 100, 0.1, FAKE, FAKE, ws - 1, None) == _lib.ERR_BUFFER_TOO_SMALL
    assert att(k, k, FAKE, 12, 100, 0.1, FAKE + 2, FAKE, ws, None) == _lib.ERR_ALIGN
    assert att(k, k, None, 12, 100, 0.1, FAKE, FAKE, ws, None) == _lib.ERR_INVALID_ARG


def test_binding_fails_loudly_without_the_library(tmp_path, monkeypatch):
    # no fallback: with the shared library absent, the first call raises
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "libspectra.so"))
    monkeypatch.setattr(_lib, "_lib", None)
    import outlier_split_bit_b200 as sp
    with pytest.raises(ImportError):
        sp.spectra_version()
    with pytest.raises(ImportError):
        sp.spectra_packed_sizes(32, 64, 0)


def test_selftest_wait_argument_checks(L):
    # unknown kinds are rejected on the host, before any CUDA call
    for kind in (-1, 2, 7):
        assert L.spectra_selftest_wait(kind, None) == _lib.ERR_INVALID_ARG


def test_chain_argument_checks(L):
    lay = _lib.Layer(64, 128, 0, FAKE, FAKE, FAKE, None, None, 0, None)
    layers = (_lib.Layer * 1)(lay)
    # the workspace size rejects bad arguments before touching the device
    assert L.spectra_gemv_chain_workspace_size(None, 1) == 0
    assert L.spectra_gemv_chain_workspace_size(layers, 0) == 0
    bad_shape = (_lib.Layer * 1)(_lib.Layer(64, 100, 0, FAKE, FAKE, FAKE, None, None, 0, None))
    assert L.spectra_gemv_chain_workspace_size(bad_shape, 1) == 0
    ws = 16
    xs = (ctypes.c_void_p * 1)(FAKE)
    ys = (ctypes.c_void_p * 1)(FAKE)
    # argument errors come back before any CUDA call
    assert L.spectra_gemv_chain(layers, xs, ys, 1, 0, None, ws, None) == _lib.ERR_INVALID_ARG
    assert L.spectra_gemv_chain(layers, xs, ys, 1, 0, FAKE, ws - 1, None) == _lib.ERR_BUFFER_TOO_SMALL
    ws = 1 << 20
    assert L.spectra_gemv_chain(layers, xs, ys, 1, 0, FAKE + 4, ws, None) == _lib.ERR_ALIGN
    assert L.spectra_gemv_chain(layers, xs, ys, 0, 0, FAKE, ws, None) == _lib.ERR_SHAPE
    assert L.spectra_gemv_chain(layers, xs, ys, _lib.MAX_BATCH + 1, 0, FAKE, ws, None) == _lib.ERR_SHAPE
    assert L.spectra_gemv_chain(layers, xs, ys, 1, 5, FAKE, ws, None) == _lib.ERR_INVALID_ARG
    bad = (_lib.Layer * 1)(_lib.Layer(64, 100, 0, FAKE, FAKE, FAKE, None, None, 0, None))
    assert L.spectra_gemv_chain(bad, xs, ys, 1, 0, FAKE, ws, None) == _lib.ERR_SHAPE


def test_staged_chain_argument_checks(L):
    lay = _lib.Layer(64, 128, 0, FAKE, FAKE, FAKE, None, None, 0, None)
    layers = (_lib.Layer * 3)(lay, lay, lay)
    xs = (ctypes.c_void_p * 3)(FAKE, FAKE, FAKE)
    ys = (ctypes.c_void_p * 3)(FAKE, FAKE, FAKE)
    ws = 1 << 20
    good = (ctypes.c_int32 * 3)(0, 0, 1)
    # the same checks as spectra_gemv_chain, then the stage array: present
    # and nondecreasing; all before any CUDA call
    assert L.spectra_gemv_chain_staged(layers, xs, ys, 3, 0, good, None, ws, None) == _lib.ERR_INVALID_ARG
    assert L.spectra_gemv_chain_staged(layers, xs, ys, 3, 0, good, FAKE, 15, None) == _lib.ERR_BUFFER_TOO_SMALL
    assert L.spectra_gemv_chain_staged(layers, xs, ys, 0, 0, good, FAKE, ws, None) == _lib.ERR_SHAPE
    assert L.spectra_gemv_chain_staged(layers, xs, ys, 3, 0, None, FAKE, ws, None) == _lib.ERR_INVALID_ARG
    down = (ctypes.c_int32 * 3)(0, 1, 0)
    assert L.spectra_gemv_chain_staged(layers, xs, ys, 3, 0, down, FAKE, ws, None) == _lib.ERR_INVALID_ARG


def test_row_table_argument_checks(L):
    lay = _lib.Layer(64, 128, 0, FAKE, FAKE, FAKE, None, None, 0, None)
    sz = _lib.Sizes()
    assert L.spectra_row_table_sizes(ctypes.byref(lay), ctypes.byref(sz)) == _lib.OK
    assert sz.codes_bytes == 64 * 4 * 16 and sz.scales_bytes == 64 * 4 * 2 and sz.zeros_bytes == 64 * 4
    assert sz.outlier_w_bytes == 0 and sz.bulk_idx_bytes == 0
    lay_o = _lib.Layer(64, 128, 5, FAKE, FAKE, FAKE, FAKE, FAKE, 0, None)
    assert L.spectra_row_table_sizes(ctypes.byref(lay_o), ctypes.byref(sz)) == _lib.OK
    assert sz.outlier_w_bytes == 64 * 5 * 2 and sz.outlier_idx_bytes == 5 * 4
    assert L.spectra_row_table_sizes(ctypes.byref(lay), None) == _lib.ERR_INVALID_ARG
    out = _lib.Layer()
    assert L.spectra_row_table_from_layer(ctypes.byref(lay), None, FAKE, FAKE, None, ctypes.byref(out),
                                          None) == _lib.ERR_INVALID_ARG
    assert L.spectra_row_table_from_layer(ctypes.byref(lay), FAKE + 4, FAKE, FAKE, None, ctypes.byref(out),
                                          None) == _lib.ERR_ALIGN
    assert L.spectra_embed_rows(None, FAKE, 1, FAKE, 0, None) == _lib.ERR_INVALID_ARG
    assert L.spectra_embed_rows(ctypes.byref(lay), FAKE, -1, FAKE, 0, None) == _lib.ERR_SHAPE
    assert L.spectra_embed_rows(ctypes.byref(lay), FAKE, 0, FAKE, 0, None) == _lib.OK

