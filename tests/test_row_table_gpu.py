"""Row tables (gathered-only tables with every row's pieces contiguous) on
the GPU vs the CPU oracle, bit for bit.

Method: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
Architecture" (Dev.to abstract), highlight 5 (SpectraFusedEmbedding: the
vocabulary table stays in the 4-bit Group-32 format and the rows a forward
pass needs are gathered and dequantised).  The conversion from a packed
layer is a permutation of its bytes, so every buffer must equal the oracle's
row-table layout of the oracle's packing; a gather from the row table must
return the same values as the gather from the layer, bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import outlier_split_bit_b200 as sp
from outlier_split_bit_b200 import _lib
from outlier_split_bit_b200 import workload as wl

from gpu_helpers import DEV, draw, np_gain, oracle_split, u8, u16, u32

from test_embed_gpu import TABLES, IDS, _expected_bits, _got_bits, _ids

pytestmark = pytest.mark.gpu


def _oracle_table(spec, tau, compact, seed=0):
    w, g, _ = draw(spec, seed=seed)
    lay = sp.pack_layer(w, g, tau, compact=compact)
    wb = wl.bits(w)
    if compact:
        ref = oracle.pack_compact(wb, np_gain(g), tau)
        can = ref.can
    else:
        ref = oracle.pack(wb, np_gain(g), tau)
        can = ref.can
    return lay, wb, ref, oracle.row_table(can, wb, ref.idx)


@pytest.mark.parametrize("compact", [False, True], ids=["masked", "compacted"])
@pytest.mark.parametrize("spec,tau", TABLES, ids=IDS)
def test_row_table_bit_exact(spec, tau, compact):
    lay, wb, ref, rt = _oracle_table(spec, tau, compact)
    table = sp.spectra_row_table_from_layer(lay)
    torch.cuda.synchronize()
    assert np.array_equal(u8(table.codes)[: rt.codes.size], rt.codes)
    assert np.array_equal(u16(table.scales)[: rt.scales.size], rt.scales)
    assert np.array_equal(u32(table.zeros)[: rt.zeros.size], rt.zeros)
    if ref.idx.size:
        assert np.array_equal(u16(table.outlier_w)[: rt.outliers.size], rt.outliers)
    for dtype in (torch.float32, torch.bfloat16):
        for m in (1, 5, 67):
            ids = _ids(spec.n, m, seed=m)
            out = sp.spectra_embed_rows(table, torch.from_numpy(ids).to(DEV), out_dtype=dtype)
            torch.cuda.synchronize()
            rows = oracle.embed_compact(ref, wb, ids) if compact else oracle.embed(ref.can, wb, ref.idx, ids)
            assert np.array_equal(_got_bits(out), _expected_bits(rows, dtype))
    sp.spectra_device_status()


@pytest.mark.parametrize("frac", [0.01, 0.10])
def test_row_table_lm_head_full_size_sampled(frac):
    """The 131072 x 3072 table at tau 3.0 (about half its columns BF16):
    sampled rows of the converted buffers and 96 gathered ids against the
    oracle's reconstruction of those rows."""
    spec = wl.lm_head_spec(frac)
    w, g, _ = draw(spec)
    lay = sp.pack_layer(w, g, 3.0)
    table = sp.spectra_row_table_from_layer(lay)
    wb = wl.bits(w)
    _, ref_idx = oracle_split(wb, np_gain(g), 3.0, key=("lm_head", frac))
    assert np.array_equal(lay.outlier_idx[: lay.n_outliers].cpu().numpy(), ref_idx)
    rng = np.random.default_rng(5)
    ids = np.unique(np.concatenate([[0, 1, spec.n - 1], rng.integers(0, spec.n, 93)])).astype(np.int32)
    sub = np.ascontiguousarray(wb[ids])
    can = oracle.quantize(sub, ref_idx)
    rt = oracle.row_table(can, sub, ref_idx)
    G, S, n_o = spec.k // 32, -(-(spec.k // 32) // 8), ref_idx.size
    codes, scales, zeros, outw = u8(table.codes), u16(table.scales), u32(table.zeros), u16(table.outlier_w)
    for r, i in enumerate(ids):
        assert np.array_equal(codes[i * G * 16:(i + 1) * G * 16], rt.codes[r * G * 16:(r + 1) * G * 16])
        assert np.array_equal(scales[i * G:(i + 1) * G], rt.scales[r * G:(r + 1) * G])
        assert np.array_equal(zeros[i * S:(i + 1) * S], rt.zeros[r * S:(r + 1) * S])
        assert np.array_equal(outw[i * n_o:(i + 1) * n_o], rt.outliers[r * n_o:(r + 1) * n_o])
    out = sp.spectra_embed_rows(table, torch.from_numpy(ids).to(DEV), out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    rows = oracle.embed(can, sub, ref_idx, np.arange(ids.size, dtype=np.int32))
    assert np.array_equal(_got_bits(out), _expected_bits(rows, torch.bfloat16))


@pytest.mark.parametrize("compact", [False, True], ids=["masked", "compacted"])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_row_table_many_rows(compact, dtype):
    """Enough ids for the warp-per-row gather (at least four rows per SM),
    with repeats and the last row, bit for bit against the oracle."""
    spec = wl.MatrixSpec("single", 3000, 1056, 16)
    lay, wb, ref, rt = _oracle_table(spec, 3.0, compact)
    table = sp.spectra_row_table_from_layer(lay)
    ids = _ids(spec.n, 1500, seed=4)
    out = sp.spectra_embed_rows(table, torch.from_numpy(ids).to(DEV), out_dtype=dtype)
    torch.cuda.synchronize()
    sp.spectra_device_status()
    rows = oracle.embed_compact(ref, wb, ids) if compact else oracle.embed(ref.can, wb, ref.idx, ids)
    assert np.array_equal(_got_bits(out), _expected_bits(rows, dtype))


def test_row_table_bad_ids_give_zero_rows_and_status():
    spec = wl.MatrixSpec("single", 64, 256, 4)
    w, g, _ = draw(spec)
    lay = sp.pack_layer(w, g, 3.0)
    table = sp.spectra_row_table_from_layer(lay)
    # few ids (a CTA per row) and many (a warp per row)
    for reps in (1, 200):
        ids = torch.tensor([3, -1, 64, 10] * reps, dtype=torch.int32, device=DEV)
        out = sp.spectra_embed_rows(table, ids, out_dtype=torch.float32)
        torch.cuda.synchronize()
        with pytest.raises(sp.SpectraError) as e:
            sp.spectra_device_status()
        assert e.value.status == _lib.ERR_INVALID_ARG
        assert torch.count_nonzero(out[1]) == 0 and torch.count_nonzero(out[2]) == 0
        ref = sp.spectra_embed(lay, ids[[0, 3]], out_dtype=torch.float32)
        torch.cuda.synchronize()
        sp.spectra_device_status()  # the layer gather of good ids raises nothing
        assert torch.equal(out[[0, 3]], ref)
