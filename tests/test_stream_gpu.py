"""The decode-step weight stream, launched exactly as the benchmark times it,
against the CPU oracle.

Method: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
Architecture" (Dev.to abstract), abstract paragraph: kurtosis split, Group-32
4-bit bulk with the heavy-tailed channels kept bit-exact in BF16, dequantised
in registers in the decode pass.  The benchmark's step is ONE grouped launch
(spectra_gemv_batched, captured in a CUDA graph and replayed) over the 196
matrices of a 28-layer 1.5B-class stack.  Its persistent CTAs walk item
ranges that cross matrix boundaries, search forward for each item's matrix
and restage x at every matrix change; this file checks that launch, built
by the benchmark's own Stream class, against the oracle: for every matrix,
the outlier indices and the packed bytes of four whole 32-row tiles (the
first two, a middle one and the last, ragged where n is) are identical, and
the matvec on those rows is within |y - y_ref| <= 2e-3 * sum|w_hat x| + 1e-5.
The oracle's split is its own (kurtosis of the whole matrix), never the GPU's.
"""
import numpy as np
import pytest
import torch

import bench
import oracle
from outlier_split_bit_b200 import workload as wl

from gpu_helpers import DEV, check_gemv, np_gain, oracle_rows, oracle_split, tile_slices, u8, u16, u32

pytestmark = pytest.mark.gpu


def _tiles(n):
    T = -(-n // 32)
    return sorted({0, 1, T // 2, T - 1})


def _check_masked(lay, wb, ref_idx, xb, y):
    tiles = _tiles(lay.n)
    rows, can, packed = oracle_rows(wb, ref_idx, tiles)
    got = tile_slices(lay, tiles)
    for key in ("codes", "scales", "zeros", "outliers"):
        assert np.array_equal(got[key], packed[key]), key
    y_ref, bound = oracle.gemm(can, np.ascontiguousarray(wb[rows]), ref_idx, xb)
    return check_gemv(y[rows], y_ref[0], bound[0])


def _check_compact(lay, wb, ref_idx, xb, y):
    kb, bidx = oracle.bulk_columns(wb.shape[1], ref_idx)
    assert lay.k_bulk == kb and np.array_equal(lay.bulk_idx.cpu().numpy(), bidx)
    G, S, O8 = kb // 32, -(-(kb // 32) // 8), -(-ref_idx.size // 8)
    codes, scales, zeros, outw = u8(lay.codes), u16(lay.scales), u32(lay.zeros), u16(lay.outlier_w)
    worst = 0.0
    for t in _tiles(lay.n):
        sub = np.ascontiguousarray(wb[32 * t:32 * t + 32])
        bulk = oracle.gather_bulk(sub, bidx)
        can = oracle.quantize(bulk, np.zeros(0, np.int32))
        p = oracle.pack_layout(can, bulk, np.zeros(0, np.int32))
        assert np.array_equal(codes[t * G * 512:(t + 1) * G * 512], p.codes)
        assert np.array_equal(scales[t * S * 256:(t + 1) * S * 256], p.scales)
        assert np.array_equal(zeros[t * S * 32:(t + 1) * S * 32], p.zeros)
        if O8:
            assert np.array_equal(outw[t * O8 * 256:(t + 1) * O8 * 256],
                                  oracle.pack_outliers(sub, ref_idx))
        part = oracle.CompactLayer(None, ref_idx, kb, bidx, can, None)
        y_ref, bound = oracle.gemm_compact(part, sub, xb)
        worst = max(worst, check_gemv(y[32 * t:32 * t + 32], y_ref[0], bound[0]))
    return worst


@pytest.mark.parametrize("compact", [False, True], ids=["masked", "compacted"])
@pytest.mark.parametrize("tau", [3.0, 6.0])
def test_decode_stream_grouped_launch_against_oracle(tau, compact):
    stream = torch.cuda.Stream()
    st = bench.Stream(torch.device(DEV), seed=0, tau=tau, compact=compact)
    graph, launches = st.capture(stream, "batched")
    assert launches == 1 and len(st.items) == 7 * wl.N_LAYERS_1P5B
    # outputs poisoned, then one replay of the captured step
    st.y_all.fill_(float("nan"))
    torch.cuda.synchronize()
    graph.replay()
    stream.synchronize()
    y_all = st.y_all.cpu()
    worst = 0.0
    for i, (spec, lay, x, y, view) in enumerate(st.items):
        layer = i // len(wl.LAYER_1P5B)
        assert spec is wl.LAYER_1P5B[i % len(wl.LAYER_1P5B)]
        w = wl.weight(spec, 0, layer, device=DEV)
        g = wl.gain(spec, 0, layer, device=DEV)
        wb = wl.bits(w)
        del w
        _, ref_idx = oracle_split(wb, np_gain(g), tau, key=("stream", layer, spec.name))
        assert lay.n_outliers == ref_idx.size, (layer, spec.name)
        if ref_idx.size:
            assert np.array_equal(lay.outlier_idx[: ref_idx.size].cpu().numpy(), ref_idx), (layer, spec.name)
        # this matrix's slice of the stream's output buffer
        off = (y.data_ptr() - st.y_all.data_ptr()) // 4
        yv = y_all[off:off + spec.n]
        assert torch.isfinite(yv).all(), (layer, spec.name)
        xb = wl.bits(x)
        chk = _check_compact if compact else _check_masked
        worst = max(worst, chk(lay, wb, ref_idx, xb, yv))
    assert worst <= 1.0
    del graph, st
    torch.cuda.empty_cache()
