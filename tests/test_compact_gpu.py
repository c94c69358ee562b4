"""Compacted bulk on the GPU vs the CPU oracle.

Method: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
Architecture" (Dev.to abstract), abstract paragraph: the heavy-tailed
coordinates are decoupled into bit-exact BF16 storage and the residual bulk
is quantised; here the outlier columns leave the 4-bit bulk.  Packing
outputs (codes, scales, zero points, bulk column list, outlier block) must be
identical bit for bit; the matvec must satisfy |y - y_ref| <= 2e-3 *
sum_j |w_hat_ij x_j| + 1e-5; the row gather must match bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import outlier_split_bit_b200 as sp
from outlier_split_bit_b200 import workload as wl

from gpu_helpers import DEV, check_gemv, draw, np_gain, oracle_split, u8, u16, u32

pytestmark = pytest.mark.gpu

SMALL = [
    (wl.SINGLE_512, 3.0),
    (wl.SINGLE_512, 6.0),
    (wl.MatrixSpec("single", 40, 96, 3), 1.2),
    (wl.MatrixSpec("single", 7, 352, 17), 3.0),
    (wl.MatrixSpec("single", 1, 32, 0), 3.0),
    (wl.MatrixSpec("single", 33, 64, 2), -np.inf),
    (wl.MatrixSpec("single", 100, 2080, 31), 6.0),
    (wl.MatrixSpec("single", 96, 256, 4), np.inf),
    (wl.MatrixSpec("single", 64, 8960, 134), 3.0),
]
SMALL_IDS = [f"{s.n}x{s.k}-tau{t}" for s, t in SMALL]


def _both(spec, tau, seed=0, m=1):
    w, g, x = draw(spec, seed=seed, m=m)
    lay = sp.pack_layer(w, g, tau, compact=True)
    wb = wl.bits(w)
    ref = oracle.pack_compact(wb, np_gain(g), tau)
    return w, g, x, lay, wb, ref


def _assert_pack_equal(lay, ref):
    assert lay.compact and lay.k_bulk == ref.k_bulk
    assert lay.n_outliers == ref.idx.size
    assert np.array_equal(lay.bulk_idx.cpu().numpy(), ref.bulk_idx)
    p = ref.packed
    assert np.array_equal(u8(lay.codes)[: p.codes.size], p.codes)
    assert np.array_equal(u16(lay.scales)[: p.scales.size], p.scales)
    assert np.array_equal(u32(lay.zeros)[: p.zeros.size], p.zeros)
    if ref.idx.size:
        assert np.array_equal(lay.outlier_idx.cpu().numpy()[: ref.idx.size], ref.idx)
        assert np.array_equal(u16(lay.outlier_w)[: p.outliers.size], p.outliers)


@pytest.mark.parametrize("spec,tau", SMALL, ids=SMALL_IDS)
def test_pack_compact_bit_exact(spec, tau):
    w, g, x, lay, wb, ref = _both(spec, tau)
    _assert_pack_equal(lay, ref)
    codes, scales, zeros = sp.spectra_unpack(lay)
    assert np.array_equal(codes.cpu().numpy(), ref.can.codes)
    assert np.array_equal(scales.cpu().numpy().view(np.uint16), ref.can.scales)
    assert np.array_equal(zeros.cpu().numpy(), ref.can.zeros)


@pytest.mark.parametrize("spec,tau", SMALL, ids=SMALL_IDS)
@pytest.mark.parametrize("ydt", [torch.float32, torch.bfloat16])
def test_gemv_compact_small(spec, tau, ydt):
    w, g, x, lay, wb, ref = _both(spec, tau)
    y = sp.spectra_gemv(lay, x[0], y_dtype=ydt)
    torch.cuda.synchronize()
    y_ref, bound = oracle.gemm_compact(ref, wb, wl.bits(x))
    check_gemv(y, y_ref[0], bound[0], bf16=(ydt == torch.bfloat16))


@pytest.mark.parametrize("spec", wl.LAYER_1P5B, ids=[s.name for s in wl.LAYER_1P5B])
@pytest.mark.parametrize("tau", [3.0, 6.0])
def test_decoder_layer_1p5b_compact(spec, tau):
    w, g, x, lay, wb, ref = _both(spec, tau)
    _assert_pack_equal(lay, ref)
    y = sp.spectra_gemv(lay, x[0])
    torch.cuda.synchronize()
    y_ref, bound = oracle.gemm_compact(ref, wb, wl.bits(x))
    check_gemv(y, y_ref[0], bound[0])
    # fewer bytes than the masked bulk whenever there are outlier columns
    masked = sp.pack_layer(w, g, tau)
    assert lay.nbytes < masked.nbytes or lay.n_outliers < 32


@pytest.mark.parametrize("m", [2, 3, 4, 7, 8, 12, 16, 20, 32])
def test_gemm_small_compact(m):
    """CUDA cores below 8 rows, the tensor cores from 8: both gather x through
    the bulk column list."""
    spec = wl.MatrixSpec("single", 600, 1536, 23)
    for tau in (3.0, 6.0):
        w, g, x, lay, wb, ref = _both(spec, tau, seed=m, m=m)
        y = sp.spectra_gemm_small(lay, x)
        torch.cuda.synchronize()
        sp.spectra_device_status()
        y_ref, bound = oracle.gemm_compact(ref, wb, wl.bits(x))
        check_gemv(y, y_ref, bound)


@pytest.mark.parametrize("m", [1, 4, 16, 32])
def test_compact_unit_vectors_extract_columns_exactly(m):
    """x = e_j: one nonzero product per output.  On the CUDA cores (m < 8) it is
    exact in FP32, so y is column j of the reconstruction; the tensor cores
    (m >= 8) take the bulk weights as FP16 operands, so a bulk column comes
    back as the reconstruction rounded once to FP16 (nearest even), bit for
    bit, and an outlier column exactly."""
    spec = wl.MatrixSpec("single", 200, 1024, 16)
    w, g, x, lay, wb, ref = _both(spec, 3.0)
    what = oracle.dequant(ref.can)  # [n, k_bulk]
    wvals = torch.from_numpy(wb.view(np.int16)).view(torch.bfloat16).double().numpy()
    pos = {int(j): p for p, j in enumerate(ref.bulk_idx) if j >= 0}
    rng = np.random.default_rng(m)
    cols = ([0, 1, 31, 1023] + ref.idx[:4].tolist() + rng.choice(1024, 32, replace=False).tolist())[:m]
    e = torch.zeros((m, 1024), dtype=torch.bfloat16, device=DEV)
    for r, j in enumerate(cols):
        e[r, j] = 1.0
    y = sp.spectra_gemm_small(lay, e).cpu().numpy().astype(np.float64)
    for r, j in enumerate(cols):
        if j in ref.idx:
            expect = wvals[:, j]
        else:
            expect = what[:, pos[j]]
            if m >= 8:
                expect = expect.astype(np.float16).astype(np.float64)
        assert np.array_equal(y[r], expect), (r, j)


def test_batched_mixes_masked_and_compacted():
    """One grouped launch over masked and compacted layers: each result, and
    each single launch of the same layer, within the oracle's tolerance (the
    grouped launch plans each matrix without clusters, so its reduction
    order differs from a lone launch's); replaying the call repeats it bit
    for bit."""
    layers, xs, ys, refs = [], [], [], []
    for i, spec in enumerate(wl.LAYER_1P5B):
        w, g, x = draw(spec, seed=4, layer=i)
        compact = i % 2 == 0
        layers.append(sp.pack_layer(w, g, 3.0, compact=compact))
        xs.append(x[0])
        ys.append(torch.empty(spec.n, device=DEV))
        wb = wl.bits(w)
        refs.append((compact, wb, oracle.pack_compact(wb, np_gain(g), 3.0) if compact
                     else oracle.pack(wb, np_gain(g), 3.0), wl.bits(x)))
    views = sp.spectra_gemv_batched(layers, xs, ys)
    torch.cuda.synchronize()
    for lay, x, y, (compact, wb, ref, xb) in zip(layers, xs, ys, refs):
        single = sp.spectra_gemv(lay, x)
        torch.cuda.synchronize()
        if compact:
            y_ref, bound = oracle.gemm_compact(ref, wb, xb)
        else:
            y_ref, bound = oracle.gemm(ref.can, wb, ref.idx, xb)
        check_gemv(y, y_ref[0], bound[0])
        check_gemv(single, y_ref[0], bound[0])
    y0 = [y.clone() for y in ys]
    sp.spectra_gemv_batched(views=views)
    torch.cuda.synchronize()
    for a, b in zip(y0, ys):
        assert torch.equal(a, b)


@pytest.mark.parametrize("frac", [0.01, 0.10])
def test_lm_head_compact_full_size_sampled(frac):
    """131072 x 3072 at tau 3 (about half the columns BF16): sampled tiles of the
    compacted pack and of the persistent matvec against the oracle."""
    spec = wl.lm_head_spec(frac)
    w, g, x = draw(spec)
    lay = sp.pack_layer(w, g, 3.0, compact=True)
    y = sp.spectra_gemv(lay, x[0])
    torch.cuda.synchronize()
    wb = wl.bits(w)
    _, ref_idx = oracle_split(wb, np_gain(g), 3.0, key=("lm_head", frac))
    assert np.array_equal(lay.outlier_idx[: lay.n_outliers].cpu().numpy(), ref_idx)
    kb, bidx = oracle.bulk_columns(spec.k, ref_idx)
    assert lay.k_bulk == kb and np.array_equal(lay.bulk_idx.cpu().numpy(), bidx)
    T = spec.n // 32
    G, S, O8 = kb // 32, -(-(kb // 32) // 8), -(-ref_idx.size // 8)
    codes, scales, zeros, outw = u8(lay.codes), u16(lay.scales), u32(lay.zeros), u16(lay.outlier_w)
    for t in (0, 1, T // 2, T - 1):
        sub = np.ascontiguousarray(wb[32 * t:32 * t + 32])
        can = oracle.quantize(oracle.gather_bulk(sub, bidx), np.zeros(0, np.int32))
        p = oracle.pack_layout(can, oracle.gather_bulk(sub, bidx), np.zeros(0, np.int32))
        assert np.array_equal(codes[t * G * 512:(t + 1) * G * 512], p.codes)
        assert np.array_equal(scales[t * S * 256:(t + 1) * S * 256], p.scales)
        assert np.array_equal(zeros[t * S * 32:(t + 1) * S * 32], p.zeros)
        assert np.array_equal(outw[t * O8 * 256:(t + 1) * O8 * 256], oracle.pack_outliers(sub, ref_idx))
        part = oracle.CompactLayer(None, ref_idx, kb, bidx, can, None)
        y_ref, bound = oracle.gemm_compact(part, sub, wl.bits(x))
        check_gemv(y[32 * t:32 * t + 32], y_ref[0], bound[0])


@pytest.mark.parametrize("spec,tau", SMALL[:6] + SMALL[8:], ids=SMALL_IDS[:6] + SMALL_IDS[8:])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_embed_compact_bit_exact(spec, tau, dtype):
    w, g, x, lay, wb, ref = _both(spec, tau)
    rng = np.random.default_rng(3)
    ids = rng.integers(0, spec.n, 9).astype(np.int32)
    ids[0] = spec.n - 1
    out = sp.spectra_embed(lay, torch.from_numpy(ids).to(DEV), out_dtype=dtype)
    torch.cuda.synchronize()
    sp.spectra_device_status()
    rows = oracle.embed_compact(ref, wb, ids)
    got = out.cpu()
    if dtype == torch.float32:
        assert np.array_equal(got.numpy().view(np.uint32), rows.astype(np.float32).view(np.uint32))
    else:
        assert np.array_equal(got.view(torch.int16).numpy().view(np.uint16), oracle.double_to_bf16(rows))
