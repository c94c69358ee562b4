"""Pins of the CPU oracle against closed forms, library routines and brute force.

Method: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
Architecture" (Dev.to abstract re-post), abstract paragraph -- kurtosis
saliency with threshold 3.0, bit-exact BF16 outlier channels, Group-32 4-bit
bulk with scale and bit-packed zero point.  None of these checks calls the
GPU library.
"""
import math
import os

import numpy as np
import pytest
import scipy.stats
import torch

from outlier_split_bit_b200 import workload as wl


def _bf16_bits(a: np.ndarray) -> np.ndarray:
    """float array -> BF16 bits (RNE) via torch, an independent library path."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _bf16_values(bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()


# ----------------------------------------------------------------- numbers

def test_bf16_to_double_matches_torch(ref):
    allb = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = ref.bf16_to_double(allb)
    lib = _bf16_values(allb)
    same = (ours == lib) | (np.isnan(ours) & np.isnan(lib))
    assert same.all()


def test_fp16_to_double_matches_numpy(ref):
    allb = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = ref.fp16_to_double(allb)
    lib = allb.view(np.float16).astype(np.float64)
    same = (ours == lib) | (np.isnan(ours) & np.isnan(lib))
    assert same.all()


def test_fp16_roundtrip_every_finite_value(ref):
    allb = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    finite = (allb & 0x7C00) != 0x7C00
    back = ref.double_to_fp16(ref.fp16_to_double(allb[finite]))
    assert np.array_equal(back, allb[finite])


def test_fp16_midpoints_match_numpy(ref):
    # every midpoint between adjacent positive finite FP16 values, and the
    # doubles one ulp either side of it: one RNE step decides all three
    pos = np.arange(0, 0x7BFF, dtype=np.uint16)
    lo = pos.view(np.float16).astype(np.float64)
    hi = (pos + 1).astype(np.uint16).view(np.float16).astype(np.float64)
    mid = (lo + hi) / 2.0  # exact in double
    vals = np.concatenate([mid, np.nextafter(mid, -np.inf), np.nextafter(mid, np.inf)])
    vals = np.concatenate([vals, -vals])
    ours = ref.double_to_fp16(vals)
    lib = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, lib)


def test_fp16_random_doubles_match_numpy(ref):
    rng = np.random.default_rng(7)
    e = rng.uniform(-30, 17, 40000)
    vals = np.exp2(e) * rng.choice([-1.0, 1.0], e.size)
    ours = ref.double_to_fp16(vals)
    with np.errstate(over="ignore"):
        lib = vals.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, lib)


def test_fp16_golden_cases(ref, golden_dir):
    for line in open(os.path.join(golden_dir, "fp16_rounding_cases.txt")):
        line = line.split("#")[0].strip() if not line.lstrip().startswith("#") else ""
        if not line:
            continue
        expr, hexbits = line.split()[:2]
        v = float(eval(expr, {"__builtins__": {}}))
        assert int(ref.double_to_fp16([v])[0]) == int(hexbits, 16), expr


# ----------------------------------------------------------------- kurtosis

def _column(values: np.ndarray) -> np.ndarray:
    return _bf16_bits(np.asarray(values, dtype=np.float32).reshape(-1, 1))


def test_kurtosis_closed_forms(ref, golden_dir):
    rows = 0
    for line in open(os.path.join(golden_dir, "kurtosis_closed_forms.txt")):
        f = line.split("#")[0].split()
        if not f:
            continue
        if f[0] == "const":
            n, v = int(f[1]), float(f[2])
            col = np.full(n, v)
            expect = 0.0
        else:
            n, m, a, expect = int(f[0]), int(f[1]), float(f[2]), float(f[3])
            col = np.zeros(n)
            col[:m] = a
            col[m:2 * m] = -a
            np.random.default_rng(n + m).shuffle(col)
        kap = ref.kurtosis(_column(col), None)
        assert kap[0] == expect, (line, kap[0])
        rows += 1
    assert rows >= 9


def test_kurtosis_matches_scipy_with_gain(ref):
    rng = np.random.default_rng(1)
    n, k = 300, 24
    w = _bf16_bits(rng.standard_t(4, (n, k)) * 0.02)
    g = (1.0 + 0.1 * rng.standard_normal(k)).astype(np.float32)
    ours = ref.kurtosis(w, g)
    a = _bf16_values(w) * g.astype(np.float64)
    lib = scipy.stats.kurtosis(a, axis=0, fisher=False, bias=True)
    np.testing.assert_allclose(ours, lib, rtol=1e-12)
    # the gain is a per-column constant factor; kurtosis is scale invariant
    np.testing.assert_allclose(ours, ref.kurtosis(w, None), rtol=1e-12)


def test_kurtosis_gaussian_is_three(ref):
    rng = np.random.default_rng(2)
    n = 1_000_000
    kap = ref.kurtosis(_column(rng.standard_normal(n)), None)[0]
    assert abs(kap - 3.0) <= 5 * math.sqrt(24.0 / n)


@pytest.mark.slow
def test_kurtosis_student_t5_is_nine(ref):
    # Student-t with nu = 5: Pearson kurtosis 3 + 6/(nu - 4) = 9; the eighth
    # moment is infinite, so the sample value converges slowly (loose band).
    vals = []
    for s in range(5):
        rng = np.random.default_rng(100 + s)
        vals.append(ref.kurtosis(_column(rng.standard_t(5, 10_000_000)), None)[0])
    assert 7.5 <= float(np.median(vals)) <= 10.5


def test_kurtosis_shift_and_scale_invariance(ref):
    rng = np.random.default_rng(3)
    base = rng.integers(-60, 60, 4096).astype(np.float64) / 64.0   # exact in BF16
    k0 = ref.kurtosis(_column(base), None)[0]
    k1 = ref.kurtosis(_column(base * 4.0), None)[0]
    k2 = ref.kurtosis(_column(base + 1.0), None)[0]
    g = np.array([3.0], dtype=np.float32)
    k3 = ref.kurtosis(_column(base), g)[0]
    for kk in (k1, k2, k3):
        assert abs(kk - k0) <= 1e-12 * k0


def test_kurtosis_nonfinite_rejected(ref):
    w = _column(np.ones(8))
    w[3, 0] = 0x7FC0  # BF16 NaN
    with pytest.raises(ref.OracleError) as e:
        ref.kurtosis(w, None)
    assert e.value.status == ref.ERR_NONFINITE
    with pytest.raises(ref.OracleError):
        ref.kurtosis(_column(np.ones(8)), np.array([np.inf], dtype=np.float32))


def test_split_strict_and_ascending(ref):
    kap = np.array([3.0, 3.5, 2.0, 9.0, 3.0000000000000004, np.nan, 0.0])
    assert ref.split(kap, 3.0).tolist() == [1, 3, 4]
    assert ref.split(kap, -np.inf).tolist() == [0, 1, 2, 3, 4, 6]
    assert ref.split(kap, np.inf).tolist() == []
    rng = np.random.default_rng(4)
    kap = rng.uniform(0, 6, 1000)
    assert np.array_equal(ref.split(kap, 3.0), np.flatnonzero(kap > 3.0))


def test_split_picks_heavy_tailed_columns(ref):
    # pages: heavy-tailed channels (kurtosis above threshold) leave the 4-bit
    # bulk.  With the excess reading (Pearson > 6) Gaussian columns never pass
    # and Student-t(3) columns of 512 rows nearly always do.
    spec = wl.SINGLE_512
    w = wl.weight(spec)
    wb = wl.bits(w)
    kap = ref.kurtosis(wb, wl.gain(spec).numpy())
    idx6 = ref.split(kap, 6.0)
    # the injected columns are those with the largest kurtosis
    heavy = np.argsort(kap)[-spec.n_t:]
    assert set(idx6.tolist()) <= set(heavy.tolist())
    assert len(idx6) >= spec.n_t - 2
    # literal 3.0 threshold: about half the Gaussian columns exceed it
    n3 = len(ref.split(kap, 3.0))
    assert 0.3 * spec.k < n3 < 0.7 * spec.k


# ----------------------------------------------------------------- quantiser

def _grid_row(S: float, z: int, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    k = rng.integers(-z, 16 - z, 32).astype(np.float64)
    k[0], k[1] = -z, 15 - z  # both ends of the grid present
    rng.shuffle(k)
    return k * S


@pytest.mark.parametrize("S,z", [(2.0 ** -7, 5), (3 * 2.0 ** -8, 0), (2.0 ** -3, 15), (5 * 2.0 ** -10, 7)])
def test_quantizer_exact_grid(ref, S, z):
    vals = np.stack([_grid_row(S, z, s) for s in range(4)])
    w = _bf16_bits(vals)
    assert np.array_equal(_bf16_values(w), vals)  # the grid is exact in BF16
    can = ref.quantize(w, np.array([], dtype=np.int32))
    assert np.all(can.scales == np.float16(S).view(np.uint16))
    assert np.all(can.zeros == z)
    assert np.array_equal(can.codes.astype(np.int64), np.rint(vals / S).astype(np.int64) + z)
    assert np.array_equal(ref.dequant(can), vals)


def test_quantizer_half_even_ties(ref):
    S = 2.0 ** -6
    # lo = -7S, hi = 8S -> S exact, z = 7; the other values sit on half steps
    half = [0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 3.5, 4.5, -3.5, 6.5, 5.5, -4.5]
    expect_rint = [0, 2, 2, 0, -2, -2, 4, 4, -4, 6, 6, -4]
    row = np.zeros(32)
    row[0], row[1] = -7 * S, 8 * S
    row[2:2 + len(half)] = np.array(half) * S
    can = ref.quantize(_bf16_bits(row[None, :]), np.array([], dtype=np.int32))
    assert can.zeros[0, 0] == 7
    assert can.codes[0, 2:2 + len(half)].astype(int).tolist() == [7 + e for e in expect_rint]
    assert can.codes[0, 0] == 0 and can.codes[0, 1] == 15


def test_quantizer_invariants_random(ref):
    rng = np.random.default_rng(5)
    n, k = 64, 256
    vals = rng.standard_normal((n, k)) * 0.02
    vals[:, 7] = rng.standard_t(3, n)  # a heavy column, masked below
    w = _bf16_bits(vals)
    idx = np.array([7, 100], dtype=np.int32)
    can = ref.quantize(w, idx)
    assert can.codes.max() <= 15 and can.zeros.max() <= 15
    wv = _bf16_values(w)
    bulk = wv.copy()
    bulk[:, idx] = 0.0
    what = ref.dequant(can)
    assert np.all(what[:, idx] == 0.0)
    # scale = FP16(range / 15) with NumPy's own FP16 rounding
    g = bulk.reshape(n, k // 32, 32)
    rngs = g.max(-1) - g.min(-1)
    assert np.array_equal(can.scales, (rngs / 15.0).astype(np.float16).view(np.uint16))
    S = can.scales.view(np.float16).astype(np.float64)
    Srep = np.repeat(S, 32, axis=1)
    err = np.abs(what - bulk)
    straddle = np.repeat((g.min(-1) <= 0) & (g.max(-1) >= 0), 32, axis=1)
    unclamped = (can.codes > 0) & (can.codes < 15)
    assert np.all(err[straddle & unclamped] <= Srep[straddle & unclamped] / 2)
    # clamping at 15 can only add the FP16 rounding of the scale (<= 15 * 2^-11 / (1 - 2^-11) steps)
    assert np.all(err[straddle] <= Srep[straddle] * (0.5 + 15 * 2.0 ** -11 / (1 - 2.0 ** -11)))
    # codes are monotone in w inside every group
    cg = can.codes.reshape(n, k // 32, 32).astype(int)
    order = np.argsort(g, axis=-1, kind="stable")
    assert np.all(np.diff(np.take_along_axis(cg, order, -1), axis=-1) >= 0)


def test_quantizer_degenerate_groups(ref):
    row = np.zeros((2, 64))
    row[0, :32] = -0.0
    row[0, 5] = 0.0
    row[1, 32:] = 0.25  # constant group: range 0 -> scale 0
    can = ref.quantize(_bf16_bits(row), np.array([], dtype=np.int32))
    assert np.all(can.scales == 0) and np.all(can.zeros == 0) and np.all(can.codes == 0)


def test_quantizer_errors(ref):
    big = np.zeros((1, 32))
    big[0, 0], big[0, 1] = 2.0 ** 20, -2.0 ** 20  # range/15 > 65504
    with pytest.raises(ref.OracleError) as e:
        ref.quantize(_bf16_bits(big), np.array([], dtype=np.int32))
    assert e.value.status == ref.ERR_RANGE
    with pytest.raises(ref.OracleError) as e:
        ref.quantize(np.zeros((2, 48), dtype=np.uint16), np.array([], dtype=np.int32))
    assert e.value.status == ref.ERR_SHAPE
    nanw = np.zeros((1, 32), dtype=np.uint16)
    nanw[0, 3] = 0x7F80
    with pytest.raises(ref.OracleError) as e:
        ref.quantize(nanw, np.array([], dtype=np.int32))
    assert e.value.status == ref.ERR_NONFINITE


def test_quantizer_outlier_column_escapes_range_error(ref):
    big = np.zeros((1, 32))
    big[0, 0], big[0, 1] = 2.0 ** 20, -2.0 ** 20
    can = ref.quantize(_bf16_bits(big), np.array([0, 1], dtype=np.int32))
    assert np.all(can.scales == 0)


# ----------------------------------------------------------------- layout

def _random_canonical(ref, n, k, seed):
    rng = np.random.default_rng(seed)
    G = k // 32
    return ref.Canonical(rng.integers(0, 16, (n, k)).astype(np.uint8),
                         rng.integers(0, 0x7C00, (n, G)).astype(np.uint16),
                         rng.integers(0, 16, (n, G)).astype(np.uint8))


@pytest.mark.parametrize("n,k,n_o", [(40, 96, 9), (32, 256, 0), (7, 352, 17), (64, 32, 1)])
def test_layout_roundtrip(ref, n, k, n_o):
    can = _random_canonical(ref, n, k, n + k)
    rng = np.random.default_rng(n_o)
    w = rng.integers(0, 0x7F00, (n, k)).astype(np.uint16)
    idx = np.sort(rng.choice(k, n_o, replace=False)).astype(np.int32)
    p = ref.pack_layout(can, w, idx)
    sz = ref.layout_sizes(n, k, n_o)
    np_ = sz["n_pad"]
    G, S, O8 = k // 32, -(-(k // 32) // 8), -(-n_o // 8)
    assert p.codes.size == np_ * k // 2 and p.scales.size == np_ * S * 8
    assert p.zeros.size == np_ * S and p.outliers.size == np_ * O8 * 8
    back = ref.unpack_layout(p)
    assert np.array_equal(back.codes, can.codes)
    assert np.array_equal(back.scales, can.scales)
    assert np.array_equal(back.zeros, can.zeros)
    # bytes per bulk weight: 4 + 16/32 + 4/32 bits = 4.625 bits when G % 8 == 0
    if G % 8 == 0:
        total_bits = 8 * (p.codes.nbytes + p.scales.nbytes + p.zeros.nbytes)
        assert total_bits == np_ * k * 4.625
    # outlier block carries exact BF16 copies; padding is zero
    ob = p.outliers.reshape(np_ // 32, max(O8, 1) if O8 else 0, 32, 8) if O8 else None
    if O8:
        for i in range(n):
            for o in range(n_o):
                assert ob[i // 32, o // 8, i % 32, o % 8] == w[i, idx[o]]
        assert np.all(ob.transpose(0, 2, 1, 3).reshape(np_, O8 * 8)[n:] == 0)
        assert np.all(ob.transpose(0, 2, 1, 3).reshape(np_, O8 * 8)[:, n_o:] == 0)


def test_layout_golden_offsets(ref, golden_dir):
    n, k, n_o = 40, 96, 9
    lines = [l.split("#")[0].split() for l in open(os.path.join(golden_dir, "layout_offsets.txt"))]
    lines = [l for l in lines if l]
    for kind, row, col, off, nib in lines:
        row, col, off = int(row), int(col), int(off)
        can = ref.Canonical(np.zeros((n, k), np.uint8), np.zeros((n, k // 32), np.uint16),
                            np.zeros((n, k // 32), np.uint8))
        w = np.zeros((n, k), np.uint16)
        idx = np.arange(n_o, dtype=np.int32) * 10
        if kind == "code":
            can.codes[row, col] = 0xA
        elif kind == "scale":
            can.scales[row, col] = 0x1234
        elif kind == "zero":
            can.zeros[row, col] = 0x9
        else:
            w[row, idx[col]] = 0x4321
        p = ref.pack_layout(can, w, idx)
        if kind == "code":
            nz = np.flatnonzero(p.codes)
            assert nz.tolist() == [off]
            assert p.codes[off] == (0x0A if nib == "low" else 0xA0)
        elif kind == "scale":
            assert np.flatnonzero(p.scales).tolist() == [off] and p.scales[off] == 0x1234
        elif kind == "zero":
            assert np.flatnonzero(p.zeros).tolist() == [off]
            assert p.zeros[off] == 0x9 << (4 * int(nib))
        else:
            assert np.flatnonzero(p.outliers).tolist() == [off] and p.outliers[off] == 0x4321


# ----------------------------------------------------------------- matvec

def _small_problem(ref, n, k, n_t, seed, tau=6.0, m=1):
    spec = wl.MatrixSpec("single", n, k, n_t)
    wb = wl.bits(wl.weight(spec, seed=seed))
    g = wl.gain(spec, seed=seed).numpy()
    layer = ref.pack(wb, g, tau)
    xb = wl.bits(wl.activations(k, m, seed=seed))
    return wb, layer, xb


def test_gemm_brute_force_8x32(ref):
    for seed in range(3):
        wb, layer, xb = _small_problem(ref, 8, 32, 2, seed, tau=1.2)
        y, b = ref.gemm(layer.can, wb, layer.idx, xb)
        codes, sc, ze = layer.can.codes, layer.can.scales, layer.can.zeros
        S = sc.view(np.float16).astype(np.float64)
        wv, xv = _bf16_values(wb), _bf16_values(xb)[0]
        for i in range(8):
            acc = 0.0
            bb = 0.0
            for kk in range(32):
                wd = (float(codes[i, kk]) - float(ze[i, 0])) * float(S[i, 0])
                acc += wd * float(xv[kk])
                bb += abs(wd) * abs(float(xv[kk]))
            for j in layer.idx:
                acc += float(wv[i, j]) * float(xv[j])
                bb += abs(float(wv[i, j])) * abs(float(xv[j]))
            assert y[0, i] == acc and b[0, i] == bb


def test_gemm_all_outliers_is_dense_product(ref):
    wb, layer, xb = _small_problem(ref, 48, 96, 3, 9, tau=-np.inf, m=3)
    assert layer.idx.size == 96
    y, _ = ref.gemm(layer.can, wb, layer.idx, xb)
    dense = _bf16_values(xb) @ _bf16_values(wb).T
    scale = np.abs(_bf16_values(xb)) @ np.abs(_bf16_values(wb)).T
    assert np.all(np.abs(y - dense) <= 1e-13 * scale)


def test_gemm_exact_grid_is_dense_product(ref):
    S = 2.0 ** -7
    vals = np.stack([_grid_row(S, 6, s) for s in range(16)])
    vals = np.concatenate([vals, vals[:, ::-1]], axis=1)  # k = 64
    w = _bf16_bits(vals)
    can = ref.quantize(w, np.array([], dtype=np.int32))
    xb = wl.bits(wl.activations(64, 2, seed=3))
    y, _ = ref.gemm(can, w, np.array([], dtype=np.int32), xb)
    dense = _bf16_values(xb) @ vals.T
    assert np.all(np.abs(y - dense) <= 1e-13 * (np.abs(_bf16_values(xb)) @ np.abs(vals).T))


def test_gemm_unit_vectors_extract_columns(ref):
    wb, layer, _ = _small_problem(ref, 40, 128, 4, 11, tau=6.0)
    what = ref.dequant(layer.can)
    wv = _bf16_values(wb)
    for j in [0, 31, 32, 77, 127] + layer.idx.tolist():
        x = np.zeros((1, 128), dtype=np.uint16)
        x[0, j] = 0x3F80  # 1.0
        y, _ = ref.gemm(layer.can, wb, layer.idx, x)
        expect = what[:, j] + (wv[:, j] if j in layer.idx else 0.0)
        assert np.array_equal(y[0], expect)
        if j in layer.idx:
            assert np.all(what[:, j] == 0.0)


def test_gemm_zero_input_and_linearity(ref):
    wb, layer, _ = _small_problem(ref, 33, 64, 2, 12, tau=3.0)
    y0, b0 = ref.gemm(layer.can, wb, layer.idx, np.zeros((1, 64), np.uint16))
    assert np.all(y0 == 0.0) and np.all(b0 == 0.0)
    rng = np.random.default_rng(0)
    x1 = rng.integers(-8, 8, 64).astype(np.float64)
    x2 = rng.integers(-8, 8, 64).astype(np.float64)
    ya, _ = ref.gemm(layer.can, wb, layer.idx, _bf16_bits(x1[None]))
    yb, _ = ref.gemm(layer.can, wb, layer.idx, _bf16_bits(x2[None]))
    yc, bc = ref.gemm(layer.can, wb, layer.idx, _bf16_bits((x1 + x2)[None]))
    assert np.all(np.abs(ya + yb - yc) <= 1e-13 * (bc + 1.0))


def test_pack_pipeline_counts_bytes(ref):
    # 4.625 bits per bulk weight plus 16 bits per outlier element
    wb, layer, _ = _small_problem(ref, 512, 512, 10, 0, tau=6.0)
    p = layer.packed
    n_o = layer.idx.size
    bulk = p.codes.nbytes + p.scales.nbytes + p.zeros.nbytes
    assert bulk * 8 == 512 * 512 * 4.625
    assert p.outliers.nbytes == 512 * (-(-n_o // 8) * 8) * 2


# ----------------------------------------------------------------- embedding

def test_bf16_golden_cases(ref, golden_dir):
    for line in open(os.path.join(golden_dir, "bf16_rounding_cases.txt")):
        line = line.split("#")[0].strip() if not line.lstrip().startswith("#") else ""
        if not line:
            continue
        expr, hexbits = line.split()[:2]
        v = float(eval(expr, {"__builtins__": {}}))
        assert int(ref.double_to_bf16([v])[0]) == int(hexbits, 16), expr


def test_bf16_midpoints_match_torch(ref):
    # every midpoint between adjacent positive finite BF16 values is exact in
    # float32, so torch's float32 -> bfloat16 (round to nearest even) decides
    # the ties; one double ulp either side must give the lower / upper value
    pos = np.arange(0, 0x7F7F, dtype=np.uint16)
    lo = _bf16_values(pos)
    hi = _bf16_values((pos + 1).astype(np.uint16))
    mid = (lo + hi) / 2.0
    assert np.array_equal(ref.double_to_bf16(mid), _bf16_bits(mid))
    assert np.array_equal(ref.double_to_bf16(np.nextafter(mid, -np.inf)), pos)
    assert np.array_equal(ref.double_to_bf16(np.nextafter(mid, np.inf)), pos + 1)
    neg = ref.double_to_bf16(-mid)
    assert np.array_equal(neg, _bf16_bits(-mid))


def test_bf16_random_floats_match_torch(ref):
    rng = np.random.default_rng(8)
    e = rng.uniform(-140, 127, 40000)
    vals = (np.exp2(e) * rng.choice([-1.0, 1.0], e.size)).astype(np.float32).astype(np.float64)
    assert np.array_equal(ref.double_to_bf16(vals), _bf16_bits(vals))


def _table(ref, n, k, n_t, seed, tau):
    spec = wl.MatrixSpec("lm_head", n, k, n_t)
    wb = wl.bits(wl.weight(spec, seed=seed))
    g = wl.gain(spec, seed=seed).numpy()
    return wb, ref.pack(wb, g, tau)


def test_embed_all_outliers_is_row_indexing(ref):
    # every column kept in BF16: the gather is plain row indexing of W
    wb, layer = _table(ref, 70, 96, 3, 21, -np.inf)
    assert layer.idx.size == 96
    ids = np.array([0, 69, 5, 5, 33, 32, 31])
    out = ref.embed(layer.can, wb, layer.idx, ids)
    expect = _bf16_values(wb)[ids]
    assert np.array_equal(out, expect)
    assert np.array_equal(np.signbit(out), np.signbit(expect))


def test_embed_exact_grid_rows(ref):
    # a table whose groups are exact quantiser grids comes back exactly
    S = 2.0 ** -7
    vals = np.stack([_grid_row(S, 6, s) for s in range(16)])
    vals = np.concatenate([vals, vals[:, ::-1]], axis=1)  # [16, 64]
    w = _bf16_bits(vals)
    can = ref.quantize(w, np.array([], dtype=np.int32))
    ids = np.array([15, 0, 7, 7, 3])
    out = ref.embed(can, w, np.array([], dtype=np.int32), ids)
    assert np.array_equal(out, vals[ids])


def test_embed_rows_agree_with_gemm(ref):
    # row i of the reconstruction dotted with x is y_i of the matvec oracle:
    # a transposed index, a wrong group or a misplaced outlier breaks it
    for tau in (3.0, 6.0):
        wb, layer = _table(ref, 80, 256, 6, 22, tau)
        assert 0 < layer.idx.size < 256
        xb = wl.bits(wl.activations(256, 1, seed=23))
        y, bound = ref.gemm(layer.can, wb, layer.idx, xb)
        ids = np.arange(80)[::-1]
        rows = ref.embed(layer.can, wb, layer.idx, ids)
        dots = rows @ _bf16_values(xb)[0]
        assert np.all(np.abs(dots - y[0, ids]) <= 1e-13 * bound[0, ids])


def test_embed_brute_force_8x32(ref):
    wb, layer = _table(ref, 8, 64, 2, 24, 3.0)
    assert 0 < layer.idx.size < 64
    codes, sc, ze = layer.can.codes, layer.can.scales, layer.can.zeros
    S = sc.view(np.float16).astype(np.float64)
    wv = _bf16_values(wb)
    ids = [3, 0, 7, 3]
    out = ref.embed(layer.can, wb, layer.idx, np.array(ids))
    for r, i in enumerate(ids):
        for j in range(64):
            if j in layer.idx:
                expect = float(wv[i, j])
            else:
                expect = (float(codes[i, j]) - float(ze[i, j // 32])) * float(S[i, j // 32])
            assert out[r, j] == expect


def test_embed_keeps_negative_zero_of_outlier_columns(ref):
    vals = np.zeros((4, 32), dtype=np.float32)
    vals[:, 5] = [-0.0, 1.5, -2.0, 0.0]
    w = _bf16_bits(vals)
    idx = np.array([5], dtype=np.int32)
    can = ref.quantize(w, idx)
    out = ref.embed(can, w, idx, np.array([0, 3]))
    assert np.signbit(out[0, 5]) and not np.signbit(out[1, 5])
    assert np.all(out[:, np.arange(32) != 5] == 0.0)


def test_embed_rejects_ids_outside_table(ref):
    wb, layer = _table(ref, 10, 32, 0, 25, 6.0)
    for bad in ([10], [-1], [0, 3, 10]):
        with pytest.raises(ref.OracleError):
            ref.embed(layer.can, wb, layer.idx, np.array(bad))
    assert ref.embed(layer.can, wb, layer.idx, np.array([], dtype=np.int32)).shape == (0, 32)


# ----------------------------------------------------------------- bulk compaction

def test_bulk_columns_are_the_complement(ref):
    rng = np.random.default_rng(30)
    for k, n_o in [(64, 0), (64, 1), (96, 95), (96, 96), (1536, 23), (1536, 720), (8960, 4193), (32, 7)]:
        idx = np.sort(rng.choice(k, n_o, replace=False)).astype(np.int32)
        kb, bidx = ref.bulk_columns(k, idx)
        rest = np.setdiff1d(np.arange(k), idx)
        assert kb == max(32, -(-rest.size // 32) * 32)
        assert np.array_equal(bidx[: rest.size], rest)
        assert np.all(bidx[rest.size:] == -1)
    for bad in ([3, 3], [5, 2], [-1], [64]):
        with pytest.raises(ref.OracleError):
            ref.bulk_columns(64, np.array(bad, dtype=np.int32))


def test_compaction_without_outliers_is_the_masked_pack(ref):
    wb, layer = _table(ref, 70, 256, 0, 31, np.inf)
    c = ref.pack_compact(wb, wl.gain(wl.MatrixSpec("lm_head", 70, 256, 0), seed=31).numpy(), np.inf)
    assert c.k_bulk == 256 and np.array_equal(c.bulk_idx, np.arange(256))
    for a, b in [(c.can.codes, layer.can.codes), (c.can.scales, layer.can.scales),
                 (c.can.zeros, layer.can.zeros), (c.packed.codes, layer.packed.codes),
                 (c.packed.scales, layer.packed.scales), (c.packed.zeros, layer.packed.zeros)]:
        assert np.array_equal(a, b)


def _compact_problem(ref, n, k, n_t, seed, tau, m=1):
    spec = wl.MatrixSpec("single", n, k, n_t)
    wb = wl.bits(wl.weight(spec, seed=seed))
    g = wl.gain(spec, seed=seed).numpy()
    lay = ref.pack_compact(wb, g, tau)
    xb = wl.bits(wl.activations(k, m, seed=seed))
    return wb, lay, xb


def test_gemm_compact_brute_force_8x64(ref):
    wb, lay, xb = _compact_problem(ref, 8, 64, 2, 24, 3.0)
    assert 0 < lay.idx.size < 64 and lay.k_bulk == 32 * -(-(64 - lay.idx.size) // 32)
    y, b = ref.gemm_compact(lay, wb, xb)
    codes, sc, ze = lay.can.codes, lay.can.scales, lay.can.zeros
    S = sc.view(np.float16).astype(np.float64)
    wv, xv = _bf16_values(wb), _bf16_values(xb)[0]
    bulk = [j for j in range(64) if j not in lay.idx]
    for i in range(8):
        acc = 0.0
        for p, j in enumerate(bulk):
            acc += (float(codes[i, p]) - float(ze[i, p // 32])) * float(S[i, p // 32]) * float(xv[j])
        for j in lay.idx:
            acc += float(wv[i, j]) * float(xv[j])
        assert y[0, i] == acc


def test_gemm_compact_exact_grid_bulk_is_dense_product(ref):
    # heavy outlier columns anywhere, the remaining columns (in order) forming
    # exact quantiser grids: the compacted reconstruction is exact, so y is
    # the dense product -- a bulk column matched with the wrong x breaks it
    S = 2.0 ** -7
    rng = np.random.default_rng(32)
    n, k, n_o = 16, 96, 32
    idx = np.sort(rng.choice(k, n_o, replace=False)).astype(np.int32)
    rest = np.setdiff1d(np.arange(k), idx)
    vals = np.zeros((n, k))
    grid = np.stack([np.concatenate([_grid_row(S, 6, s), _grid_row(S, 9, s + 50)]) for s in range(n)])
    vals[:, rest] = grid
    vals[:, idx] = rng.standard_t(3, (n, n_o)) * 0.5
    w = _bf16_bits(vals)
    kb, bidx = ref.bulk_columns(k, idx)
    can = ref.quantize(ref.gather_bulk(w, bidx), np.zeros(0, np.int32))
    lay = ref.CompactLayer(None, idx, kb, bidx, can, None)
    xb = wl.bits(wl.activations(k, 3, seed=33))
    y, _ = ref.gemm_compact(lay, w, xb)
    wvals = _bf16_values(w)
    dense = _bf16_values(xb) @ wvals.T
    assert np.all(np.abs(y - dense) <= 1e-13 * (np.abs(_bf16_values(xb)) @ np.abs(wvals).T))


def test_gemm_compact_unit_vectors_extract_columns(ref):
    wb, lay, _ = _compact_problem(ref, 40, 128, 4, 34, 3.0)
    what = ref.dequant(lay.can)  # [n, k_bulk]
    wv = _bf16_values(wb)
    pos = {int(j): p for p, j in enumerate(lay.bulk_idx) if j >= 0}
    for j in [0, 31, 32, 77, 127] + lay.idx[:6].tolist():
        x = np.zeros((1, 128), dtype=np.uint16)
        x[0, j] = 0x3F80  # 1.0
        y, _ = ref.gemm_compact(lay, wb, x)
        expect = wv[:, j] if j in lay.idx else what[:, pos[j]]
        assert np.array_equal(y[0], expect)


def test_gemm_compact_all_outliers_is_dense_product(ref):
    wb, lay, xb = _compact_problem(ref, 48, 96, 3, 35, -np.inf, m=2)
    assert lay.idx.size == 96 and lay.k_bulk == 32 and np.all(lay.bulk_idx == -1)
    y, _ = ref.gemm_compact(lay, wb, xb)
    dense = _bf16_values(xb) @ _bf16_values(wb).T
    assert np.all(np.abs(y - dense) <= 1e-13 * (np.abs(_bf16_values(xb)) @ np.abs(_bf16_values(wb)).T))


def test_embed_compact_rows_agree_with_gemm(ref):
    wb, lay, xb = _compact_problem(ref, 64, 256, 6, 36, 3.0)
    y, bound = ref.gemm_compact(lay, wb, xb)
    ids = np.arange(64)[::-1].astype(np.int32)
    rows = ref.embed_compact(lay, wb, ids)
    assert not np.isnan(rows).any()  # the bulk and outlier columns cover every column
    dots = rows @ _bf16_values(xb)[0]
    assert np.all(np.abs(dots - y[0, ids]) <= 1e-13 * bound[0, ids])


def test_compact_outlier_block_is_the_masked_one(ref):
    # compaction changes only the bulk: the BF16 outlier block (pinned by the
    # layout offsets) is the same array
    for tau in (3.0, 6.0):
        spec = wl.MatrixSpec("single", 45, 192, 5)
        wb = wl.bits(wl.weight(spec, seed=37))
        g = wl.gain(spec, seed=37).numpy()
        masked, comp = ref.pack(wb, g, tau), ref.pack_compact(wb, g, tau)
        assert np.array_equal(masked.idx, comp.idx) and comp.idx.size > 0
        assert np.array_equal(masked.packed.outliers, comp.packed.outliers)


# ----------------------------------------------------------------- KV cache

def _kv_tokens(n_tok, H, D, seed):
    return wl.bits(wl.activations(H * D, n_tok, seed=seed)).reshape(n_tok, H, D)


def test_kv_quantize_is_the_weight_quantiser_per_token(ref):
    H, cap, D = 3, 20, 96
    x = _kv_tokens(7, H, D, 40)
    c = ref.kv_cache(H, cap, D)
    ref.kv_quantize(c, x, pos=5)
    for t in range(7):
        for h in range(H):
            row = ref.quantize(x[t, h][None, :], np.zeros(0, np.int32))
            assert np.array_equal(c.codes[h, 5 + t], row.codes[0])
            assert np.array_equal(c.scales[h, 5 + t], row.scales[0])
            assert np.array_equal(c.zeros[h, 5 + t], row.zeros[0])
    assert not c.codes[:, :5].any() and not c.codes[:, 12:].any()
    with pytest.raises(ref.OracleError):
        ref.kv_quantize(c, x, pos=14)  # past the capacity


def _grid_cache(ref, H, T, D, seed, S=2.0 ** -6):
    """A cache whose token vectors are exact quantiser grids: dequantisation
    returns them exactly."""
    rng = np.random.default_rng(seed)
    vals = np.stack([np.concatenate([_grid_row(S, int(rng.integers(0, 16)), int(rng.integers(1e6)))
                                     for _ in range(D // 32)]) for _ in range(T * H)]).reshape(T, H, D)
    c = ref.kv_cache(H, T, D)
    ref.kv_quantize(c, _bf16_bits(vals), 0)
    return c, vals


def _textbook_attention(q, K, V, scale, Hq, Hkv):
    from scipy.special import softmax
    grp = Hq // Hkv
    out = np.empty((Hq, K.shape[2]))
    for i in range(Hq):
        h = i // grp
        p = softmax(scale * (K[:, h, :] @ q[i]))
        out[i] = p @ V[:, h, :]
    return out


def test_attention_exact_grid_is_textbook(ref):
    Hq, Hkv, T, D = 6, 2, 50, 64
    kc, K = _grid_cache(ref, Hkv, T, D, 41)
    vc, V = _grid_cache(ref, Hkv, T, D, 42)
    qb = wl.bits(wl.activations(D, Hq, seed=43))
    out, vb, sm = ref.attention(kc, vc, qb, T, 1.0 / np.sqrt(D))
    want = _textbook_attention(_bf16_values(qb), K, V, 1.0 / np.sqrt(D), Hq, Hkv)
    assert np.allclose(out, want, rtol=1e-12, atol=1e-14)
    assert np.all(vb >= np.abs(out) - 1e-15) and np.all(sm > 0)


def test_attention_one_token_and_zero_query(ref):
    Hkv, D = 2, 64
    kc, K = _grid_cache(ref, Hkv, 9, D, 44)
    vc, V = _grid_cache(ref, Hkv, 9, D, 45)
    qb = wl.bits(wl.activations(D, 4, seed=46))
    out, _, _ = ref.attention(kc, vc, qb, 1, 0.125)
    assert np.array_equal(out[:2], np.stack([V[0, 0]] * 2)) and np.array_equal(out[2:], np.stack([V[0, 1]] * 2))
    out, _, _ = ref.attention(kc, vc, np.zeros((4, D), np.uint16), 9, 0.125)
    assert np.allclose(out[0], V[:, 0].mean(0), rtol=0, atol=1e-15)
    assert np.allclose(out[3], V[:, 1].mean(0), rtol=0, atol=1e-15)


def test_kv_pack_golden_offsets(ref, golden_dir):
    H, cap, D = 2, 3, 64
    c = ref.kv_cache(H, cap, D)
    rng = np.random.default_rng(47)
    c.codes[:] = rng.integers(0, 16, c.codes.shape)
    c.scales[:] = rng.integers(0, 1 << 15, c.scales.shape)
    c.zeros[:] = rng.integers(0, 16, c.zeros.shape)
    pc, ps, pz = ref.kv_pack(c)
    n = 0
    for line in open(os.path.join(golden_dir, "kv_layout_offsets.txt")):
        if line.startswith("#") or not line.strip():
            continue
        h, t, ch, byte, hi, se, zw, zs = (int(v) for v in line.split()[:8])
        got = (pc[byte] >> 4) if hi else (pc[byte] & 0xF)
        assert got == c.codes[h, t, ch]
        assert ps[se] == c.scales[h, t, ch // 32]
        assert ((pz[zw] >> zs) & 0xF) == c.zeros[h, t, ch // 32]
        n += 1
    assert n == 4


def test_attention_tolerance_covers_its_budget(ref):
    # perturb every score by up to 2e-3 S_t and every weighted-sum term by up
    # to 2e-3 of its size, in the worst direction; the output stays inside
    # the stated tolerance
    Hq, Hkv, T, D = 2, 1, 40, 64
    kc, K = _grid_cache(ref, Hkv, T, D, 48)
    vc, V = _grid_cache(ref, Hkv, T, D, 49)
    qb = wl.bits(wl.activations(D, Hq, seed=50))
    scale = 1.0 / np.sqrt(D)
    out, vb, sm = ref.attention(kc, vc, qb, T, scale)
    tol = ref.attention_tolerance(vb, sm)
    q = _bf16_values(qb)
    for i in range(Hq):
        s = scale * (K[:, 0, :] @ q[i])
        S = scale * (np.abs(K[:, 0, :]) @ np.abs(q[i]))
        for d in range(D):
            for sign in (1, -1):
                bump = sign * np.sign(V[:, 0, d] - out[i, d])  # raise the weights that move o_d away
                s2 = s + 2e-3 * S * bump
                p = np.exp(s2 - s2.max()); p /= p.sum()
                o2 = p @ V[:, 0, d] + sign * 2e-3 * (p @ np.abs(V[:, 0, d]))
                assert abs(o2 - out[i, d]) <= tol[i, d]


# ----------------------------------------------------------------- row table

def test_row_table_golden_offsets(ref, golden_dir):
    """Each hand-derived offset of the row table holds the one planted value."""
    lines = [l.split("#")[0].split() for l in open(os.path.join(golden_dir, "row_table_offsets.txt"))]
    lines = [l for l in lines if l]
    assert len(lines) == 14
    for n, k, n_o, kind, row, col, off, nib in lines:
        n, k, n_o, row, col, off = int(n), int(k), int(n_o), int(row), int(col), int(off)
        G = k // 32
        can = ref.Canonical(np.zeros((n, k), np.uint8), np.zeros((n, G), np.uint16), np.zeros((n, G), np.uint8))
        w = np.zeros((n, k + 7), np.uint16)  # a wider BF16 matrix: the outlier values come by its stride
        idx = np.arange(n_o, dtype=np.int32) * 3 + 1
        if kind == "code":
            can.codes[row, col] = 0xA
        elif kind == "scale":
            can.scales[row, col] = 0x1234
        elif kind == "zero":
            can.zeros[row, col] = 0x9
        else:
            w[row, idx[col]] = 0x4321
        t = ref.row_table(can, w, idx)
        if kind == "code":
            assert np.flatnonzero(t.codes).tolist() == [off]
            assert t.codes[off] == (0x0A if nib == "low" else 0xA0)
        elif kind == "scale":
            assert np.flatnonzero(t.scales).tolist() == [off] and t.scales[off] == 0x1234
        elif kind == "zero":
            assert np.flatnonzero(t.zeros).tolist() == [off]
            assert t.zeros[off] == 0x9 << (4 * int(nib))
        else:
            assert np.flatnonzero(t.outliers).tolist() == [off] and t.outliers[off] == 0x4321


def test_row_table_rows_are_the_packed_rows(ref):
    """A row of the row table holds the same code records, scales, zero words
    and outlier values as that row's lane of the RT32 layout (a permutation,
    nothing rounded)."""
    rng = np.random.default_rng(8)
    n, k, n_o = 70, 320, 13
    # BF16 bits of N(0, 0.02) values (the high half of their FP32 bits)
    w = (rng.standard_normal((n, k)).astype(np.float32) * 0.02).view(np.uint32) >> 16
    w = w.astype(np.uint16)
    idx = np.sort(rng.choice(k, n_o, replace=False)).astype(np.int32)
    can = ref.quantize(w, idx)
    p = ref.pack_layout(can, w, idx)
    t = ref.row_table(can, w, idx)
    G, S, O8 = k // 32, -(-(k // 32) // 8), -(-n_o // 8)
    for i in range(n):
        tt, r = divmod(i, 32)
        for g in range(G):
            a = ((tt * G + g) * 32 + r) * 16
            assert np.array_equal(t.codes[(i * G + g) * 16:(i * G + g + 1) * 16], p.codes[a:a + 16])
            assert t.scales[i * G + g] == p.scales[((tt * S + g // 8) * 32 + r) * 8 + g % 8]
        for s_ in range(S):
            assert t.zeros[i * S + s_] == p.zeros[(tt * S + s_) * 32 + r]
        for o in range(n_o):
            assert t.outliers[i * n_o + o] == p.outliers[((tt * O8 + o // 8) * 32 + r) * 8 + o % 8]
