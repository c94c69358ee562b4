"""Shared helpers of the GPU parity tests: draw one workload, run it through
the CUDA library and through the CPU oracle, and compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import outlier_split_bit_b200 as sp
from outlier_split_bit_b200 import workload as wl

DEV = "cuda"


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy().view(np.uint16).ravel()


def u32(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy().view(np.uint32).ravel()


def u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy().view(np.uint8).ravel()


def draw(spec, seed=0, layer=0, m=1, with_gain=True):
    w = wl.weight(spec, seed, layer, device=DEV)
    g = wl.gain(spec, seed, layer, device=DEV) if with_gain else None
    x = wl.activations(spec.k, m, seed, layer, device=DEV)
    return w, g, x


def np_gain(g):
    return None if g is None else g.detach().cpu().numpy().astype(np.float32)


def tile_slices(layer: sp.PackedLayer, tiles):
    """Per-array slices of the packed buffers that belong to the given tiles."""
    G, S, O8 = layer.k // 32, -(-(layer.k // 32) // 8), -(-layer.n_outliers // 8)
    codes, scales, zeros, outw = u8(layer.codes), u16(layer.scales), u32(layer.zeros), u16(layer.outlier_w)
    out = {"codes": [], "scales": [], "zeros": [], "outliers": []}
    for t in tiles:
        out["codes"].append(codes[t * G * 512:(t + 1) * G * 512])
        out["scales"].append(scales[t * S * 256:(t + 1) * S * 256])
        out["zeros"].append(zeros[t * S * 32:(t + 1) * S * 32])
        if O8:
            out["outliers"].append(outw[t * O8 * 256:(t + 1) * O8 * 256])
    return {k: (np.concatenate(v) if v else np.zeros(0)) for k, v in out.items()}


def oracle_rows(wb: np.ndarray, idx: np.ndarray, tiles):
    """Oracle canonical + packed arrays of whole 32-row tiles of W."""
    n = wb.shape[0]
    rows = np.concatenate([np.arange(32 * t, min(n, 32 * t + 32)) for t in tiles])
    sub = np.ascontiguousarray(wb[rows])
    can = oracle.quantize(sub, idx)
    # pack tile by tile so that a short last tile is padded like on the GPU
    parts = {"codes": [], "scales": [], "zeros": [], "outliers": []}
    off = 0
    for t in tiles:
        nr = min(n, 32 * t + 32) - 32 * t
        c = oracle.Canonical(can.codes[off:off + nr], can.scales[off:off + nr], can.zeros[off:off + nr])
        p = oracle.pack_layout(c, sub[off:off + nr], idx)
        parts["codes"].append(p.codes)
        parts["scales"].append(p.scales)
        parts["zeros"].append(p.zeros)
        parts["outliers"].append(p.outliers)
        off += nr
    return rows, can, {k: np.concatenate(v) for k, v in parts.items()}


def check_gemv(y_gpu: torch.Tensor, y_ref: np.ndarray, bound: np.ndarray, bf16: bool = False):
    """Tolerance of the matvec: |y - y_ref| <= 2e-3 * sum|w_hat x| + 1e-5; a BF16
    output adds its own rounding (half an ulp, 2^-9 relative)."""
    y = y_gpu.detach().float().cpu().numpy().astype(np.float64).reshape(y_ref.shape)
    tol = oracle.tolerance(bound)
    if bf16:
        tol = tol + np.abs(y_ref) * 2.0 ** -8
    err = np.abs(y - y_ref)
    bad = err > tol
    assert not bad.any(), (f"{bad.sum()} outputs out of tolerance; worst ratio "
                           f"{float((err / tol).max()):.3g}")
    return float((err / tol).max())


_KAPPA_CACHE = {}


def oracle_split(wb: np.ndarray, gain, tau: float, key=None):
    """The oracle's kurtosis and outlier indices of a large matrix.  Kurtosis
    is computed per column, so the oracle is called on contiguous blocks of 64
    columns (the same values, read with unit stride instead of one cache miss
    per element).  `key` caches the kurtosis of a matrix drawn more than once
    (it does not depend on tau)."""
    if key is not None and key in _KAPPA_CACHE:
        kap = _KAPPA_CACHE[key]
    else:
        k = wb.shape[1]
        kap = np.empty(k, dtype=np.float64)
        for j0 in range(0, k, 64):
            j1 = min(k, j0 + 64)
            kap[j0:j1] = oracle.kurtosis(np.ascontiguousarray(wb[:, j0:j1]),
                                         None if gain is None else gain[j0:j1])
        if key is not None:
            _KAPPA_CACHE[key] = kap
    return kap, oracle.split(kap, tau)
