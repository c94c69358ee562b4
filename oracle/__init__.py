"""CPU oracle for the SPECTRA outlier-split INT4 decode matvec.

TEST INFRASTRUCTURE ONLY: the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package; the library under
``outlier_split_bit_b200`` never does, and this package never imports it.

The arithmetic lives in ``spectra_ref.c`` (plain C99, IEEE double,
``-O2 -ffp-contract=off``); this module compiles it with gcc and wraps it with
ctypes on NumPy arrays.  Method source: "SPECTRA: Sparse-Precision Exact
Channel Tensor Reconstruction Architecture" (aiwithghost.com re-post of the
Dev.to abstract), abstract paragraph (kurtosis split with threshold 3.0,
Group-32 4-bit codes with scale and bit-packed zero point, exact floating-point
outlier channels).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "spectra_ref.c")
_LIB = os.path.join(_HERE, "libspectra_ref.so")

# Oracle status codes (its own numbering, see spectra_ref.c).
OK, ERR_INVALID_ARG, ERR_SHAPE, ERR_NONFINITE, ERR_RANGE = 0, 1, 2, 3, 4
STATUS_NAMES = {OK: "ok", ERR_INVALID_ARG: "invalid_arg", ERR_SHAPE: "shape",
                ERR_NONFINITE: "nonfinite", ERR_RANGE: "range"}


class OracleError(RuntimeError):
    def __init__(self, status: int):
        super().__init__(f"oracle status {STATUS_NAMES.get(status, status)}")
        self.status = status


def build(force: bool = False) -> str:
    """Compile the oracle into a shared library next to its source."""
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC)):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    subprocess.check_call(["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math",
                           "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
    os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


def _declare(L):
    P = ctypes.c_void_p
    i32, i64, f64, u16 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double, ctypes.c_uint16
    L.spectra_ref_bf16_to_double.argtypes = [u16]
    L.spectra_ref_bf16_to_double.restype = f64
    L.spectra_ref_fp16_to_double.argtypes = [u16]
    L.spectra_ref_fp16_to_double.restype = f64
    L.spectra_ref_double_to_fp16.argtypes = [f64]
    L.spectra_ref_double_to_fp16.restype = u16
    L.spectra_ref_kurtosis.argtypes = [P, P, i32, i32, P]
    L.spectra_ref_kurtosis.restype = ctypes.c_int
    L.spectra_ref_split.argtypes = [P, i32, f64, P]
    L.spectra_ref_split.restype = i32
    L.spectra_ref_quantize.argtypes = [P, i32, i32, P, i32, P, P, P]
    L.spectra_ref_quantize.restype = ctypes.c_int
    L.spectra_ref_layout_sizes.argtypes = [i32, i32, i32, P]
    L.spectra_ref_layout_sizes.restype = None
    L.spectra_ref_pack_layout.argtypes = [i32, i32, P, P, P, P, P, i32, P, P, P, P]
    L.spectra_ref_pack_layout.restype = None
    L.spectra_ref_unpack_layout.argtypes = [i32, i32, P, P, P, P, P, P]
    L.spectra_ref_unpack_layout.restype = None
    L.spectra_ref_dequant.argtypes = [i32, i32, P, P, P, P]
    L.spectra_ref_dequant.restype = None
    L.spectra_ref_gemm.argtypes = [i32, i32, P, P, P, P, P, i32, P, i32, P, P]
    L.spectra_ref_gemm.restype = None
    L.spectra_ref_double_to_bf16.argtypes = [f64]
    L.spectra_ref_double_to_bf16.restype = u16
    L.spectra_ref_embed.argtypes = [i32, i32, P, P, P, P, P, i32, P, i32, P]
    L.spectra_ref_embed.restype = ctypes.c_int
    L.spectra_ref_bulk_columns.argtypes = [i32, P, i32, P]
    L.spectra_ref_bulk_columns.restype = i32
    L.spectra_ref_gather_bulk.argtypes = [P, i32, i32, P, i32, P]
    L.spectra_ref_gather_bulk.restype = None
    L.spectra_ref_pack_outliers.argtypes = [i32, i32, P, P, i32, P]
    L.spectra_ref_pack_outliers.restype = None
    L.spectra_ref_row_table.argtypes = [i32, i32, P, P, P, P, i32, P, i32, P, P, P, P]
    L.spectra_ref_row_table.restype = None
    L.spectra_ref_gemm_compact.argtypes = [i32, i32, i32, P, P, P, P, P, P, i32, P, i32, P, P]
    L.spectra_ref_gemm_compact.restype = None
    L.spectra_ref_embed_compact.argtypes = [i32, i32, i32, P, P, P, P, P, P, i32, P, i32, P]
    L.spectra_ref_embed_compact.restype = ctypes.c_int
    L.spectra_ref_kv_quantize.argtypes = [P, i32, i32, i32, i32, i32, P, P, P]
    L.spectra_ref_kv_quantize.restype = ctypes.c_int
    L.spectra_ref_attention.argtypes = [i32, i32, i32, i32, i32, P, P, P, P, P, P, P, f64, P, P, P]
    L.spectra_ref_attention.restype = ctypes.c_int
    L.spectra_ref_kv_pack.argtypes = [i32, i32, i32, P, P, P, P, P, P]
    L.spectra_ref_kv_pack.restype = None


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ------------------------------------------------------------------ numbers

def bf16_to_double(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).ravel()
    f = lib().spectra_ref_bf16_to_double
    return np.array([f(int(v)) for v in b], dtype=np.float64).reshape(np.shape(bits))


def fp16_to_double(bits) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).ravel()
    f = lib().spectra_ref_fp16_to_double
    return np.array([f(int(v)) for v in b], dtype=np.float64).reshape(np.shape(bits))


def double_to_fp16(values) -> np.ndarray:
    v = np.asarray(values, dtype=np.float64).ravel()
    f = lib().spectra_ref_double_to_fp16
    return np.array([f(float(a)) for a in v], dtype=np.uint16).reshape(np.shape(values))


# ------------------------------------------------------------------ pipeline

def kurtosis(w_bits: np.ndarray, gain: np.ndarray | None) -> np.ndarray:
    """Per-column Pearson kurtosis of W*g (FP64). w_bits: uint16 [n, k]."""
    w = _c(w_bits, np.uint16)
    n, k = w.shape
    g = None if gain is None else _c(gain, np.float32)
    kap = np.empty(k, dtype=np.float64)
    st = lib().spectra_ref_kurtosis(_p(w), _p(g), n, k, _p(kap))
    if st != OK:
        raise OracleError(st)
    return kap


def split(kappa: np.ndarray, tau: float) -> np.ndarray:
    """Ascending int32 indices of the columns with kappa > tau."""
    kap = _c(kappa, np.float64)
    idx = np.empty(max(1, kap.size), dtype=np.int32)
    n_o = lib().spectra_ref_split(_p(kap), kap.size, float(tau), _p(idx))
    return idx[:n_o].copy()


@dataclass
class Canonical:
    """Row-major canonical quantised bulk: one code / zero per byte."""
    codes: np.ndarray   # uint8 [n, k]
    scales: np.ndarray  # uint16 (FP16 bits) [n, k/32]
    zeros: np.ndarray   # uint8 [n, k/32]


def quantize(w_bits: np.ndarray, idx: np.ndarray) -> Canonical:
    w = _c(w_bits, np.uint16)
    n, k = w.shape
    ix = _c(idx, np.int32)
    G = k // 32 if k % 32 == 0 else 1
    codes = np.zeros((n, k), dtype=np.uint8)
    scales = np.zeros((n, G), dtype=np.uint16)
    zeros = np.zeros((n, G), dtype=np.uint8)
    st = lib().spectra_ref_quantize(_p(w), n, k, _p(ix) if ix.size else None, ix.size,
                                    _p(codes), _p(scales), _p(zeros))
    if st != OK:
        raise OracleError(st)
    return Canonical(codes, scales, zeros)


def layout_sizes(n: int, k: int, n_o: int) -> dict:
    out = np.zeros(5, dtype=np.int64)
    lib().spectra_ref_layout_sizes(n, k, n_o, _p(out))
    return {"codes": int(out[0]), "scales": int(out[1]), "zeros": int(out[2]),
            "outliers": int(out[3]), "n_pad": int(out[4])}


@dataclass
class Packed:
    codes: np.ndarray     # uint8 [code bytes]
    scales: np.ndarray    # uint16 FP16 bits
    zeros: np.ndarray     # uint32 words
    outliers: np.ndarray  # uint16 BF16 bits
    idx: np.ndarray       # int32 [n_o]
    n: int
    k: int


def pack_layout(can: Canonical, w_bits: np.ndarray, idx: np.ndarray) -> Packed:
    w = _c(w_bits, np.uint16)
    n, k = w.shape
    ix = _c(idx, np.int32)
    sz = layout_sizes(n, k, ix.size)
    pc = np.zeros(sz["codes"], dtype=np.uint8)
    ps = np.zeros(sz["scales"], dtype=np.uint16)
    pz = np.zeros(sz["zeros"], dtype=np.uint32)
    po = np.zeros(max(1, sz["outliers"]), dtype=np.uint16)
    lib().spectra_ref_pack_layout(n, k, _p(_c(can.codes, np.uint8)), _p(_c(can.scales, np.uint16)),
                                  _p(_c(can.zeros, np.uint8)), _p(w),
                                  _p(ix) if ix.size else None, ix.size,
                                  _p(pc), _p(ps), _p(pz), _p(po))
    return Packed(pc, ps, pz, po[:sz["outliers"]], ix.copy(), n, k)


def unpack_layout(p: Packed) -> Canonical:
    n, k = p.n, p.k
    G = k // 32
    codes = np.zeros((n, k), dtype=np.uint8)
    scales = np.zeros((n, G), dtype=np.uint16)
    zeros = np.zeros((n, G), dtype=np.uint8)
    lib().spectra_ref_unpack_layout(n, k, _p(_c(p.codes, np.uint8)), _p(_c(p.scales, np.uint16)),
                                    _p(_c(p.zeros, np.uint32)), _p(codes), _p(scales), _p(zeros))
    return Canonical(codes, scales, zeros)


def dequant(can: Canonical) -> np.ndarray:
    n, k = can.codes.shape
    out = np.empty((n, k), dtype=np.float64)
    lib().spectra_ref_dequant(n, k, _p(_c(can.codes, np.uint8)), _p(_c(can.scales, np.uint16)),
                              _p(_c(can.zeros, np.uint8)), _p(out))
    return out


def gemm(can: Canonical, w_bits: np.ndarray, idx: np.ndarray, x_bits: np.ndarray):
    """(y [m, n], bound [m, n]) in FP64; x_bits: uint16 BF16 [m, k] (or [k])."""
    w = _c(w_bits, np.uint16)
    n, k = w.shape
    x = _c(x_bits, np.uint16).reshape(-1, k)
    m = x.shape[0]
    ix = _c(idx, np.int32)
    y = np.empty((m, n), dtype=np.float64)
    b = np.empty((m, n), dtype=np.float64)
    lib().spectra_ref_gemm(n, k, _p(_c(can.codes, np.uint8)), _p(_c(can.scales, np.uint16)),
                           _p(_c(can.zeros, np.uint8)), _p(w), _p(ix) if ix.size else None,
                           ix.size, _p(x), m, _p(y), _p(b))
    return y, b


@dataclass
class Layer:
    """Everything the oracle derives from one weight matrix."""
    kappa: np.ndarray
    idx: np.ndarray
    can: Canonical
    packed: Packed


def pack(w_bits: np.ndarray, gain: np.ndarray | None, tau: float) -> Layer:
    """Saliency split, group quantiser and packed layout, in that order."""
    kap = kurtosis(w_bits, gain)
    idx = split(kap, tau)
    can = quantize(w_bits, idx)
    return Layer(kap, idx, can, pack_layout(can, w_bits, idx))


def double_to_bf16(values) -> np.ndarray:
    v = np.asarray(values, dtype=np.float64).ravel()
    f = lib().spectra_ref_double_to_bf16
    return np.array([f(float(a)) for a in v], dtype=np.uint16).reshape(np.shape(values))


def embed(can: Canonical, w_bits: np.ndarray, idx: np.ndarray, ids) -> np.ndarray:
    """Rows ids of the reconstructed table (FP64 [m, k]); w_bits: uint16 [n, k]."""
    w = _c(w_bits, np.uint16)
    n, k = w.shape
    ix = _c(idx, np.int32)
    tok = _c(np.asarray(ids).ravel(), np.int32)
    out = np.zeros((tok.size, k), dtype=np.float64)
    st = lib().spectra_ref_embed(n, k, _p(_c(can.codes, np.uint8)), _p(_c(can.scales, np.uint16)),
                                 _p(_c(can.zeros, np.uint8)), _p(w), _p(ix) if ix.size else None,
                                 ix.size, _p(tok) if tok.size else None, tok.size,
                                 _p(out) if tok.size else None)
    if st != OK:
        raise OracleError(st)
    return out


# ------------------------------------------------------------------ row table

@dataclass
class RowTable:
    """A table that is only gathered, every row's pieces contiguous."""
    codes: np.ndarray     # uint8 [n * G * 16]
    scales: np.ndarray    # uint16 [n * G]
    zeros: np.ndarray     # uint32 [n * S]
    outliers: np.ndarray  # uint16 [n * n_o]


def row_table(can: Canonical, w_bits: np.ndarray, idx: np.ndarray) -> RowTable:
    """Row-table layout of canonical arrays over k bulk columns (can.codes is
    [n, k]); w_bits is the BF16 matrix [n, kw] the outlier values come from."""
    codes = _c(can.codes, np.uint8)
    n, k = codes.shape
    w = _c(w_bits, np.uint16)
    ix = _c(idx, np.int32)
    G, S = k // 32, -(-(k // 32) // 8)
    out = RowTable(np.zeros(n * G * 16, np.uint8), np.zeros(n * G, np.uint16),
                   np.zeros(n * S, np.uint32), np.zeros(max(1, n * ix.size), np.uint16))
    lib().spectra_ref_row_table(n, k, _p(codes), _p(_c(can.scales, np.uint16)), _p(_c(can.zeros, np.uint8)),
                                _p(w), w.shape[1], _p(ix) if ix.size else None, ix.size, _p(out.codes),
                                _p(out.scales), _p(out.zeros), _p(out.outliers))
    out.outliers = out.outliers[: n * ix.size]
    return out


# ------------------------------------------------------------------ bulk compaction

def bulk_columns(k: int, idx: np.ndarray):
    """(k_bulk, bulk_idx int32 [k_bulk]) of the compacted bulk."""
    ix = _c(idx, np.int32)
    out = np.full(max(32, k + 31), -7, dtype=np.int32)
    kb = lib().spectra_ref_bulk_columns(k, _p(ix) if ix.size else None, ix.size, _p(out))
    if kb < 0:
        raise OracleError(ERR_INVALID_ARG)
    return kb, out[:kb].copy()


def gather_bulk(w_bits: np.ndarray, bulk_idx: np.ndarray) -> np.ndarray:
    w = _c(w_bits, np.uint16)
    n, k = w.shape
    bi = _c(bulk_idx, np.int32)
    out = np.empty((n, bi.size), dtype=np.uint16)
    lib().spectra_ref_gather_bulk(_p(w), n, k, _p(bi), bi.size, _p(out))
    return out


def pack_outliers(w_bits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    w = _c(w_bits, np.uint16)
    n, k = w.shape
    ix = _c(idx, np.int32)
    sz = layout_sizes(n, 32, ix.size)["outliers"]
    out = np.zeros(max(1, sz), dtype=np.uint16)
    lib().spectra_ref_pack_outliers(n, k, _p(w), _p(ix) if ix.size else None, ix.size, _p(out))
    return out[:sz]


@dataclass
class CompactLayer:
    """Everything the oracle derives from one matrix with a compacted bulk."""
    kappa: np.ndarray
    idx: np.ndarray
    k_bulk: int
    bulk_idx: np.ndarray  # int32 [k_bulk], -1 = padding
    can: Canonical        # bulk [n, k_bulk]
    packed: Packed        # bulk layout over k_bulk columns + outlier block


def pack_compact(w_bits: np.ndarray, gain: np.ndarray | None, tau: float) -> CompactLayer:
    """Saliency split, compaction of the bulk, group quantiser of the compacted
    bulk, packed layout: in that order."""
    w = _c(w_bits, np.uint16)
    kap = kurtosis(w, gain)
    idx = split(kap, tau)
    k_bulk, bidx = bulk_columns(w.shape[1], idx)
    wb = gather_bulk(w, bidx)
    can = quantize(wb, np.zeros(0, np.int32))
    bulk = pack_layout(can, wb, np.zeros(0, np.int32))
    packed = Packed(bulk.codes, bulk.scales, bulk.zeros, pack_outliers(w, idx), idx.copy(),
                    w.shape[0], w.shape[1])
    return CompactLayer(kap, idx, k_bulk, bidx, can, packed)


def gemm_compact(lay: CompactLayer, w_bits: np.ndarray, x_bits: np.ndarray):
    """(y [m, n], bound [m, n]) of a compacted layer in FP64."""
    w = _c(w_bits, np.uint16)
    n, k = w.shape
    x = _c(x_bits, np.uint16).reshape(-1, k)
    m = x.shape[0]
    ix = _c(lay.idx, np.int32)
    y = np.empty((m, n), dtype=np.float64)
    b = np.empty((m, n), dtype=np.float64)
    lib().spectra_ref_gemm_compact(n, k, lay.k_bulk, _p(_c(lay.can.codes, np.uint8)),
                                   _p(_c(lay.can.scales, np.uint16)), _p(_c(lay.can.zeros, np.uint8)),
                                   _p(_c(lay.bulk_idx, np.int32)), _p(w),
                                   _p(ix) if ix.size else None, ix.size, _p(x), m, _p(y), _p(b))
    return y, b


def embed_compact(lay: CompactLayer, w_bits: np.ndarray, ids) -> np.ndarray:
    """Rows ids of the reconstructed compacted table (FP64 [m, k])."""
    w = _c(w_bits, np.uint16)
    n, k = w.shape
    ix = _c(lay.idx, np.int32)
    tok = _c(np.asarray(ids).ravel(), np.int32)
    out = np.full((tok.size, k), np.nan, dtype=np.float64)
    st = lib().spectra_ref_embed_compact(n, k, lay.k_bulk, _p(_c(lay.can.codes, np.uint8)),
                                         _p(_c(lay.can.scales, np.uint16)),
                                         _p(_c(lay.can.zeros, np.uint8)),
                                         _p(_c(lay.bulk_idx, np.int32)), _p(w),
                                         _p(ix) if ix.size else None, ix.size,
                                         _p(tok) if tok.size else None, tok.size,
                                         _p(out) if tok.size else None)
    if st != OK:
        raise OracleError(st)
    return out


# ------------------------------------------------------------------ KV cache

@dataclass
class KVCache:
    """Canonical 4-bit cache of one of K or V: [H][cap][D] codes, [H][cap][D/32]
    scales (FP16 bits) and zero points."""
    codes: np.ndarray
    scales: np.ndarray
    zeros: np.ndarray

    @property
    def shape(self):
        return self.codes.shape  # (H, cap, D)


def kv_cache(H: int, cap: int, D: int) -> KVCache:
    return KVCache(np.zeros((H, cap, D), np.uint8), np.zeros((H, cap, D // 32), np.uint16),
                   np.zeros((H, cap, D // 32), np.uint8))


def kv_quantize(cache: KVCache, x_bits: np.ndarray, pos: int) -> None:
    """Quantise tokens x [n_tok, H, D] (BF16 bits) into positions pos.. of cache."""
    H, cap, D = cache.shape
    x = _c(x_bits, np.uint16).reshape(-1, H, D)
    st = lib().spectra_ref_kv_quantize(_p(x), x.shape[0], H, D, pos, cap, _p(cache.codes),
                                       _p(cache.scales), _p(cache.zeros))
    if st != OK:
        raise OracleError(st)


def kv_pack(cache: KVCache):
    """(codes bytes, scales u16, zeros u32) in the packed KV layout."""
    H, cap, D = cache.shape
    pc = np.zeros(H * cap * D // 2, np.uint8)
    ps = np.zeros(H * cap * (D // 32), np.uint16)
    pz = np.zeros(H * cap, np.uint32)
    lib().spectra_ref_kv_pack(H, cap, D, _p(cache.codes), _p(cache.scales), _p(cache.zeros),
                              _p(pc), _p(ps), _p(pz))
    return pc, ps, pz


def attention(kc: KVCache, vc: KVCache, q_bits: np.ndarray, T: int, scale: float):
    """(out [Hq, D], vbound [Hq, D], smax [Hq]) of decode attention in FP64."""
    H, cap, D = kc.shape
    q = _c(q_bits, np.uint16).reshape(-1, D)
    Hq = q.shape[0]
    out = np.empty((Hq, D)); vb = np.empty((Hq, D)); sm = np.empty(Hq)
    st = lib().spectra_ref_attention(Hq, H, D, T, cap, _p(kc.codes), _p(kc.scales), _p(kc.zeros),
                                     _p(vc.codes), _p(vc.scales), _p(vc.zeros), _p(q), float(scale),
                                     _p(out), _p(vb), _p(sm))
    if st != OK:
        raise OracleError(st)
    return out, vb, sm


def attention_tolerance(vbound: np.ndarray, smax: np.ndarray) -> np.ndarray:
    """Acceptance bound of a GPU decode-attention output.  Each score is a dot
    product held to the matvec's budget, |ds_t| <= 2e-3 * S_t with
    S_t = scale * sum_d |q_d k_hat_td| (so |ds_t| <= D_s = 2e-3 * max_t S_t);
    score errors of at most D_s move every softmax weight by a factor within
    [exp(-2 D_s), exp(2 D_s)], so the output moves by at most
    (exp(2 D_s) - 1) * sum_t p_t |v_hat_td|; the weighted sum over V has its
    own 2e-3 * sum_t p_t |v_hat_td|.  Plus 1e-5 absolute."""
    ds = 2e-3 * smax[:, None]
    return (2e-3 + np.expm1(2.0 * ds)) * vbound + 1e-5


def tolerance(bound: np.ndarray) -> np.ndarray:
    """Acceptance bound of a GPU matvec result: 2e-3 * sum|w_hat||x| + 1e-5."""
    return 2e-3 * bound + 1e-5
