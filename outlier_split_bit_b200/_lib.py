"""ctypes declarations of the C ABI in include/spectra.h (no logic here)."""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libspectra.so")

# spectra_status values
OK = 0
ERR_INVALID_ARG = 1
ERR_SHAPE = 2
ERR_ALIGN = 3
ERR_NONFINITE = 4
ERR_RANGE = 5
ERR_BUFFER_TOO_SMALL = 6
ERR_CUDA = 7
ERR_UNSUPPORTED = 8
ERR_INTERNAL = 9
ERR_IO = 10
ERR_FORMAT = 11

MEM_DEVICE = 0
MEM_HOST = 1

F32 = 0
BF16 = 1


class Layer(ctypes.Structure):
    """spectra_layer: a view of caller-owned device buffers."""
    _fields_ = [("n", ctypes.c_int32), ("k", ctypes.c_int32), ("n_outliers", ctypes.c_int32),
                ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("zeros", ctypes.c_void_p),
                ("outlier_idx", ctypes.c_void_p), ("outlier_w", ctypes.c_void_p),
                ("k_bulk", ctypes.c_int32), ("bulk_idx", ctypes.c_void_p)]


class Sizes(ctypes.Structure):
    _fields_ = [("n_pad", ctypes.c_int64), ("codes_bytes", ctypes.c_size_t),
                ("scales_bytes", ctypes.c_size_t), ("zeros_bytes", ctypes.c_size_t),
                ("outlier_idx_bytes", ctypes.c_size_t), ("outlier_w_bytes", ctypes.c_size_t),
                ("k_bulk", ctypes.c_int32), ("bulk_idx_bytes", ctypes.c_size_t)]


class KV(ctypes.Structure):
    """spectra_kv: a view of one packed 4-bit KV cache (device buffers)."""
    _fields_ = [("n_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("capacity", ctypes.c_int32), ("codes", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("zeros", ctypes.c_void_p)]


class TrdcLayer(ctypes.Structure):
    """spectra_trdc_layer: one layer record of a TRDC container."""
    _fields_ = [("name", ctypes.c_char * 96), ("n", ctypes.c_int32), ("k", ctypes.c_int32),
                ("n_outliers", ctypes.c_int32), ("k_bulk", ctypes.c_int32), ("tau", ctypes.c_double),
                ("flags", ctypes.c_uint32), ("offset", ctypes.c_uint64 * 6),
                ("bytes", ctypes.c_uint64 * 6), ("crc32", ctypes.c_uint32 * 6)]


# name -> (restype, argtypes), mirroring spectra.h
P = ctypes.c_void_p
i32, f64, sz = ctypes.c_int32, ctypes.c_double, ctypes.c_size_t
LP = ctypes.POINTER(Layer)
SIGNATURES = {
    "spectra_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "spectra_version": (i32, []),
    "spectra_packed_sizes": (ctypes.c_int, [i32, i32, i32, ctypes.POINTER(Sizes)]),
    "spectra_pack_plan_workspace_size": (sz, [i32]),
    "spectra_pack_workspace_size": (sz, []),
    "spectra_pack_plan": (ctypes.c_int, [P, P, i32, i32, f64, P, P, ctypes.POINTER(i32), P, sz, P]),
    "spectra_pack": (ctypes.c_int, [P, i32, i32, P, i32, P, P, P, P, P, sz, LP, P]),
    "spectra_packed_sizes_compact": (ctypes.c_int, [i32, i32, i32, ctypes.POINTER(Sizes)]),
    "spectra_pack_compact": (ctypes.c_int, [P, i32, i32, P, i32, P, P, P, P, P, P, sz, LP, P]),
    "spectra_unpack": (ctypes.c_int, [LP, P, P, P, P]),
    "spectra_gemv": (ctypes.c_int, [LP, P, P, ctypes.c_int, P]),
    "spectra_gemm_small": (ctypes.c_int, [LP, P, i32, P, ctypes.c_int, P]),
    "spectra_gemv_batched": (ctypes.c_int, [LP, P, P, i32, ctypes.c_int, P]),
    "spectra_gemv_chain_workspace_size": (sz, [LP, i32]),
    "spectra_gemv_chain": (ctypes.c_int, [LP, P, P, i32, ctypes.c_int, P, sz, P]),
    "spectra_gemv_chain_staged": (ctypes.c_int, [LP, P, P, i32, ctypes.c_int, P, P, sz, P]),
    "spectra_device_status": (ctypes.c_int, [P]),
    "spectra_selftest_wait": (ctypes.c_int, [i32, P]),
    "spectra_embed": (ctypes.c_int, [LP, P, i32, P, ctypes.c_int, P]),
    "spectra_row_table_sizes": (ctypes.c_int, [LP, ctypes.POINTER(Sizes)]),
    "spectra_row_table_from_layer": (ctypes.c_int, [LP, P, P, P, P, LP, P]),
    "spectra_embed_rows": (ctypes.c_int, [LP, P, i32, P, ctypes.c_int, P]),
    "spectra_pack_plan_noalloc": (ctypes.c_int, [P, P, i32, i32, f64, P, P, ctypes.POINTER(i32), P]),
    "spectra_crc32": (ctypes.c_uint32, [ctypes.c_uint32, P, sz]),
    "spectra_kv_sizes": (ctypes.c_int, [i32, i32, i32, ctypes.POINTER(sz), ctypes.POINTER(sz),
                                        ctypes.POINTER(sz)]),
    "spectra_kv_append": (ctypes.c_int, [ctypes.POINTER(KV), P, i32, i32, P]),
    "spectra_attention_workspace_size": (sz, [i32, i32, i32]),
    "spectra_attention_decode": (ctypes.c_int, [ctypes.POINTER(KV), ctypes.POINTER(KV), P, i32, i32,
                                                ctypes.c_float, P, P, sz, P]),
    "spectra_trdc_write": (ctypes.c_int, [ctypes.c_char_p, i32, P, LP, P, ctypes.c_int, P, sz, P]),
    "spectra_trdc_open": (ctypes.c_int, [ctypes.c_char_p, ctypes.POINTER(P)]),
    "spectra_trdc_count": (i32, [P]),
    "spectra_trdc_info": (ctypes.c_int, [P, i32, ctypes.POINTER(TrdcLayer)]),
    "spectra_trdc_load": (ctypes.c_int, [P, i32, P, P, P, P, P, P, ctypes.c_int, P, sz, i32, LP, P]),
    "spectra_trdc_close": (None, [P]),
}

NOALLOC_MAX_K = 65536

MAX_BATCH = 224

_lib = None


def load() -> ctypes.CDLL:
    """Load libspectra.so from the package directory; raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m outlier_split_bit_b200.build` "
                "(there is no fallback implementation)")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib
