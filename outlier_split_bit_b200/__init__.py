"""B200 (sm_100a) SPECTRA outlier-split INT4 decode matvec.

Thin Python binding of the C ABI in ``include/spectra.h``: argument
marshalling only.  Every step of the path (kurtosis, split, quantisation,
packing, fused dequantise+matvec) runs in the library's CUDA kernels; PyTorch
provides device memory and streams.  There is no CPU fallback: importing
the binding loads ``libspectra.so`` on first use and raises ImportError when
it is missing.

Method: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
Architecture" (Dev.to abstract re-post), abstract paragraph.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import KV, Layer, Sizes, TrdcLayer

__all__ = ["SpectraError", "PackedLayer", "spectra_status_string", "spectra_version",
           "spectra_packed_sizes", "spectra_packed_sizes_compact", "spectra_pack_plan",
           "spectra_pack", "spectra_pack_compact", "spectra_unpack",
           "spectra_gemv", "spectra_gemm_small", "spectra_gemv_batched", "spectra_embed",
           "spectra_device_status",
           "pack_layer", "library", "spectra_crc32", "write_container", "Container", "KVCache",
           "spectra_attention_decode"]

class _Lazy:
    """Loads libspectra.so on first attribute access."""

    def __getattr__(self, name):
        return getattr(_lib.load(), name)


_L = _Lazy()


def library() -> ctypes.CDLL:
    return _lib.load()


class SpectraError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        msg = _L.spectra_status_string(status).decode()
        super().__init__(f"{where}: {msg} (status {status})" if where else msg)
        self.status = status


def _check(status: int, where: str):
    if status != _lib.OK:
        raise SpectraError(status, where)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def spectra_status_string(status: int) -> str:
    return _L.spectra_status_string(status).decode()


def spectra_version() -> int:
    return _L.spectra_version()


def spectra_device_status(*, stream=None) -> None:
    """Raise SpectraError if a bounded wait in a matvec kernel gave up."""
    _check(_L.spectra_device_status(_stream(stream)), "spectra_device_status")


def spectra_selftest_wait(kind: int = 0, *, stream=None) -> None:
    """Launch a kernel whose bounded wait can never be satisfied; the next
    spectra_device_status reports SPECTRA_ERR_INTERNAL."""
    _check(_L.spectra_selftest_wait(int(kind), _stream(stream)), "spectra_selftest_wait")


def _sizes(s: Sizes) -> dict:
    return {"n_pad": s.n_pad, "codes": s.codes_bytes, "scales": s.scales_bytes,
            "zeros": s.zeros_bytes, "outlier_idx": s.outlier_idx_bytes,
            "outlier_w": s.outlier_w_bytes, "k_bulk": s.k_bulk, "bulk_idx": s.bulk_idx_bytes}


def spectra_packed_sizes(n: int, k: int, n_outliers: int) -> dict:
    s = Sizes()
    _check(_L.spectra_packed_sizes(n, k, n_outliers, ctypes.byref(s)), "spectra_packed_sizes")
    return _sizes(s)


def spectra_packed_sizes_compact(n: int, k: int, n_outliers: int) -> dict:
    s = Sizes()
    _check(_L.spectra_packed_sizes_compact(n, k, n_outliers, ctypes.byref(s)),
           "spectra_packed_sizes_compact")
    return _sizes(s)


def spectra_pack_plan(w: torch.Tensor, gain: torch.Tensor | None, tau: float, *,
                      want_kappa: bool = False, stream=None):
    """Kurtosis split.  Returns (idx int32 [n_o], kappa float64 [k] or None)."""
    n, k = w.shape
    dev = w.device
    kappa = torch.empty(k, dtype=torch.float64, device=dev) if want_kappa else None
    idx = torch.empty(max(k, 1), dtype=torch.int32, device=dev)
    ws_bytes = _L.spectra_pack_plan_workspace_size(k)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    n_o = ctypes.c_int32(0)
    _check(_L.spectra_pack_plan(_ptr(w), _ptr(gain), n, k, float(tau), _ptr(kappa), _ptr(idx),
                                ctypes.byref(n_o), _ptr(ws), ws_bytes, _stream(stream)),
           "spectra_pack_plan")
    return idx[: n_o.value], kappa


@dataclass
class PackedLayer:
    """Device buffers of one packed layer plus the C view over them."""
    n: int
    k: int
    n_outliers: int
    codes: torch.Tensor        # uint8
    scales: torch.Tensor       # int16 storage of FP16 bits
    zeros: torch.Tensor        # int32 storage of u32 words
    outlier_idx: torch.Tensor  # int32
    outlier_w: torch.Tensor    # int16 storage of BF16 bits
    bulk_idx: torch.Tensor | None = None  # int32 [k_bulk]: compacted bulk only
    k_bulk: int = 0                       # bulk columns (k when masked)

    def __post_init__(self):
        if self.k_bulk == 0:
            self.k_bulk = self.k

    @property
    def compact(self) -> bool:
        return self.bulk_idx is not None

    def view(self) -> Layer:
        return Layer(self.n, self.k, self.n_outliers, _ptr(self.codes), _ptr(self.scales),
                     _ptr(self.zeros), _ptr(self.outlier_idx) if self.n_outliers else None,
                     _ptr(self.outlier_w) if self.n_outliers else None,
                     self.k_bulk, _ptr(self.bulk_idx))

    @property
    def nbytes(self) -> int:
        """Bytes a matvec streams from these buffers (codes, scales, zeros,
        outlier weights and indices, and the bulk column list)."""
        return (self.codes.numel() + 2 * self.scales.numel() + 4 * self.zeros.numel()
                + 4 * self.n_outliers + 2 * self.outlier_w.numel()
                + (4 * self.bulk_idx.numel() if self.compact else 0))


def _alloc(nbytes: int, dtype, dev):
    item = torch.empty((), dtype=dtype).element_size()
    return torch.zeros(max(nbytes // item, 1), dtype=dtype, device=dev)


def spectra_pack(w: torch.Tensor, idx: torch.Tensor, *, stream=None) -> PackedLayer:
    """Quantise and pack W given the outlier indices from spectra_pack_plan."""
    n, k = w.shape
    n_o = int(idx.numel())
    dev = w.device
    sz = spectra_packed_sizes(n, k, n_o)
    codes = _alloc(sz["codes"], torch.uint8, dev)
    scales = _alloc(sz["scales"], torch.int16, dev)
    zeros = _alloc(sz["zeros"], torch.int32, dev)
    outw = _alloc(sz["outlier_w"], torch.int16, dev)
    idx_c = idx.contiguous() if n_o else torch.zeros(1, dtype=torch.int32, device=dev)
    ws_bytes = _L.spectra_pack_workspace_size()
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    view = Layer()
    _check(_L.spectra_pack(_ptr(w), n, k, _ptr(idx_c) if n_o else None, n_o, _ptr(codes),
                           _ptr(scales), _ptr(zeros), _ptr(outw) if n_o else None, _ptr(ws),
                           ws_bytes, ctypes.byref(view), _stream(stream)), "spectra_pack")
    return PackedLayer(n, k, n_o, codes, scales, zeros, idx_c, outw)


def spectra_pack_compact(w: torch.Tensor, idx: torch.Tensor, *, stream=None) -> PackedLayer:
    """Quantise and pack W with the outlier columns removed from the bulk."""
    n, k = w.shape
    n_o = int(idx.numel())
    dev = w.device
    sz = spectra_packed_sizes_compact(n, k, n_o)
    codes = _alloc(sz["codes"], torch.uint8, dev)
    scales = _alloc(sz["scales"], torch.int16, dev)
    zeros = _alloc(sz["zeros"], torch.int32, dev)
    outw = _alloc(sz["outlier_w"], torch.int16, dev)
    bidx = torch.empty(sz["k_bulk"], dtype=torch.int32, device=dev)
    idx_c = idx.contiguous() if n_o else torch.zeros(1, dtype=torch.int32, device=dev)
    ws_bytes = _L.spectra_pack_workspace_size()
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    view = Layer()
    _check(_L.spectra_pack_compact(_ptr(w), n, k, _ptr(idx_c) if n_o else None, n_o, _ptr(codes),
                                   _ptr(scales), _ptr(zeros), _ptr(outw) if n_o else None,
                                   _ptr(bidx), _ptr(ws), ws_bytes, ctypes.byref(view),
                                   _stream(stream)), "spectra_pack_compact")
    return PackedLayer(n, k, n_o, codes, scales, zeros, idx_c, outw, bidx, sz["k_bulk"])


def pack_layer(w: torch.Tensor, gain: torch.Tensor | None, tau: float, *, compact: bool = False,
               stream=None):
    """spectra_pack_plan followed by spectra_pack (or spectra_pack_compact)."""
    idx, _ = spectra_pack_plan(w, gain, tau, stream=stream)
    if compact:
        return spectra_pack_compact(w, idx, stream=stream)
    return spectra_pack(w, idx, stream=stream)


def spectra_unpack(layer: PackedLayer, *, stream=None):
    """Canonical (codes u8 [n,kb], scales int16-bits [n,kb/32], zeros u8 [n,kb/32]),
    kb = k_bulk (k for a masked bulk)."""
    dev = layer.codes.device
    G = layer.k_bulk // 32
    codes = torch.empty((layer.n, layer.k_bulk), dtype=torch.uint8, device=dev)
    scales = torch.empty((layer.n, G), dtype=torch.int16, device=dev)
    zeros = torch.empty((layer.n, G), dtype=torch.uint8, device=dev)
    v = layer.view()
    _check(_L.spectra_unpack(ctypes.byref(v), _ptr(codes), _ptr(scales), _ptr(zeros),
                             _stream(stream)), "spectra_unpack")
    return codes, scales, zeros


_DT = {torch.float32: _lib.F32, torch.bfloat16: _lib.BF16}


def spectra_gemv(layer: PackedLayer, x: torch.Tensor, y: torch.Tensor | None = None, *,
                 y_dtype=torch.float32, view: Layer | None = None, stream=None) -> torch.Tensor:
    """y = W_hat x for one BF16 vector x [k]."""
    if y is None:
        y = torch.empty(layer.n, dtype=y_dtype, device=x.device)
    v = layer.view() if view is None else view
    _check(_L.spectra_gemv(ctypes.byref(v), _ptr(x), _ptr(y), _DT[y.dtype], _stream(stream)),
           "spectra_gemv")
    return y


def spectra_gemm_small(layer: PackedLayer, x: torch.Tensor, y: torch.Tensor | None = None, *,
                       y_dtype=torch.float32, view: Layer | None = None,
                       stream=None) -> torch.Tensor:
    """y [m, n] = x [m, k] W_hat^T for 1 <= m <= 32."""
    m = x.shape[0]
    if y is None:
        y = torch.empty((m, layer.n), dtype=y_dtype, device=x.device)
    v = layer.view() if view is None else view
    _check(_L.spectra_gemm_small(ctypes.byref(v), _ptr(x), m, _ptr(y), _DT[y.dtype],
                                 _stream(stream)), "spectra_gemm_small")
    return y


def spectra_embed(table: PackedLayer, ids: torch.Tensor, out: torch.Tensor | None = None, *,
                  out_dtype=torch.bfloat16, view: Layer | None = None,
                  stream=None) -> torch.Tensor:
    """Rows ids (int32 [m]) of a packed table, dequantised: out [m, k]."""
    m = int(ids.numel())
    if out is None:
        out = torch.empty((m, table.k), dtype=out_dtype, device=ids.device)
    v = table.view() if view is None else view
    _check(_L.spectra_embed(ctypes.byref(v), _ptr(ids) if m else None, m,
                            _ptr(out) if m else None, _DT[out.dtype], _stream(stream)),
           "spectra_embed")
    return out


@dataclass
class RowTable:
    """Row-table buffers of a packed table (every row's pieces contiguous,
    for gathers only) and the view over them; the index lists are the
    layer's own."""
    layer: PackedLayer
    codes: torch.Tensor
    scales: torch.Tensor
    zeros: torch.Tensor
    outlier_w: torch.Tensor
    _view: Layer

    def view(self) -> Layer:
        return self._view

    @property
    def n(self) -> int:
        return self.layer.n

    @property
    def k(self) -> int:
        return self.layer.k


def spectra_row_table_from_layer(layer: PackedLayer, *, stream=None) -> RowTable:
    """Convert a packed layer (RT32) into a row table (new device buffers)."""
    v = layer.view()
    sz = Sizes()
    _check(_L.spectra_row_table_sizes(ctypes.byref(v), ctypes.byref(sz)), "spectra_row_table_sizes")
    dev = layer.codes.device
    codes = _alloc(sz.codes_bytes, torch.uint8, dev)
    scales = _alloc(sz.scales_bytes, torch.int16, dev)
    zeros = _alloc(sz.zeros_bytes, torch.int32, dev)
    outw = _alloc(max(2, sz.outlier_w_bytes), torch.int16, dev)
    out = Layer()
    _check(_L.spectra_row_table_from_layer(ctypes.byref(v), _ptr(codes), _ptr(scales), _ptr(zeros),
                                           _ptr(outw) if layer.n_outliers else None, ctypes.byref(out),
                                           _stream(stream)), "spectra_row_table_from_layer")
    return RowTable(layer, codes, scales, zeros, outw, out)


def spectra_embed_rows(table: RowTable, ids: torch.Tensor, out: torch.Tensor | None = None, *,
                       out_dtype=torch.bfloat16, stream=None) -> torch.Tensor:
    """spectra_embed over a row table: rows ids (int32 [m]) dequantised, out [m, k]."""
    m = int(ids.numel())
    if out is None:
        out = torch.empty((m, table.k), dtype=out_dtype, device=ids.device)
    _check(_L.spectra_embed_rows(ctypes.byref(table.view()), _ptr(ids) if m else None, m,
                                 _ptr(out) if m else None, _DT[out.dtype], _stream(stream)),
           "spectra_embed_rows")
    return out


class BatchViews:
    """Host arrays of layer views and device pointers for spectra_gemv_batched,
    built once and reused (e.g. for graph capture)."""

    def __init__(self, layers, xs, ys):
        n = len(layers)
        self.count = n
        self.layers = (Layer * n)(*[l.view() for l in layers])
        self.xs = (ctypes.c_void_p * n)(*[x.data_ptr() for x in xs])
        self.ys = (ctypes.c_void_p * n)(*[y.data_ptr() for y in ys])
        dts = {y.dtype for y in ys}
        if len(dts) != 1:
            raise ValueError("all outputs of one batched call share one dtype")
        self.y_dtype = _DT[dts.pop()]
        self._keep = (list(layers), list(xs), list(ys))


def spectra_gemv_batched(layers=None, xs=None, ys=None, *, views: BatchViews | None = None,
                         stream=None) -> BatchViews:
    """Independent batch-1 matvecs ys[i] = W_i xs[i] in one launch."""
    v = views if views is not None else BatchViews(layers, xs, ys)
    _check(_L.spectra_gemv_batched(v.layers, v.xs, v.ys, v.count, v.y_dtype, _stream(stream)),
           "spectra_gemv_batched")
    return v


def spectra_gemv_chain(layers=None, xs=None, ys=None, *, views: BatchViews | None = None,
                       stages=None, workspace: torch.Tensor | None = None,
                       stream=None) -> BatchViews:
    """Dependent batch-1 matvecs ys[i] = W_i xs[i], i in order, in one launch;
    xs[i] may be an earlier ys[j].  With `stages` (a nondecreasing sequence of
    ints, one per matvec) matvec i waits only for the matvecs of earlier
    stages (spectra_gemv_chain_staged).  `workspace` (device, >=
    spectra_gemv_chain_workspace_size(layers, count) bytes) holds the launch's
    completion counter; one is allocated and kept with the views when none is
    given."""
    v = views if views is not None else BatchViews(layers, xs, ys)
    if workspace is None:
        workspace = getattr(v, "_chain_ws", None)
    if workspace is None:
        dev = v._keep[2][0].device
        nbytes = _L.spectra_gemv_chain_workspace_size(v.layers, v.count)
        if nbytes == 0:
            raise SpectraError(_lib.ERR_INVALID_ARG, "spectra_gemv_chain_workspace_size")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        v._chain_ws = workspace
    wsb = workspace.numel() * workspace.element_size()
    if stages is None:
        _check(_L.spectra_gemv_chain(v.layers, v.xs, v.ys, v.count, v.y_dtype, workspace.data_ptr(),
                                     wsb, _stream(stream)), "spectra_gemv_chain")
    else:
        st = (ctypes.c_int32 * len(stages))(*[int(s) for s in stages])
        if len(stages) != v.count:
            raise SpectraError(_lib.ERR_INVALID_ARG, "spectra_gemv_chain_staged: one stage per matvec")
        _check(_L.spectra_gemv_chain_staged(v.layers, v.xs, v.ys, v.count, v.y_dtype, st,
                                            workspace.data_ptr(), wsb, _stream(stream)),
               "spectra_gemv_chain_staged")
    return v


# ---------------------------------------------------------------- TRDC container

_BUFFERS = ("codes", "scales", "zeros", "outlier_idx", "outlier_w", "bulk_idx")


def spectra_crc32(data, crc: int = 0) -> int:
    """CRC-32 of a bytes-like object (the checksum stored in containers)."""
    buf = (ctypes.c_char * len(data)).from_buffer_copy(bytes(data))
    return int(_L.spectra_crc32(crc, buf, len(data)))


def _pinned(nbytes: int) -> torch.Tensor:
    return torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)


def write_container(path: str, layers, names, taus=None, *, staging_bytes: int = 64 << 20,
                    stream=None) -> None:
    """Write packed layers (device buffers) into a TRDC container, streaming
    them through a pinned staging buffer of staging_bytes."""
    n = len(layers)
    views = (Layer * n)(*[l.view() for l in layers])
    cnames = (ctypes.c_char_p * n)(*[nm.encode() for nm in names])
    ctaus = (ctypes.c_double * n)(*(taus if taus is not None else [0.0] * n))
    staging = _pinned(staging_bytes)
    _check(_L.spectra_trdc_write(str(path).encode(), n, cnames, views, ctaus, _lib.MEM_DEVICE,
                                 _ptr(staging), staging_bytes, _stream(stream)),
           "spectra_trdc_write")


class Container:
    """An open TRDC container: layer records, and layers streamed into device
    buffers that this binding allocates with torch."""

    def __init__(self, path: str):
        h = ctypes.c_void_p()
        _check(_L.spectra_trdc_open(str(path).encode(), ctypes.byref(h)), "spectra_trdc_open")
        self._h = h

    def close(self):
        if self._h:
            _L.spectra_trdc_close(self._h)
            self._h = None

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __len__(self) -> int:
        return int(_L.spectra_trdc_count(self._h))

    def info(self, i: int) -> dict:
        r = TrdcLayer()
        _check(_L.spectra_trdc_info(self._h, i, ctypes.byref(r)), "spectra_trdc_info")
        return {"name": r.name.decode(), "n": r.n, "k": r.k, "n_outliers": r.n_outliers,
                "k_bulk": r.k_bulk, "tau": r.tau, "compact": bool(r.flags & 1),
                "offset": list(r.offset), "bytes": list(r.bytes), "crc32": list(r.crc32)}

    def load(self, i: int, device="cuda", *, staging: torch.Tensor | None = None,
             staging_bytes: int = 64 << 20, verify: bool = True, stream=None) -> PackedLayer:
        """Stream layer i into new device buffers; returns the PackedLayer."""
        inf = self.info(i)
        nb = dict(zip(_BUFFERS, inf["bytes"]))
        codes = _alloc(nb["codes"], torch.uint8, device)
        scales = _alloc(nb["scales"], torch.int16, device)
        zeros = _alloc(nb["zeros"], torch.int32, device)
        oidx = _alloc(max(nb["outlier_idx"], 4), torch.int32, device)
        outw = _alloc(max(nb["outlier_w"], 2), torch.int16, device)
        bidx = _alloc(nb["bulk_idx"], torch.int32, device) if inf["compact"] else None
        if staging is None:
            staging = _pinned(staging_bytes)
        view = Layer()
        _check(_L.spectra_trdc_load(self._h, i, _ptr(codes), _ptr(scales), _ptr(zeros), _ptr(oidx),
                                    _ptr(outw), _ptr(bidx), _lib.MEM_DEVICE, _ptr(staging),
                                    staging.numel(), 1 if verify else 0, ctypes.byref(view),
                                    _stream(stream)), "spectra_trdc_load")
        return PackedLayer(inf["n"], inf["k"], inf["n_outliers"], codes, scales, zeros, oidx, outw,
                           bidx, inf["k_bulk"] if inf["compact"] else 0)


# ---------------------------------------------------------------- KV cache

class KVCache:
    """One Group-32 4-bit KV cache (K or V) in device buffers allocated here
    with torch: n_heads x capacity positions of head_dim channels."""

    def __init__(self, n_heads: int, head_dim: int, capacity: int, device="cuda"):
        cb, sb, zb = ctypes.c_size_t(), ctypes.c_size_t(), ctypes.c_size_t()
        _check(_L.spectra_kv_sizes(n_heads, head_dim, capacity, ctypes.byref(cb), ctypes.byref(sb),
                                   ctypes.byref(zb)), "spectra_kv_sizes")
        self.n_heads, self.head_dim, self.capacity = n_heads, head_dim, capacity
        self.codes = torch.zeros(cb.value, dtype=torch.uint8, device=device)
        self.scales = torch.zeros(sb.value // 2, dtype=torch.int16, device=device)
        self.zeros = torch.zeros(zb.value // 4, dtype=torch.int32, device=device)
        self._view = KV(n_heads, head_dim, capacity, _ptr(self.codes), _ptr(self.scales),
                        _ptr(self.zeros))

    def view(self) -> KV:
        return self._view

    @property
    def nbytes(self) -> int:
        return self.codes.numel() + 2 * self.scales.numel() + 4 * self.zeros.numel()

    def append(self, x: torch.Tensor, pos: int, *, stream=None) -> None:
        """Quantise x (BF16 [n_tok, n_heads, head_dim]) into positions pos.."""
        n_tok = x.shape[0] if x.numel() else 0
        _check(_L.spectra_kv_append(ctypes.byref(self._view), _ptr(x) if n_tok else None, n_tok, pos,
                                    _stream(stream)), "spectra_kv_append")


def spectra_attention_decode(k: KVCache, v: KVCache, q: torch.Tensor, length: int,
                             scale: float | None = None, out: torch.Tensor | None = None, *,
                             workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Decode attention of q (BF16 [n_q_heads, head_dim]) over positions
    0..length-1 of the caches; returns float [n_q_heads, head_dim]."""
    hq, d = q.shape
    if scale is None:
        scale = 1.0 / d ** 0.5
    if out is None:
        out = torch.empty((hq, d), dtype=torch.float32, device=q.device)
    need = _L.spectra_attention_workspace_size(hq, d, length)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    _check(_L.spectra_attention_decode(ctypes.byref(k.view()), ctypes.byref(v.view()), _ptr(q), hq,
                                       length, float(scale), _ptr(out), _ptr(workspace),
                                       workspace.numel(), _stream(stream)),
           "spectra_attention_decode")
    return out
