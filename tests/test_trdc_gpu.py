"""TRDC container on the GPU: device buffers out to a file and back.

Source: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
Architecture" (Dev.to abstract), abstract paragraph: weights, scales and
offsets are serialised into one self-contained binary container and
streamed into GPU memory with a bounded memory spike.  Packing on the GPU is
bit-exact against the oracle, so a container written from device buffers
must equal, byte for byte, the oracle's container of the oracle's packing;
loading it back through a small staging buffer must reproduce the device
buffers exactly.
"""
import numpy as np
import pytest
import torch

import oracle
import outlier_split_bit_b200 as sp
from oracle import trdc
from outlier_split_bit_b200 import workload as wl

from gpu_helpers import draw, np_gain

pytestmark = pytest.mark.gpu

SPECS = [(wl.LAYER_1P5B[0], 3.0, False), (wl.LAYER_1P5B[1], 6.0, True),
         (wl.MatrixSpec("single", 100, 2080, 31), 3.0, True), (wl.SINGLE_512, np.inf, False)]


def _packed():
    layers, entries, names = [], [], []
    for i, (spec, tau, compact) in enumerate(SPECS):
        w, g, _ = draw(spec, seed=7, layer=i)
        lay = sp.pack_layer(w, g, tau, compact=compact)
        wb = wl.bits(w)
        name = f"layers.{i}.{spec.name}"
        if compact:
            c = oracle.pack_compact(wb, np_gain(g), tau)
            entries.append(trdc.entry_from_packed(name, c.packed, tau, c.k_bulk, c.bulk_idx))
        else:
            p = oracle.pack(wb, np_gain(g), tau)
            entries.append(trdc.entry_from_packed(name, p.packed, tau))
        layers.append(lay)
        names.append(name)
    return layers, entries, names


def _same_buffers(a: sp.PackedLayer, b: sp.PackedLayer):
    for x, y in [(a.codes, b.codes), (a.scales, b.scales), (a.zeros, b.zeros)]:
        assert torch.equal(x, y)
    if a.n_outliers:
        assert torch.equal(a.outlier_idx[: a.n_outliers], b.outlier_idx[: b.n_outliers])
        assert torch.equal(a.outlier_w, b.outlier_w)
    assert (a.bulk_idx is None) == (b.bulk_idx is None)
    if a.bulk_idx is not None:
        assert torch.equal(a.bulk_idx, b.bulk_idx) and a.k_bulk == b.k_bulk


@pytest.mark.parametrize("staging_bytes", [8192, 1 << 20])
def test_device_container_round_trip(tmp_path, staging_bytes):
    layers, entries, names = _packed()
    taus = [t for _, t, _ in SPECS]
    path = tmp_path / "model.trdc"
    sp.write_container(path, layers, names, taus, staging_bytes=staging_bytes)
    assert path.read_bytes() == trdc.write_bytes(entries)
    with sp.Container(path) as c:
        assert len(c) == len(layers)
        for i, lay in enumerate(layers):
            inf = c.info(i)
            assert inf["name"] == names[i] and inf["compact"] == lay.compact
            back = c.load(i, staging_bytes=staging_bytes)
            torch.cuda.synchronize()
            _same_buffers(lay, back)
            x = wl.activations(lay.k, 1, seed=i, device="cuda")[0]
            assert torch.equal(sp.spectra_gemv(lay, x), sp.spectra_gemv(back, x))


def test_device_load_reports_a_damaged_buffer(tmp_path):
    layers, entries, names = _packed()
    data = bytearray(trdc.write_bytes(entries))
    off = int(np.frombuffer(bytes(data), dtype="<u8", count=1, offset=64 + 128)[0])
    data[off + 7] ^= 0x01
    path = tmp_path / "bad.trdc"
    path.write_bytes(bytes(data))
    with sp.Container(path) as c:
        with pytest.raises(sp.SpectraError) as e:
            c.load(0, staging_bytes=8192)
        assert e.value.status == 11
        c.load(0, staging_bytes=8192, verify=False)
        c.load(1, staging_bytes=8192)  # the other layers load
