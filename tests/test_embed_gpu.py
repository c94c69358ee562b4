"""Embedding-row gather on the GPU vs the CPU oracle, bit for bit.

Method: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
Architecture" (Dev.to abstract), abstract paragraph and highlight 5
(SpectraFusedEmbedding: vocabulary tables in the 4-bit Group-32 format,
rows gathered and dequantised during the forward pass).  Every gathered value
is exact -- (c - z) * s in FP32, or the stored BF16 of an outlier column --
and a BF16 output rounds it once, so both output types must match the
oracle's values bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import outlier_split_bit_b200 as sp
from outlier_split_bit_b200 import workload as wl

from gpu_helpers import DEV, draw, np_gain, oracle_split

pytestmark = pytest.mark.gpu

TABLES = [
    (wl.MatrixSpec("lm_head", 512, 512, 10), 3.0),
    (wl.MatrixSpec("lm_head", 512, 512, 10), 6.0),
    (wl.MatrixSpec("single", 40, 96, 3), 1.2),
    (wl.MatrixSpec("single", 7, 352, 17), 3.0),
    (wl.MatrixSpec("single", 1, 32, 0), 3.0),
    (wl.MatrixSpec("single", 33, 64, 2), -np.inf),
    (wl.MatrixSpec("single", 96, 256, 4), np.inf),
    (wl.MatrixSpec("single", 100, 9000 // 32 * 32, 60), 6.0),
]
IDS = [f"{s.n}x{s.k}-tau{t}" for s, t in TABLES]


def _ids(n, m, seed):
    rng = np.random.default_rng(seed)
    ids = rng.integers(0, n, m)
    ids[0] = n - 1 if m == 1 else 0
    if m > 1:
        ids[1] = n - 1
    if m > 4:
        ids[4] = ids[3]  # a repeated id
    return ids.astype(np.int32)


def _expected_bits(rows: np.ndarray, dtype) -> np.ndarray:
    if dtype == torch.float32:
        return rows.astype(np.float32).view(np.uint32)  # every value is exact in FP32
    return oracle.double_to_bf16(rows)


def _got_bits(out: torch.Tensor) -> np.ndarray:
    a = out.detach().cpu()
    if a.dtype == torch.float32:
        return a.numpy().view(np.uint32)
    return a.view(torch.int16).numpy().view(np.uint16)


def _pack_both(spec, tau, seed=0):
    w, g, _ = draw(spec, seed=seed)
    lay = sp.pack_layer(w, g, tau)
    wb = wl.bits(w)
    ref = oracle.pack(wb, np_gain(g), tau)
    return lay, wb, ref


@pytest.mark.parametrize("spec,tau", TABLES, ids=IDS)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_embed_rows_bit_exact(spec, tau, dtype):
    lay, wb, ref = _pack_both(spec, tau)
    assert lay.n_outliers == ref.idx.size
    assert np.array_equal(lay.outlier_idx.cpu().numpy()[: ref.idx.size], ref.idx)
    for m in (1, 5, 67):
        ids = _ids(spec.n, m, seed=m)
        out = sp.spectra_embed(lay, torch.from_numpy(ids).to(DEV), out_dtype=dtype)
        torch.cuda.synchronize()
        rows = oracle.embed(ref.can, wb, ref.idx, ids)
        assert np.array_equal(_got_bits(out), _expected_bits(rows, dtype))
    sp.spectra_device_status()


@pytest.mark.parametrize("frac", [0.01, 0.10])
def test_embed_lm_head_full_size_sampled(frac):
    """The 131072 x 3072 table (the LM head's packed buffers, as a tied
    embedding would use them): 96 ids drawn over the whole vocabulary, checked
    against the oracle's reconstruction of those rows."""
    spec = wl.lm_head_spec(frac)
    w, g, _ = draw(spec)
    lay = sp.pack_layer(w, g, 6.0)
    wb = wl.bits(w)
    _, ref_idx = oracle_split(wb, np_gain(g), 6.0, key=("lm_head", frac))
    assert lay.n_outliers == ref_idx.size
    assert np.array_equal(lay.outlier_idx.cpu().numpy()[: ref_idx.size], ref_idx)
    ids = _ids(spec.n, 96, seed=5)
    for dtype in (torch.bfloat16, torch.float32):
        out = sp.spectra_embed(lay, torch.from_numpy(ids).to(DEV), out_dtype=dtype)
        torch.cuda.synchronize()
        uniq, inv = np.unique(ids, return_inverse=True)
        sub = np.ascontiguousarray(wb[uniq])
        can = oracle.quantize(sub, ref_idx)
        rows = oracle.embed(can, sub, ref_idx, inv.astype(np.int32))
        assert np.array_equal(_got_bits(out), _expected_bits(rows, dtype))


def test_embed_bad_ids_give_zero_rows_and_a_status():
    spec = wl.MatrixSpec("single", 70, 128, 3)
    lay, wb, ref = _pack_both(spec, 3.0)
    assert ref.idx.size > 0
    sp.spectra_device_status()
    ids = np.array([3, -1, 69, 70, 1 << 30, 0], dtype=np.int32)
    out = sp.spectra_embed(lay, torch.from_numpy(ids).to(DEV), out_dtype=torch.float32)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    assert np.all(got[[1, 3, 4]] == 0.0)
    good = ids[[0, 2, 5]]
    rows = oracle.embed(ref.can, wb, ref.idx, good)
    assert np.array_equal(got[[0, 2, 5]].view(np.uint32), rows.astype(np.float32).view(np.uint32))
    with pytest.raises(sp.SpectraError) as e:
        sp.spectra_device_status()
    assert e.value.status == 1
    sp.spectra_device_status()  # the flag was cleared


def test_embed_no_rows_touches_nothing():
    spec = wl.MatrixSpec("single", 64, 64, 1)
    lay, _, _ = _pack_both(spec, 3.0)
    out = sp.spectra_embed(lay, torch.empty(0, dtype=torch.int32, device=DEV))
    assert out.shape == (0, 64)


def test_embed_feeds_a_dependent_matvec():
    """Gathered BF16 rows are the x of the next matvec on the same stream: the
    programmatic dependent launch of the matvec must wait for the gather; the
    gather, launched after a matvec whose output it does not read, must still
    read ids written before it."""
    table_spec = wl.MatrixSpec("lm_head", 4096, 1536, 23)
    lay_t, wb_t, ref_t = _pack_both(table_spec, 6.0, seed=1)
    q_spec = wl.MatrixSpec("q", 1536, 1536, 23)
    w, g, _ = draw(q_spec, seed=2)
    lay_q = sp.pack_layer(w, g, 6.0)
    ref_q = oracle.pack(wl.bits(w), np_gain(g), 6.0)
    ids_host = np.array([17, 4095, 0, 2048], dtype=np.int32)
    ids = torch.empty(4, dtype=torch.int32, device=DEV)
    xs = torch.empty((4, 1536), dtype=torch.bfloat16, device=DEV)
    ys = torch.empty((4, 1536), dtype=torch.float32, device=DEV)
    for rep in range(3):
        ids.copy_(torch.from_numpy(np.roll(ids_host, rep)))
        for r in range(4):
            sp.spectra_embed(lay_t, ids[r:r + 1], xs[r:r + 1])
            sp.spectra_gemv(lay_q, xs[r], ys[r])
        torch.cuda.synchronize()
        rows = oracle.embed(ref_t.can, wb_t, ref_t.idx, np.roll(ids_host, rep))
        x_bits = oracle.double_to_bf16(rows)
        assert np.array_equal(xs.cpu().view(torch.int16).numpy().view(np.uint16), x_bits)
        y_ref, bound = oracle.gemm(ref_q.can, wl.bits(w), ref_q.idx, x_bits)
        y = ys.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(y - y_ref) <= oracle.tolerance(bound))


def test_embed_graph_capture_and_replay():
    spec = wl.MatrixSpec("lm_head", 2048, 3072, 31)
    lay, _, _ = _pack_both(spec, 6.0)
    ids = torch.from_numpy(_ids(spec.n, 33, seed=9)).to(DEV)
    eager = sp.spectra_embed(lay, ids).clone()
    out = torch.empty_like(eager)
    view = lay.view()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            sp.spectra_embed(lay, ids, out, view=view, stream=s)
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
