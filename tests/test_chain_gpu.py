"""spectra_gemv_chain: a dependent sequence of batch-1 matvecs in one launch,
against the CPU oracle.

Method: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
Architecture" (Dev.to abstract), abstract paragraph and highlights: the
decode step, replayed as a CUDA graph, is a sequence of fused dequantise +
matvec calls whose inputs are earlier outputs.  Each matvec of the chain must
satisfy |y - y_ref| <= 2e-3 * sum|w_hat x| + 1e-5 against the oracle given
the x it actually read (a BF16 output adds its own rounding), every stage
must have read its predecessor's finished output, and the counter's bounded
wait must give up (reported, no fault) when its target is never reached.
spectra_gemv_chain_staged groups the matvecs as a decoder layer's dataflow
does (q, k, v share an input; so do gate and up): a matvec reads the output
of an earlier stage only.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import outlier_split_bit_b200 as sp
from outlier_split_bit_b200 import _lib
from outlier_split_bit_b200 import workload as wl

from gpu_helpers import DEV, check_gemv, draw, np_gain

pytestmark = pytest.mark.gpu

# (n, k) of each stage: the output of one stage is the input of the next
CHAIN = [(1536, 1536), (1536, 1536), (8960, 1536), (1536, 8960), (256, 1536), (1536, 256),
         (64, 1536), (96, 64), (2080, 96), (40, 2080)]


def _stages(tau, seed=11):
    stages = []
    for i, (n, k) in enumerate(CHAIN):
        spec = wl.MatrixSpec("single", n, k, max(1, round(0.015 * k)))
        w, g, _ = draw(spec, seed=seed, layer=i)
        stages.append((spec, w, g, sp.pack_layer(w, g, tau)))
    return stages


@pytest.mark.parametrize("tau", [3.0, 6.0])
def test_chain_feeds_each_stage_its_predecessor(tau):
    stages = _stages(tau)
    x0 = wl.activations(CHAIN[0][1], 1, seed=5, device=DEV)[0]
    bufs = [x0.clone()] + [torch.full((n,), float("nan"), dtype=torch.bfloat16, device=DEV)
                           for n, _ in CHAIN]
    layers = [lay for *_, lay in stages]
    sp.spectra_gemv_chain(layers, bufs[:-1], bufs[1:])
    torch.cuda.synchronize()
    sp.spectra_device_status()
    for i, (spec, w, g, lay) in enumerate(stages):
        x_in, y = bufs[i], bufs[i + 1]
        assert torch.isfinite(y.float()).all(), i
        wb = wl.bits(w)
        ref = oracle.pack(wb, np_gain(g), tau)
        y_ref, bound = oracle.gemm(ref.can, wb, ref.idx, wl.bits(x_in))
        check_gemv(y, y_ref[0], bound[0], bf16=True)


def test_chain_of_independent_matrices_against_oracle():
    """The 7 projections of two 1.5B-class layers, each with its own x (FP32
    y): every output against the oracle; a replay is bit-identical."""
    layers, xs, ys, refs = [], [], [], []
    for layer in range(2):
        for spec in wl.LAYER_1P5B:
            w, g, x = draw(spec, seed=7, layer=layer)
            layers.append(sp.pack_layer(w, g, 3.0))
            xs.append(x[0])
            ys.append(torch.full((spec.n,), float("nan"), device=DEV))
            refs.append((wl.bits(w), np_gain(g), wl.bits(x)))
    views = sp.spectra_gemv_chain(layers, xs, ys)
    torch.cuda.synchronize()
    sp.spectra_device_status()
    for y, (wb, gn, xb) in zip(ys, refs):
        ref = oracle.pack(wb, gn, 3.0)
        y_ref, bound = oracle.gemm(ref.can, wb, ref.idx, xb)
        check_gemv(y, y_ref[0], bound[0])
    y0 = [y.clone() for y in ys]
    sp.spectra_gemv_chain(views=views)
    torch.cuda.synchronize()
    for a, b in zip(y0, ys):
        assert torch.equal(a, b)


def test_chain_graph_capture_and_replay():
    stages = _stages(6.0, seed=12)
    x0 = wl.activations(CHAIN[0][1], 1, seed=6, device=DEV)[0]
    bufs = [x0.clone()] + [torch.empty((n,), dtype=torch.bfloat16, device=DEV) for n, _ in CHAIN]
    views = sp.spectra_gemv_chain([lay for *_, lay in stages], bufs[:-1], bufs[1:])
    torch.cuda.synchronize()
    eager = bufs[-1].clone()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            sp.spectra_gemv_chain(views=views, stream=s)
    for _ in range(3):
        for b in bufs[1:]:
            b.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(bufs[-1], eager)
    sp.spectra_device_status()


def _decoder_stages(tau, layers=2, seed=13):
    """Two 1.5B-class decoder layers as the staged chain runs them: q, k, v
    read one input (stage 0), o reads q's output (stage 1), gate and up read
    o's output (stage 2), down reads gate's output (stage 3); the next layer's
    q, k, v read down's output.  Outputs are BF16, every buffer distinct."""
    specs = {s.name: s for s in wl.LAYER_1P5B}
    x0 = wl.activations(specs["q"].k, 1, seed=7, device=DEV)[0]
    mats, xs, ys, stage = [], [], [], []
    cur = x0
    for layer in range(layers):
        def add(name, x, st):
            spec = specs[name]
            w, g, _ = draw(spec, seed=seed, layer=layer)
            mats.append((spec, w, g, sp.pack_layer(w, g, tau)))
            y = torch.full((spec.n,), float("nan"), dtype=torch.bfloat16, device=DEV)
            xs.append(x)
            ys.append(y)
            stage.append(st)
            return y
        base = 4 * layer
        yq = add("q", cur, base)
        add("k", cur, base)
        add("v", cur, base)
        yo = add("o", yq, base + 1)
        yg = add("gate", yo, base + 2)
        add("up", yo, base + 2)
        cur = add("down", yg, base + 3)
    return mats, xs, ys, stage


@pytest.mark.parametrize("tau", [3.0, 6.0])
def test_staged_chain_against_oracle(tau):
    """Each matvec reads the output of an earlier stage, never of its own;
    every output against the oracle given the x it read."""
    mats, xs, ys, stage = _decoder_stages(tau)
    views = sp.spectra_gemv_chain([m[3] for m in mats], xs, ys, stages=stage)
    torch.cuda.synchronize()
    sp.spectra_device_status()
    for (spec, w, g, lay), x_in, y in zip(mats, xs, ys):
        assert torch.isfinite(y.float()).all(), spec.name
        wb = wl.bits(w)
        ref = oracle.pack(wb, np_gain(g), tau)
        y_ref, bound = oracle.gemm(ref.can, wb, ref.idx, wl.bits(x_in))
        check_gemv(y, y_ref[0], bound[0], bf16=True)
    # a replay repeats every output bit for bit
    first = [y.clone() for y in ys]
    for y in ys:
        y.fill_(float("nan"))
    sp.spectra_gemv_chain(views=views, stages=stage)
    torch.cuda.synchronize()
    for a, b in zip(first, ys):
        assert torch.equal(a, b)


def test_staged_chain_with_one_stage_is_independent_matvecs():
    """One stage: no waits at all, the matvecs independent as in a grouped
    launch; every output against the oracle."""
    layers, xs, ys, refs = [], [], [], []
    for spec in wl.LAYER_1P5B:
        w, g, x = draw(spec, seed=9, layer=1)
        layers.append(sp.pack_layer(w, g, 3.0))
        xs.append(x[0])
        ys.append(torch.full((spec.n,), float("nan"), device=DEV))
        refs.append((wl.bits(w), np_gain(g), wl.bits(x)))
    sp.spectra_gemv_chain(layers, xs, ys, stages=[0] * len(layers))
    torch.cuda.synchronize()
    sp.spectra_device_status()
    for y, (wb, gn, xb) in zip(ys, refs):
        ref = oracle.pack(wb, gn, 3.0)
        y_ref, bound = oracle.gemm(ref.can, wb, ref.idx, xb)
        check_gemv(y, y_ref[0], bound[0])


def test_staged_chain_with_one_matvec_per_stage_is_the_chain():
    mats, xs, ys, _ = _decoder_stages(3.0, layers=1)
    layers = [m[3] for m in mats]
    sp.spectra_gemv_chain(layers, xs, ys)
    torch.cuda.synchronize()
    plain = [y.clone() for y in ys]
    for y in ys:
        y.fill_(float("nan"))
    sp.spectra_gemv_chain(layers, xs, ys, stages=list(range(len(layers))))
    torch.cuda.synchronize()
    for a, b in zip(plain, ys):
        assert torch.equal(a, b)


def test_counter_wait_runs_out_and_reports_internal():
    sp.spectra_device_status()
    t0 = time.perf_counter()
    sp.spectra_selftest_wait(1)
    torch.cuda.synchronize()
    assert 0.9 < time.perf_counter() - t0 < 30.0
    with pytest.raises(sp.SpectraError) as e:
        sp.spectra_device_status()
    assert e.value.status == _lib.ERR_INTERNAL
    sp.spectra_device_status()
    # the context still runs a chain correctly
    test_chain_of_independent_matrices_against_oracle()
