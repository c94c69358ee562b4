"""Group-32 4-bit KV cache on the GPU vs the CPU oracle.

Method: "SPECTRA: Sparse-Precision Exact Channel Tensor Reconstruction
Architecture" (Dev.to abstract), abstract paragraph: microscaled Group-32
4-bit key-value caching.  Appended tokens must be quantised and laid out bit
for bit like the oracle's; decode attention must stay within the tolerance
the oracle derives (the matvec's 2e-3 per dot product carried through the
softmax).
"""
import numpy as np
import pytest
import torch

import oracle
import outlier_split_bit_b200 as sp
from outlier_split_bit_b200 import workload as wl

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _tokens(n_tok, H, D, seed):
    x = wl.activations(H * D, n_tok, seed=seed, device=DEV)
    return x.reshape(n_tok, H, D)


def _fill(H, D, cap, T, seed, steps=(None,)):
    """GPU and oracle caches holding T tokens, appended as one prefill of
    T - len(tail) tokens followed by single tokens."""
    gk, gv = sp.KVCache(H, D, cap), sp.KVCache(H, D, cap)
    ok, ov = oracle.kv_cache(H, cap, D), oracle.kv_cache(H, cap, D)
    tail = min(3, T - 1)
    spans = [(0, T - tail)] + [(T - tail + i, 1) for i in range(tail)]
    for j, (pos, n) in enumerate(spans):
        if n == 0:
            continue
        xk, xv = _tokens(n, H, D, seed + 2 * j), _tokens(n, H, D, seed + 2 * j + 1)
        gk.append(xk, pos)
        gv.append(xv, pos)
        oracle.kv_quantize(ok, wl.bits(xk), pos)
        oracle.kv_quantize(ov, wl.bits(xv), pos)
    torch.cuda.synchronize()
    return gk, gv, ok, ov


def _packed(g: sp.KVCache):
    return (g.codes.cpu().numpy(), g.scales.cpu().numpy().view(np.uint16),
            g.zeros.cpu().numpy().view(np.uint32))


@pytest.mark.parametrize("H,D,T,cap", [(2, 128, 40, 64), (8, 64, 7, 7), (1, 256, 130, 200),
                                       (3, 32, 1, 5), (2, 96, 33, 33)])
def test_append_bit_exact(H, D, T, cap):
    gk, gv, ok, ov = _fill(H, D, cap, T, seed=H * 1000 + D)
    for g, o in ((gk, ok), (gv, ov)):
        got, want = _packed(g), oracle.kv_pack(o)
        for a, b in zip(got, want):
            assert np.array_equal(a, b)
    sp.spectra_device_status()


CASES = [(12, 2, 128, 1), (12, 2, 128, 127), (12, 2, 128, 128), (12, 2, 128, 129),
         (12, 2, 128, 2048), (32, 8, 128, 8192), (8, 8, 64, 300), (16, 2, 256, 777),
         (4, 1, 32, 50), (6, 3, 96, 200)]


@pytest.mark.parametrize("Hq,Hkv,D,T", CASES, ids=[f"q{a}-kv{b}-d{c}-t{d}" for a, b, c, d in CASES])
def test_attention_within_tolerance(Hq, Hkv, D, T):
    cap = T + 5
    gk, gv, ok, ov = _fill(Hkv, D, cap, T, seed=T + D)
    q = wl.activations(D, Hq, seed=T, device=DEV)
    scale = 1.0 / np.sqrt(D)
    out = sp.spectra_attention_decode(gk, gv, q, T, scale)
    torch.cuda.synchronize()
    ref, vb, sm = oracle.attention(ok, ov, wl.bits(q), T, np.float32(scale))
    err = np.abs(out.cpu().numpy().astype(np.float64) - ref)
    tol = oracle.attention_tolerance(vb, sm)
    assert (err <= tol).all(), f"worst ratio {(err / tol).max():.3g}"
    again = sp.spectra_attention_decode(gk, gv, q, T, scale)
    torch.cuda.synchronize()
    assert torch.equal(out, again)  # fixed reduction order


def test_attention_exact_cases():
    Hkv, D, T = 2, 128, 300
    gk, gv, ok, ov = _fill(Hkv, D, T, T, seed=7)
    what = (ov.codes.astype(np.float64) - np.repeat(ov.zeros, 32, axis=2)) * \
        np.repeat(ov.scales.view(np.float16).astype(np.float64), 32, axis=2)
    q = wl.activations(D, 4, seed=8, device=DEV)
    # one position: the softmax weight is exactly 1 and the output is v_hat
    out = sp.spectra_attention_decode(gk, gv, q, 1, 0.1).cpu().numpy()
    assert np.array_equal(out[:2].astype(np.float64), np.stack([what[0, 0]] * 2))
    assert np.array_equal(out[2:].astype(np.float64), np.stack([what[1, 0]] * 2))
    # a zero query: uniform weights, the mean of v_hat
    out = sp.spectra_attention_decode(gk, gv, torch.zeros_like(q), T, 0.1).cpu().numpy()
    assert np.allclose(out[0], what[0].mean(0), rtol=1e-5, atol=1e-6)
    assert np.allclose(out[3], what[1].mean(0), rtol=1e-5, atol=1e-6)


def test_append_reports_nonfinite_values():
    g = sp.KVCache(2, 64, 8)
    sp.spectra_device_status()
    x = _tokens(2, 2, 64, 3)
    x[1, 0, 40] = float("inf")
    g.append(x, 0)
    torch.cuda.synchronize()
    with pytest.raises(sp.SpectraError) as e:
        sp.spectra_device_status()
    assert e.value.status == 4
    o = oracle.kv_cache(2, 8, 64)
    ok = wl.bits(x).copy()
    oracle.kv_quantize(o, ok[:1], 0)  # token 0 is finite and stored normally
    codes, scales, zeros = _packed(g)
    want = oracle.kv_pack(o)
    assert np.array_equal(codes[: 64 // 2], want[0][: 64 // 2])
    # the bad group (head 0, token 1, channels 32..63) is all zeros
    slot, G = 0 * 8 + 1, 2
    assert not codes[(slot * G + 1) * 16:(slot * G + 2) * 16].any()
    assert scales[slot * G + 1] == 0
    sp.spectra_device_status()


def test_append_and_attention_graph_capture():
    H, D, cap = 2, 128, 64
    gk, gv, ok, ov = _fill(H, D, cap, 20, seed=11)
    xk, xv = _tokens(1, H, D, 12), _tokens(1, H, D, 13)
    q = wl.activations(D, 12, seed=14, device=DEV)
    out = torch.empty((12, D), device=DEV)
    ws = torch.empty(sp.library().spectra_attention_workspace_size(12, D, 21), dtype=torch.uint8,
                     device=DEV)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(graph, stream=s):
            gk.append(xk, 20, stream=s)
            gv.append(xv, 20, stream=s)
            sp.spectra_attention_decode(gk, gv, q, 21, None, out, workspace=ws, stream=s)
    graph.replay()
    torch.cuda.synchronize()
    oracle.kv_quantize(ok, wl.bits(xk), 20)
    oracle.kv_quantize(ov, wl.bits(xv), 20)
    ref, vb, sm = oracle.attention(ok, ov, wl.bits(q), 21, np.float32(1.0 / np.sqrt(D)))
    err = np.abs(out.cpu().numpy().astype(np.float64) - ref)
    assert (err <= oracle.attention_tolerance(vb, sm)).all()
