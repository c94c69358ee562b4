"""spectra_pack_plan_noalloc: the saliency split for callers that cannot call
cudaMalloc (code running under a foreign allocator or a pre-carved pool,
tools that must leave a process's allocations untouched).  It must give the
same kurtosis values and outlier indices as spectra_pack_plan, which takes a
caller workspace, on consecutive calls, while allocating nothing itself.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import ctypes
import gc

import numpy as np
import pytest
import torch

import outlier_split_bit_b200 as sp
from outlier_split_bit_b200 import _lib
from outlier_split_bit_b200 import workload as wl

pytestmark = pytest.mark.gpu

DEV = "cuda"


def _noalloc(L, w, g, tau, kappa_out):
    n, k = w.shape
    idx = torch.full((k,), -7, dtype=torch.int32, device=DEV)
    n_o = ctypes.c_int32(-1)
    stream = torch.cuda.current_stream().cuda_stream
    torch.cuda.synchronize()
    gc.collect()  # no collection of earlier tests' tensors inside the measured call
    gc.disable()
    args = (w.data_ptr(), None if g is None else g.data_ptr(), n, k, float(tau),
            None if kappa_out is None else kappa_out.data_ptr(), idx.data_ptr(), ctypes.byref(n_o),
            stream)
    try:
        # one call first: the library's code and its fixed array are loaded on
        # first use, which the device-wide count below would otherwise see
        assert L.spectra_pack_plan_noalloc(*args) == _lib.OK
        before = torch.cuda.memory_allocated()
        reserved = torch.cuda.memory_reserved()
        # device-wide free bytes also see a cudaMalloc inside the library,
        # which torch's allocator counters cannot
        free = torch.cuda.mem_get_info()[0]
        st = L.spectra_pack_plan_noalloc(*args)
        assert torch.cuda.memory_allocated() == before
        assert torch.cuda.memory_reserved() == reserved
        assert torch.cuda.mem_get_info()[0] == free
    finally:
        gc.enable()
    assert st == _lib.OK, sp.spectra_status_string(st)
    return idx[: n_o.value].clone()


@pytest.mark.parametrize("with_kappa", [True, False])
def test_noalloc_matches_workspace_entry_point_on_consecutive_calls(with_kappa):
    L = _lib.load()
    specs = [wl.MatrixSpec("gate", 8960, 1536, 23), wl.SINGLE_512, wl.MatrixSpec("single", 33, 4096, 60)]
    for call, spec in enumerate(specs):
        w = wl.weight(spec, seed=call, device=DEV)
        g = wl.gain(spec, seed=call, device=DEV) if call != 2 else None
        for tau in (3.0, 6.0):
            idx_ref, kap_ref = sp.spectra_pack_plan(w, g, tau, want_kappa=True)
            kap = torch.full((spec.k,), float("nan"), dtype=torch.float64, device=DEV) if with_kappa else None
            idx = _noalloc(L, w, g, tau, kap)
            torch.cuda.synchronize()
            assert torch.equal(idx, idx_ref)
            if with_kappa:
                assert np.array_equal(kap.cpu().numpy().view(np.uint64),
                                      kap_ref.cpu().numpy().view(np.uint64))


def test_noalloc_rejects_k_above_its_scratch():
    L = _lib.load()
    n_o = ctypes.c_int32(-1)
    big = _lib.NOALLOC_MAX_K + 32
    w = torch.zeros((1, big), dtype=torch.bfloat16, device=DEV)
    idx = torch.empty(big, dtype=torch.int32, device=DEV)
    st = L.spectra_pack_plan_noalloc(w.data_ptr(), None, 1, big, 3.0, None, idx.data_ptr(),
                                     ctypes.byref(n_o), None)
    assert st == _lib.ERR_SHAPE and n_o.value == -1


def test_noalloc_reports_nonfinite_weights():
    L = _lib.load()
    w = torch.zeros((16, 64), dtype=torch.bfloat16, device=DEV)
    w[2, 3] = float("inf")
    idx = torch.empty(64, dtype=torch.int32, device=DEV)
    n_o = ctypes.c_int32(-1)
    st = L.spectra_pack_plan_noalloc(w.data_ptr(), None, 16, 64, 3.0, None, idx.data_ptr(),
                                     ctypes.byref(n_o), None)
    assert st == _lib.ERR_NONFINITE
    # the error word is cleared by the next call
    w[2, 3] = 1.0
    st = L.spectra_pack_plan_noalloc(w.data_ptr(), None, 16, 64, 3.0, None, idx.data_ptr(),
                                     ctypes.byref(n_o), None)
    assert st == _lib.OK
