"""The kernels' bounded waits give up instead of hanging, report it, and leave
the context usable.

A weight-ring wait that nothing can satisfy is launched on purpose
(spectra_selftest_wait): no fault, no trap, no endless loop -- the wait runs
out after its one-second limit and raises the flag that
spectra_device_status reports as SPECTRA_ERR_INTERNAL.
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


def _matvec_still_correct():
    spec = wl.SINGLE_512
    w, g, x = draw(spec)
    lay = sp.pack_layer(w, g, 3.0)
    y = sp.spectra_gemv(lay, x[0])
    torch.cuda.synchronize()
    wb = wl.bits(w)
    ref = oracle.pack(wb, np_gain(g), 3.0)
    y_ref, bound = oracle.gemm(ref.can, wb, ref.idx, wl.bits(x))
    check_gemv(y, y_ref[0], bound[0])


def test_ring_wait_runs_out_and_reports_internal():
    sp.spectra_device_status()  # start from a clear flag
    t0 = time.perf_counter()
    sp.spectra_selftest_wait(0)
    torch.cuda.synchronize()
    waited = time.perf_counter() - t0
    # the limit is one second of %globaltimer time
    assert 0.9 < waited < 30.0, waited
    with pytest.raises(sp.SpectraError) as e:
        sp.spectra_device_status()
    assert e.value.status == _lib.ERR_INTERNAL
    # read once, the flag is clear again, and the context still computes
    sp.spectra_device_status()
    _matvec_still_correct()
    sp.spectra_device_status()
