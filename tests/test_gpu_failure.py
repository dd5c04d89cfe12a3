"""Failure detection on the GPU without a GPU fault.

Every mbarrier wait of the library's tensor-core and decode kernels is
bounded in time; a wait that runs out records its code in a device status
word, the kernel frees its tensor memory and returns, and the host reads the
word with hga_device_status.  hga_selftest_wait runs that path on purpose:
its kernel waits (1 ms here) on an mbarrier that nothing arrives at.  The
test checks that the status word names the wait, that clearing resets it,
and that the device is still usable: a small forward and backward run
afterwards match the oracle.
"""
import numpy as np
import pytest
import torch

import hierarchical_routed_sparse_b200 as hga
from hierarchical_routed_sparse_b200.workloads import Workload

from parity_util import compare_all, f64, run_gpu, run_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup(oracle_mod):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_routed_sparse_b200 import build
    build.build()
    hga.load()


def test_bounded_wait_runs_out_and_is_reported():
    assert hga.device_status(clear=True) == 0
    site = hga.selftest_wait(1000)
    torch.cuda.synchronize()
    assert site != 0
    assert hga.device_status() == site            # recorded, not yet cleared
    assert hga.device_status(clear=True) == site  # read and cleared
    assert hga.device_status() == 0


def test_device_usable_after_a_wait_ran_out():
    hga.selftest_wait(200)
    torch.cuda.synchronize()
    hga.device_status(clear=True)
    w = Workload("after_timeout", B=1, Hq=4, Hkv=2, d=128, T_hist=256, T_seg=256, k_c=2, k_g=7,
                 keys="clustered", backward=True, seed=31)
    x = w.full()
    orc = run_oracle(w, f64(x), backward=True)
    gpu, _ = run_gpu(w, x, gidx_in=orc["gidx"])
    compare_all(w, gpu, orc)
    assert np.isfinite(gpu["dQ"]).all()


def test_selftest_rejects_bad_limits():
    for bad in (0, -5, 2_000_000):
        with pytest.raises(hga.HGAError) as ei:
            hga.selftest_wait(bad)
        assert ei.value.code == hga.HGA_ERR_INVALID_ARG
