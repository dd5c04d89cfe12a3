"""The bounds-checked build (libhga_checked.so, -DHGA_CHECK_BOUNDS) on the GPU.

That build checks on the device every routed group or chunk index it reads
from a caller's index row before using it as an address (valid: before the
row's own chunk).  An index outside records a site code, is replaced by an
in-bounds index (so no access leaves the tensors) and the call returns
HGA_ERR_DEVICE_CHECK.  Checked here:
  * on valid inputs the checked build returns HGA_OK, reports no failed
    check and gives the release build's results (and the oracle's);
  * one planted out-of-range entry in an index row makes the forward, the
    backward, the float32 path, the strictly causal forward and the group
    router report HGA_ERR_DEVICE_CHECK without a fault, and the device is
    usable afterwards; so does an out-of-range entry of a causal window
    schedule in the causal forward and backward.
The release build never sees a planted index.
"""
import numpy as np
import pytest
import torch

import hierarchical_routed_sparse_b200 as hga
from hierarchical_routed_sparse_b200.workloads import Workload

from parity_util import compare_all, f64, maxabs, run_gpu, run_oracle, to_dev

pytestmark = pytest.mark.gpu

W_BF16 = Workload("checked_bf16", B=1, Hq=4, Hkv=2, d=128, T_hist=256, T_seg=256, k_c=2, k_g=7,
                  keys="clustered", backward=True, seed=61)
W_FP32 = Workload("checked_fp32_d64", B=1, Hq=2, Hkv=1, d=64, T_hist=128, T_seg=192, k_c=2, k_g=5,
                  dtype="fp32", keys="clustered", backward=True, seed=62)


@pytest.fixture(scope="module", autouse=True)
def _checked_library(oracle_mod):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_routed_sparse_b200 import build
    build.build()
    build.build(checked=True)
    hga.use_library(hga.CHECKED_LIB_PATH)
    assert hga.checked_build()
    yield
    hga.use_library(build.LIB)
    assert not hga.checked_build()


@pytest.mark.parametrize("w", [W_BF16, W_FP32], ids=lambda w: w.name)
def test_valid_inputs_pass_the_checks(w):
    x = w.full()
    orc = run_oracle(w, f64(x), backward=True)
    gpu, _ = run_gpu(w, x, gidx_in=orc["gidx"])
    assert hga.device_check() == 0
    compare_all(w, gpu, orc)


def _planted(w, orc, value):
    """The oracle's routing with one entry of one row replaced."""
    g = orc["gidx"].copy()
    g[0, w.Hkv - 1, w.T_seg // 64 - 1, 0] = value
    return g


def _expect_check(fn):
    with pytest.raises(hga.HGAError) as ei:
        fn()
    assert ei.value.code == hga.HGA_ERR_DEVICE_CHECK, str(ei.value)
    assert "bounds check" in str(ei.value)
    assert hga.device_check() == 0            # reported and cleared by the call


@pytest.mark.parametrize("w", [W_BF16, W_FP32], ids=lambda w: w.name)
@pytest.mark.parametrize("where", ["beyond_context", "own_chunk", "negative_in_prefix"])
def test_planted_index_is_reported(w, where):
    x = w.full()
    orc = run_oracle(w, f64(x), backward=True)
    nQB = w.T_seg // 64
    c0 = w.T_hist // 64 + nQB - 1                      # own chunk of the planted row
    value = {"beyond_context": w.T // 8 + 3, "own_chunk": 8 * c0 + 1, "negative_in_prefix": -1}[where]
    gidx = torch.from_numpy(_planted(w, orc, value)).to("cuda")
    p = hga.Params.from_workload(w)
    buf = hga.Buffers(p)
    Q, K, V, dO = (to_dev(x[k], w.dtype) for k in ("Q", "K", "V", "dO"))
    _expect_check(lambda: buf.forward(Q, K, V, gidx=gidx))
    _expect_check(lambda: buf.backward(Q, K, V, dO, gidx=gidx))
    # The device is usable: the same call on the valid routing passes.
    good = torch.from_numpy(orc["gidx"]).to("cuda")
    buf.forward(Q, K, V, gidx=good)
    torch.cuda.synchronize()
    assert maxabs(buf.O.cpu().numpy(), orc["O"]) <= (2e-3 if w.dtype == "bf16" else 1e-4)


def test_planted_chunk_in_group_routing_is_reported():
    w = W_BF16
    x = w.full()
    orc = run_oracle(w, f64(x), backward=False)
    p = hga.Params.from_workload(w)
    buf = hga.Buffers(p)
    buf.summaries(to_dev(x["K"], w.dtype), 0, w.T)
    buf.route(to_dev(x["Q"], w.dtype))
    cidx = buf.cidx.clone()
    cidx[0, 0, 2, 0] = w.T_hist // 64 + 2              # block 2's own chunk: not eligible
    _expect_check(lambda: hga.route_groups(p, buf.qbar, buf.gsum, cidx, buf.gidx))
    hga.route_groups(p, buf.qbar, buf.gsum, buf.cidx, buf.gidx)
    torch.cuda.synchronize()


def test_planted_index_in_causal_rows_is_reported():
    w = W_BF16
    x = w.full()
    p = hga.Params.from_workload(w)
    cb = hga.CausalBuffers(p)
    Q, K, V = (to_dev(x[k], w.dtype) for k in ("Q", "K", "V"))
    cb.summaries(K, 0, w.T)
    cb.route(Q)
    bad = cb.gidx.clone()
    bad[0, 1, w.T_seg - 1, 0] = w.T // 8 + 9
    _expect_check(lambda: cb.forward(Q, K, V, gidx=bad))
    cb.forward(Q, K, V)
    torch.cuda.synchronize()
    assert torch.isfinite(cb.O).all()


def test_planted_schedule_entry_is_reported():
    # A window schedule entry outside the grid: every build runs the CTA's
    # own item instead (no item index leaves the grid's range); the checked
    # build also reports it.
    w = W_BF16
    x = w.full()
    p = hga.Params.from_workload(w)
    cb = hga.CausalBuffers(p)
    Q, K, V, dO = (to_dev(x[k], w.dtype) for k in ("Q", "K", "V", "dO"))
    cb.summaries(K, 0, w.T)
    cb.route(Q)
    n = hga.causal_sched_size(p) // 8
    for entry in (n + 5, -1):
        sched = cb.sched.clone()
        sched[1] = entry
        _expect_check(lambda: hga.attn_fwd_causal(p, Q, K, V, cb.gidx, cb.O, cb.lse, sched=sched))
        _expect_check(lambda: hga.attn_bwd_causal(p, Q, K, V, cb.O, cb.lse, dO, cb.gidx, cb.dQ, cb.dK, cb.dV,
                                                  sched=sched))
    cb.forward(Q, K, V)
    cb.backward(Q, K, V, dO)
    torch.cuda.synchronize()
    assert hga.device_check() == 0
    assert torch.isfinite(cb.O).all() and torch.isfinite(cb.dQ).all()
