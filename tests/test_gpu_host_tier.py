"""Host-RAM KV tier on the GPU: history K/V in pinned host memory, routed
groups staged in device memory (hga_stage_routed), attention on the staged
problem (article "BMW's 16 GB GPU just did what needs an A100", section
"How it fits in 16 GB": older KV in host RAM, only the selected groups'
exact tokens brought to the GPU after routing).

The staged attention must compute what the full problem computes: O, lse
and dQ bit for bit (same tiles in the same order), dK / dV up to the order
of their float32 atomics; and, with the oracle's routing fed in, it must
meet the oracle gates directly.
"""
import numpy as np
import pytest
import torch

import hierarchical_routed_sparse_b200 as hga
from hierarchical_routed_sparse_b200 import workloads as W
from hierarchical_routed_sparse_b200.workloads import Workload

from parity_util import TOL, f64, maxabs, run_oracle, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup(oracle_mod):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_routed_sparse_b200 import build
    build.build()
    hga.load()


CASES = [
    Workload("tier_gqa4_bf16_ragged", B=2, Hq=8, Hkv=2, d=128, T_hist=512, T_seg=512, k_c=3, k_g=13,
             keys="clustered", backward=True, seed=21),
    Workload("tier_fp32_d64", B=1, Hq=4, Hkv=2, d=64, T_hist=256, T_seg=384, k_c=2, k_g=11,
             dtype="fp32", keys="clustered", backward=True, seed=22),
    Workload("tier_all_routing", B=1, Hq=4, Hkv=1, d=128, T_hist=192, T_seg=256, k_c=-1, k_g=-1,
             backward=True, seed=23),
    Workload("tier_no_history", B=1, Hq=2, Hkv=2, d=128, T_hist=0, T_seg=256, k_c=2, k_g=5,
             backward=True, seed=24),
]


def _split(x, w, on_host: bool):
    """History rows (pinned host or device) and segment rows (device)."""
    K, V = x["K"], x["V"]
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    kh = torch.from_numpy(np.ascontiguousarray(K[:, :, :w.T_hist])).to(dt)
    vh = torch.from_numpy(np.ascontiguousarray(V[:, :, :w.T_hist])).to(dt)
    if on_host:
        kh, vh = kh.pin_memory(), vh.pin_memory()
    else:
        kh, vh = kh.cuda(), vh.cuda()
    ks = to_dev(np.ascontiguousarray(K[:, :, w.T_hist:]), w.dtype)
    vs = to_dev(np.ascontiguousarray(V[:, :, w.T_hist:]), w.dtype)
    return kh, vh, ks, vs


def _attention(p, Q, K, V, gidx, dO):
    B, Hq, Hkv, Ts, d = p.B, p.Hq, p.Hkv, p.T_seg, p.d
    f32 = dict(device="cuda", dtype=torch.float32)
    O = torch.empty(B, Hq, Ts, d, **f32)
    lse = torch.empty(B, Hq, Ts, **f32)
    dQ = torch.empty(B, Hq, Ts, d, **f32)
    dK = torch.empty(B, Hkv, Ts, d, **f32)
    dV = torch.empty(B, Hkv, Ts, d, **f32)
    ws = torch.empty(max(1, hga.workspace_size(p) // 4), **f32)
    hga.attn_fwd(p, Q, K, V, gidx, O, lse)
    hga.attn_bwd(p, Q, K, V, O, lse, dO, gidx, dQ, dK, dV, ws)
    return dict(O=O, lse=lse, dQ=dQ, dK=dK, dV=dV)


def _check_stage_rows(w, gidx: np.ndarray, staged: np.ndarray, T_stage: int):
    # A history group becomes its rank among the distinct routed history
    # groups of its (batch, kv-head); a segment group moves past the staged
    # history; padding stays -1.
    fsg = w.T_hist // 8
    want = np.full_like(gidx, -1)
    for b in range(gidx.shape[0]):
        for g in range(gidx.shape[1]):
            row = gidx[b, g]
            hist = np.unique(row[(row >= 0) & (row < fsg)])
            assert 8 * len(hist) <= T_stage
            want[b, g] = np.where(row < 0, -1, np.where(row < fsg, np.searchsorted(hist, row), T_stage // 8 + row - fsg))
    assert np.array_equal(staged, want)


@pytest.mark.parametrize("on_host", [True, False], ids=["host_history", "device_history"])
@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_staged_equals_full_and_oracle(w, on_host):
    x = w.full()
    p = hga.Params.from_workload(w)
    Q, K, V, dO = (to_dev(x[k], w.dtype) for k in ("Q", "K", "V", "dO"))
    buf = hga.Buffers(p)
    buf.summaries(K, 0, w.T)
    buf.route(Q)
    full = _attention(p, Q, K, V, buf.gidx, dO)
    kh, vh, ks, vs = _split(x, w, on_host)
    st = hga.StagedKV(p)
    st.stage(kh, vh, ks, vs, buf.gidx)
    staged = _attention(st.ps, Q, st.K, st.V, st.gidx, dO)
    torch.cuda.synchronize()
    assert hga.device_status() == 0
    _check_stage_rows(w, buf.gidx.cpu().numpy(), st.gidx.cpu().numpy(), st.ps.T_hist)
    for k in ("O", "lse", "dQ"):
        assert torch.equal(full[k], staged[k]), k
    for k in ("dK", "dV"):
        assert maxabs(full[k].cpu(), staged[k].cpu()) <= 1e-5, k

    # Directly against the oracle, with the oracle's routing staged.
    orc = run_oracle(w, f64(x), backward=True)
    st.stage(kh, vh, ks, vs, torch.from_numpy(orc["gidx"]).to("cuda"))
    got = _attention(st.ps, Q, st.K, st.V, st.gidx, dO)
    torch.cuda.synchronize()
    for k in ("O", "lse", "dQ", "dK", "dV"):
        err = maxabs(got[k].cpu(), orc[k])
        assert err <= TOL[w.dtype], f"{k}: {err:.3g}"


def test_staged_full_size_workload():
    w = W.QWEN3_CTX16K_TRAIN
    x = w.full()
    p = hga.Params.from_workload(w)
    Q, K, V, dO = (to_dev(x[k], w.dtype) for k in ("Q", "K", "V", "dO"))
    buf = hga.Buffers(p)
    buf.summaries(K, 0, w.T)
    buf.route(Q)
    full = _attention(p, Q, K, V, buf.gidx, dO)
    kh, vh, ks, vs = _split(x, w, on_host=True)
    st = hga.StagedKV(p)
    st.stage(kh, vh, ks, vs, buf.gidx)
    staged = _attention(st.ps, Q, st.K, st.V, st.gidx, dO)
    torch.cuda.synchronize()
    assert hga.device_status() == 0
    _check_stage_rows(w, buf.gidx.cpu().numpy(), st.gidx.cpu().numpy(), st.ps.T_hist)
    for k in ("O", "lse", "dQ"):
        assert torch.equal(full[k], staged[k]), k
    for k in ("dK", "dV"):
        assert maxabs(full[k].cpu(), staged[k].cpu()) <= 1e-5, k


def test_pageable_history_is_refused():
    w = CASES[0]
    x = w.full()
    p = hga.Params.from_workload(w)
    kh = torch.from_numpy(np.ascontiguousarray(x["K"][:, :, :w.T_hist])).to(torch.bfloat16)
    vh = torch.from_numpy(np.ascontiguousarray(x["V"][:, :, :w.T_hist])).to(torch.bfloat16)
    ks = to_dev(np.ascontiguousarray(x["K"][:, :, w.T_hist:]), w.dtype)
    vs = to_dev(np.ascontiguousarray(x["V"][:, :, w.T_hist:]), w.dtype)
    st = hga.StagedKV(p)
    gidx = torch.full(st.gidx.shape, -1, dtype=torch.int32, device="cuda")
    # The binding refuses unpinned host tensors before the call...
    with pytest.raises(ValueError):
        st.stage(kh, vh, ks, vs, gidx)
    # ...and the library refuses pageable host memory given as a raw pointer.
    import ctypes
    lib = hga.load()
    code = lib.hga_stage_routed(ctypes.byref(p.c()), ctypes.c_void_p(kh.data_ptr()),
                                ctypes.c_void_p(vh.data_ptr()), ctypes.c_void_p(ks.data_ptr()),
                                ctypes.c_void_p(vs.data_ptr()), ctypes.c_void_p(gidx.data_ptr()),
                                ctypes.c_void_p(st.K.data_ptr()), ctypes.c_void_p(st.V.data_ptr()),
                                ctypes.c_void_p(st.gidx.data_ptr()), None)
    assert code == hga.HGA_ERR_INVALID_ARG
    assert b"host memory" in lib.hga_last_error()


@pytest.mark.parametrize("w", CASES[:2], ids=lambda w: w.name)
def test_summaries_from_the_rows_alone(w):
    # hga_build_summaries_rows on a K holding only rows [t0, t1) writes the
    # same csum / gsum rows, bit for bit, as hga_build_summaries on the full K.
    x = w.full()
    p = hga.Params.from_workload(w)
    K = to_dev(x["K"], w.dtype)
    a, b = hga.Buffers(p), hga.Buffers(p)
    a.summaries(K, 0, w.T)
    t0 = w.T_hist
    b.summaries(K, 0, t0)
    hga.build_summaries_rows(p, to_dev(np.ascontiguousarray(x["K"][:, :, t0:]), w.dtype), t0, w.T,
                             b.csum, b.gsum)
    torch.cuda.synchronize()
    assert torch.equal(a.csum, b.csum) and torch.equal(a.gsum, b.gsum)
