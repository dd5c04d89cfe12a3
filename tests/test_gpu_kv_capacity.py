"""K / V (and summary) buffers with spare rows (hga_params.kv_capacity).

A caller that keeps a KV cache growing segment by segment hands the library
buffers of `kv_capacity` rows per (batch, kv-head) with only the first
T_hist + T_seg in use.  Every call must then give exactly what it gives on
dense buffers of T rows: the same kernels on the same values, only the row
stride differs.  The spare rows hold NaN, so a read of any of them would
show.  Covered: summaries, fused routing, forward and backward (bf16 d 128
on the tensor cores, float32 d 64 on the FMA path), the strictly causal
variant and a decode step.
"""
import numpy as np
import pytest
import torch

import hierarchical_routed_sparse_b200 as hga
from hierarchical_routed_sparse_b200.workloads import Workload

from parity_util import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_routed_sparse_b200 import build
    build.build()
    hga.load()


CASES = [
    Workload("cap_bf16", B=2, Hq=8, Hkv=2, d=128, T_hist=320, T_seg=256, k_c=3, k_g=11, keys="clustered",
             backward=True, seed=71),
    Workload("cap_fp32_d64", B=1, Hq=4, Hkv=2, d=64, T_hist=192, T_seg=192, k_c=2, k_g=7, dtype="fp32",
             keys="clustered", backward=True, seed=72),
]


def _padded(t, cap):
    """[B][H][T][d] -> [B][H][cap][d] with NaN in rows T.."""
    out = torch.full(t.shape[:2] + (cap,) + t.shape[3:], float("nan"), device=t.device, dtype=t.dtype)
    out[:, :, :t.shape[2]] = t
    return out


def _run(p, Q, K, V, dO, csum, gsum):
    wc, wg = hga.route_widths(p)
    Bn, Hq, Hkv, d, Ts, nQB = p.B, p.Hq, p.Hkv, p.d, p.T_seg, p.nQB
    f32 = dict(device="cuda", dtype=torch.float32)
    o = dict(qbar=torch.empty(Bn, Hkv, nQB, d, **f32),
             cidx=torch.empty(Bn, Hkv, nQB, wc, device="cuda", dtype=torch.int32),
             gidx=torch.empty(Bn, Hkv, nQB, wg, device="cuda", dtype=torch.int32),
             O=torch.empty(Bn, Hq, Ts, d, **f32), lse=torch.empty(Bn, Hq, Ts, **f32),
             dQ=torch.empty(Bn, Hq, Ts, d, **f32), dK=torch.empty(Bn, Hkv, Ts, d, **f32),
             dV=torch.empty(Bn, Hkv, Ts, d, **f32))
    ws = torch.empty(max(1, hga.workspace_size(p) // 4), **f32)
    hga.build_summaries(p, K, 0, p.T, csum, gsum)
    hga.route(p, Q, csum, gsum, o["qbar"], o["cidx"], o["gidx"])
    hga.attn_fwd(p, Q, K, V, o["gidx"], o["O"], o["lse"])
    hga.attn_bwd(p, Q, K, V, o["O"], o["lse"], dO, o["gidx"], o["dQ"], o["dK"], o["dV"], ws)
    torch.cuda.synchronize()
    assert hga.device_status() == 0
    return o


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_block_path_with_spare_rows_equals_dense(w):
    x = w.full()
    Q, K, V, dO = (to_dev(x[k], w.dtype) for k in ("Q", "K", "V", "dO"))
    p = hga.Params.from_workload(w)
    cap = w.T + 192
    pc = hga.Params.from_workload(w)
    pc.kv_capacity = cap
    f32 = dict(device="cuda", dtype=torch.float32)
    dense = _run(p, Q, K, V, dO, torch.zeros(w.B, w.Hkv, w.T // 64, w.d, **f32),
                 torch.zeros(w.B, w.Hkv, w.T // 8, w.d, **f32))
    spare = _run(pc, Q, _padded(K, cap), _padded(V, cap), dO,
                 torch.full((w.B, w.Hkv, cap // 64, w.d), float("nan"), **f32),
                 torch.full((w.B, w.Hkv, cap // 8, w.d), float("nan"), **f32))
    for k in ("qbar", "cidx", "gidx", "O", "lse", "dQ"):
        assert torch.equal(dense[k], spare[k]), k
    for k in ("dK", "dV"):        # float atomics: the order of the additions may differ
        assert float((dense[k] - spare[k]).abs().max()) <= 1e-5, k


def test_causal_and_decode_with_spare_rows_equal_dense():
    w = CASES[0]
    x = w.full()
    Q, K, V, dO = (to_dev(x[k], w.dtype) for k in ("Q", "K", "V", "dO"))
    cap = w.T + 128
    p = hga.Params.from_workload(w)
    pc = hga.Params.from_workload(w)
    pc.kv_capacity = cap
    a, b = hga.CausalBuffers(p), hga.CausalBuffers(pc)
    b.csum.fill_(float("nan"))
    b.gsum.fill_(float("nan"))
    Kc, Vc = _padded(K, cap), _padded(V, cap)
    a.summaries(K, 0, w.T)
    b.summaries(Kc, 0, w.T)
    a.route(Q)
    b.route(Q)
    a.forward(Q, K, V)
    b.forward(Q, Kc, Vc)
    a.backward(Q, K, V, dO)
    b.backward(Q, Kc, Vc, dO)
    torch.cuda.synchronize()
    for k in ("cidx", "gidx", "O", "lse", "dQ"):
        assert torch.equal(getattr(a, k), getattr(b, k)), k
    for k in ("dK", "dV"):
        assert float((getattr(a, k) - getattr(b, k)).abs().max()) <= 1e-5, k
    # A decode step at the last position of the context.
    pos = w.T - 1
    q = Q[:, :, -1].contiguous()
    outs = []
    for pp, KK, VV, cs, gs in ((p, K, V, a.csum, a.gsum), (pc, Kc, Vc, b.csum, b.gsum)):
        O = torch.empty(w.B, w.Hq, w.d, device="cuda")
        lse = torch.empty(w.B, w.Hq, device="cuda")
        wc, wg = hga.route_widths(pp)
        ci = torch.empty(w.B, w.Hkv, wc, device="cuda", dtype=torch.int32)
        gi = torch.empty(w.B, w.Hkv, wg, device="cuda", dtype=torch.int32)
        hga.decode(pp, pos, q, KK, VV, cs, gs, O, lse, ci, gi)
        outs.append((O, lse, ci, gi))
    torch.cuda.synchronize()
    assert hga.device_status() == 0
    for u, v in zip(*outs):
        assert torch.equal(u, v)
