"""The strictly causal variant on the GPU against the oracle (article "BMW's
16 GB GPU just did what needs an A100", section "The one real caveat: causal
leakage"; every query position routes on its own query).

Gates as for the block path: routing rows equal to the oracle's except on
rows whose oracle gap is below 1e-4; the attention stages run on the
oracle's routing and meet 2e-3 (bf16) / 1e-4 (float32) max-abs on O, lse,
dQ, dK, dV.  A property check runs on the GPU alone: changing the inputs
after position p leaves the routing at positions <= p bit for bit and the
outputs there bit for bit (float32, one warp per position) or within float
rounding (bf16 on the tensor cores, where windows of 32 positions share key
tiles: see the test).
"""
import numpy as np
import pytest
import torch

import hierarchical_routed_sparse_b200 as hga
from hierarchical_routed_sparse_b200 import workloads as W
from hierarchical_routed_sparse_b200.workloads import Workload

import oracle
from parity_util import TOL, check_causal_routing, dims_of, maxabs, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup(oracle_mod):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_routed_sparse_b200 import build
    build.build()
    hga.load()


CASES = [
    Workload("causal_gqa4_bf16", B=2, Hq=8, Hkv=2, d=128, T_hist=320, T_seg=256, k_c=3, k_g=13,
             keys="clustered", backward=True, seed=41),
    Workload("causal_fp32_d64", B=1, Hq=4, Hkv=2, d=64, T_hist=256, T_seg=192, k_c=2, k_g=9,
             dtype="fp32", keys="clustered", backward=True, seed=42),
    Workload("causal_all_routing", B=1, Hq=4, Hkv=1, d=128, T_hist=128, T_seg=192, k_c=-1, k_g=-1,
             backward=True, seed=43),
    Workload("causal_gqa8_bf16_d64", B=1, Hq=16, Hkv=2, d=64, T_hist=192, T_seg=128, k_c=2, k_g=6,
             keys="clustered", backward=True, seed=44),
    Workload("causal_no_history", B=1, Hq=2, Hkv=2, d=128, T_hist=0, T_seg=256, k_c=2, k_g=40,
             backward=True, seed=45),
    Workload("causal_fp32_d128_k1", B=1, Hq=4, Hkv=1, d=128, T_hist=192, T_seg=128, k_c=1, k_g=1,
             dtype="fp32", keys="clustered", backward=True, seed=46),
]


def _run(w, x, gidx_in=None):
    p = hga.Params.from_workload(w)
    Q, K, V, dO = (to_dev(x[k], w.dtype) for k in ("Q", "K", "V", "dO"))
    cb = hga.CausalBuffers(p)
    cb.summaries(K, 0, w.T)
    cb.route(Q)
    gidx = cb.gidx if gidx_in is None else torch.from_numpy(gidx_in).to("cuda")
    cb.forward(Q, K, V, gidx=gidx)
    cb.backward(Q, K, V, dO, gidx=gidx)
    torch.cuda.synchronize()
    assert hga.device_status() == 0
    return {k: getattr(cb, k).cpu().numpy() for k in ("cidx", "gidx", "O", "lse", "dQ", "dK", "dV")}


def _oracle(w, x):
    dims = dims_of(w)
    x64 = {k: v.astype(np.float64) for k, v in x.items()}
    csum, gsum = oracle.build_summaries(dims, x64["K"])
    r = oracle.causal_route(dims, x64["Q"], csum, gsum)
    O, lse = oracle.causal_attn_fwd(dims, x64["Q"], x64["K"], x64["V"], r["gidx"])
    dQ, dK, dV = oracle.causal_attn_bwd(dims, x64["Q"], x64["K"], x64["V"], x64["dO"], r["gidx"])
    r.update(O=O, lse=lse, dQ=dQ, dK=dK, dV=dV, csum=csum, gsum=gsum, Q64=x64["Q"])
    return r


def _compare(w, x):
    orc = _oracle(w, x)
    got = _run(w, x)
    check_causal_routing(w, got["cidx"], got["gidx"], orc["Q64"], orc["csum"], orc["gsum"], orc)
    att = _run(w, x, gidx_in=orc["gidx"])
    for k in ("O", "lse", "dQ", "dK", "dV"):
        err = maxabs(att[k], orc[k])
        assert err <= TOL[w.dtype], f"{k}: max-abs error {err:.3g}"
    return orc


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_causal_matches_oracle(w):
    _compare(w, w.full())


def test_causal_full_size_workload():
    # The 16K-context Qwen3-8B layer segment (2048 positions, 8 kv-heads):
    # every routing row and every output against the oracle.
    _compare(W.QWEN3_CTX16K_TRAIN, W.QWEN3_CTX16K_TRAIN.full())


@pytest.mark.parametrize("w", [CASES[0], CASES[1], W.QWEN3_CTX16K_TRAIN], ids=lambda w: w.name)
def test_outputs_do_not_see_later_positions(w):
    x = w.full()
    a = _run(w, x)
    p = w.T_seg // 2 + 5
    rng = np.random.default_rng(1)
    y = {k: v.copy() for k, v in x.items()}
    y["Q"][:, :, p + 1:] = rng.standard_normal(y["Q"][:, :, p + 1:].shape).astype(np.float32)
    y["K"][:, :, w.T_hist + p + 1:] = rng.standard_normal(y["K"][:, :, w.T_hist + p + 1:].shape).astype(np.float32)
    y["V"][:, :, w.T_hist + p + 1:] = rng.standard_normal(y["V"][:, :, w.T_hist + p + 1:].shape).astype(np.float32)
    if w.dtype == "bf16":
        for k in ("Q", "K", "V"):
            y[k] = W.round_bf16(y[k])
    b = _run(w, y)
    assert np.array_equal(a["cidx"][:, :, :p + 1], b["cidx"][:, :, :p + 1])
    assert np.array_equal(a["gidx"][:, :, :p + 1], b["gidx"][:, :, :p + 1])
    if w.dtype == "fp32":        # one warp per position: bit for bit
        assert np.array_equal(a["O"][:, :, :p + 1], b["O"][:, :, :p + 1])
        assert np.array_equal(a["lse"][:, :, :p + 1], b["lse"][:, :, :p + 1])
    else:
        # Tensor cores: a window of 32 positions runs over the union of their
        # routed groups, so a later position of the same window can change
        # which tile holds a key; its own keys are masked to exactly zero, but
        # the order in which a row's keys are summed may move.  Equal within
        # float rounding, far below any real change of the inputs' effect.
        assert maxabs(a["O"][:, :, :p + 1], b["O"][:, :, :p + 1]) <= 1e-5
        assert maxabs(a["lse"][:, :, :p + 1], b["lse"][:, :, :p + 1]) <= 1e-5
    assert maxabs(a["O"][:, :, p + 1:], b["O"][:, :, p + 1:]) > 1e-2


@pytest.mark.parametrize("T,k_c,k_g", [(32768, 16, 64), (131072, 16, 64), (32768, 8, 32)])
def test_causal_long_context_sampled_units(T, k_c, k_g):
    # Per-position routing over up to 511 / 2047 eligible chunks: at 32K the
    # window router (k_c 16: rounds over the scores in shared memory; k_c 8:
    # eight lanes a row past 256 candidates), at 128K the warp-per-row
    # router.  The whole problem on the GPU, two (batch, kv-head) units
    # against the oracle.
    from parity_util import unit_slice
    w = W.sweep_point(T, k_c, k_g).with_(B=1)
    x = w.full()
    got = _run(w, x)
    for g in (0, w.Hkv - 1):
        wu, xu = unit_slice(w, x, 0, g)
        orc = _oracle(wu, xu)
        hs = slice(g * w.G, (g + 1) * w.G)
        check_causal_routing(wu, got["cidx"][:, g:g + 1], got["gidx"][:, g:g + 1], orc["Q64"],
                             orc["csum"], orc["gsum"], orc)
        att = _run(wu, xu, gidx_in=orc["gidx"])
        for k in ("O", "lse", "dQ", "dK", "dV"):
            err = maxabs(att[k], orc[k])
            assert err <= TOL[w.dtype], f"{k}: {err:.3g}"
        # The whole-problem run gives the same outputs on rows whose routing matched.
        same = (got["gidx"][:, g:g + 1] == orc["gidx"]).all(axis=-1)       # [1, 1, T_seg]
        rows = np.repeat(same, w.G, axis=1)
        assert maxabs(got["O"][:, hs][rows], orc["O"][rows]) <= TOL[w.dtype]


def _window_costs(w, gidx):
    """Cost of every window item as the schedule counts it, from the index
    rows alone: 2 * (union tiles + own chunk) + segment tiles, where the union
    is that of the window's 32 rows over the groups before its own chunk."""
    n_y = (w.G + 3) // 4
    cost = []
    for b in range(w.B):
        for g in range(w.Hkv):
            for w0 in range(0, w.T_seg, 32):
                rows = gidx[b, g, w0:w0 + 32]
                limit = 8 * ((w.T_hist + w0) // 64)
                u = np.unique(rows[(rows >= 0) & (rows < limit)])
                n, c_hist = len(u), int((u < w.T_hist // 8).sum())
                n_rt = (n + 7) // 8
                n_seg = n_rt - c_hist // 8 + 1 if c_hist < n else 1
                cost += [min(2 * (n_rt + 1) + n_seg, 1023)] * n_y
    return np.array(cost, dtype=np.int64)


@pytest.mark.parametrize("w", [CASES[0], CASES[3], CASES[4], W.QWEN3_CTX16K_TRAIN], ids=lambda w: w.name)
def test_window_schedule(w):
    # The schedule orders the window items by cost, heaviest first, equal
    # costs in index order (a stable sort of the costs counted from the
    # index rows here), and changes only the order the items run in: O, lse
    # and dQ equal the unscheduled launch's bit for bit, dK / dV (float
    # atomics in another order) within float rounding.
    x = w.full()
    p = hga.Params.from_workload(w)
    Q, K, V, dO = (to_dev(x[k], w.dtype) for k in ("Q", "K", "V", "dO"))
    cb = hga.CausalBuffers(p)
    cb.summaries(K, 0, w.T)
    cb.route(Q)
    torch.cuda.synchronize()
    n = hga.causal_sched_size(p) // 8
    sched = cb.sched.cpu().numpy()
    cost = _window_costs(w, cb.gidx.cpu().numpy())
    assert len(cost) == n
    assert np.array_equal(sched[n:], cost)
    assert np.array_equal(sched[:n], np.argsort(-cost, kind="stable"))
    out = {}
    for use in (True, False):
        s = cb.sched if use else None
        hga.attn_fwd_causal(p, Q, K, V, cb.gidx, cb.O, cb.lse, sched=s)
        hga.attn_bwd_causal(p, Q, K, V, cb.O, cb.lse, dO, cb.gidx, cb.dQ, cb.dK, cb.dV, sched=s)
        torch.cuda.synchronize()
        assert hga.device_status() == 0
        out[use] = {k: getattr(cb, k).cpu().numpy() for k in ("O", "lse", "dQ", "dK", "dV")}
    for k in ("O", "lse", "dQ"):
        assert np.array_equal(out[True][k], out[False][k]), k
    for k in ("dK", "dV"):
        ref = out[False][k]
        assert maxabs(out[True][k], ref) <= 1e-5 * (1.0 + np.abs(ref).max()), k
