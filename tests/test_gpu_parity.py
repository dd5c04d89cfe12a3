"""GPU parity of every hot-path stage against the CPU oracle, through the C ABI.

Small cases span several key tiles and ragged tails (group counts that are
not multiples of 8, partial summary ranges, GQA ratios 1/2/4, d 64 and 128,
bf16 and float32, empty history, "all" routing, k above the eligible count).
The named workloads run at their full sizes; the scale-sweep points, too
large for the oracle, are checked on sampled (batch, kv-head) units, which
are independent problems.
"""
import numpy as np
import pytest
import torch

import hierarchical_routed_sparse_b200 as hga
from hierarchical_routed_sparse_b200 import workloads as W
from hierarchical_routed_sparse_b200.workloads import Workload

from parity_util import (check_block_routing, compare_all, f64, maxabs, run_gpu, run_oracle,
                         to_dev, unit_slice, TOL)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup(oracle_mod):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_routed_sparse_b200 import build
    build.build()
    hga.load()


SMALL = [
    Workload("gqa4_bf16_ragged", B=2, Hq=8, Hkv=2, d=128, T_hist=512, T_seg=512, k_c=3, k_g=13,
             keys="clustered", backward=True, seed=1),
    Workload("gqa2_fp32_d64", B=1, Hq=4, Hkv=2, d=64, T_hist=256, T_seg=384, k_c=2, k_g=11,
             dtype="fp32", keys="clustered", backward=True, seed=2),
    Workload("mha_bf16_nohist", B=1, Hq=2, Hkv=2, d=128, T_hist=0, T_seg=512, k_c=2, k_g=5,
             backward=True, seed=3),
    Workload("all_routing_bf16", B=1, Hq=4, Hkv=1, d=128, T_hist=192, T_seg=256, k_c=-1, k_g=-1,
             backward=True, seed=4),
    Workload("all_routing_fp32_d64", B=1, Hq=2, Hkv=1, d=64, T_hist=128, T_seg=256, k_c=-1,
             k_g=-1, dtype="fp32", backward=True, seed=5),
    Workload("k_above_eligible", B=1, Hq=4, Hkv=2, d=128, T_hist=128, T_seg=256, k_c=50,
             k_g=1000, keys="clustered", backward=True, seed=6),
    Workload("groups_all_of_chunks", B=1, Hq=4, Hkv=2, d=64, T_hist=512, T_seg=128, k_c=3,
             k_g=-1, backward=True, seed=7),
    Workload("single_block", B=3, Hq=3, Hkv=1, d=64, T_hist=0, T_seg=64, k_c=4, k_g=16,
             backward=True, seed=8),
    Workload("k1_bf16_long_hist", B=1, Hq=4, Hkv=1, d=128, T_hist=2048, T_seg=192, k_c=1, k_g=1,
             keys="clustered", backward=True, seed=9),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
def test_small_cases(w):
    x = w.full()
    orc = run_oracle(w, f64(x), backward=w.backward)
    gpu, _ = run_gpu(w, x, gidx_in=orc["gidx"], full_summaries=False)
    errs = compare_all(w, gpu, orc)
    print(w.name, errs)


def test_summary_partial_range_leaves_other_rows():
    w = Workload("t", B=2, Hq=2, Hkv=2, d=128, T_hist=256, T_seg=256, k_c=2, k_g=4)
    x = w.full()
    p = hga.Params.from_workload(w)
    K = to_dev(x["K"], "bf16")
    csum = torch.full((2, 2, w.T // 64, 128), 7.0, device="cuda")
    gsum = torch.full((2, 2, w.T // 8, 128), 7.0, device="cuda")
    hga.build_summaries(p, K, 128, 320, csum, gsum)
    torch.cuda.synchronize()
    c, g = csum.cpu().numpy(), gsum.cpu().numpy()
    assert (c[:, :, :2] == 7).all() and (c[:, :, 5:] == 7).all()
    assert (g[:, :, :16] == 7).all() and (g[:, :, 40:] == 7).all()
    ref_c = x["K"].astype(np.float64).reshape(2, 2, -1, 64, 128).mean(axis=3)
    assert maxabs(c[:, :, 2:5], ref_c[:, :, 2:5]) < 1e-5


def test_exact_ties_lowest_index_on_gpu():
    # Every history chunk repeats the same keys: all chunk scores tie bit for
    # bit on the GPU too, so the lowest indices must win.
    rng = np.random.default_rng(0)
    base = rng.standard_normal((64, 128)).astype(np.float32)
    K = np.concatenate([np.tile(base, (6, 1)), rng.standard_normal((64, 128)).astype(np.float32)])
    K = W.round_bf16(K)[None, None]
    Q = W.round_bf16(rng.standard_normal((1, 1, 64, 128)).astype(np.float32))
    w = Workload("t", B=1, Hq=1, Hkv=1, d=128, T_hist=384, T_seg=64, k_c=3, k_g=4)
    p = hga.Params.from_workload(w)
    buf = hga.Buffers(p)
    buf.summaries(to_dev(K, "bf16"), 0, w.T)
    buf.route(to_dev(Q, "bf16"))
    torch.cuda.synchronize()
    assert buf.cidx.cpu().tolist() == [[[[0, 1, 2]]]]
    g = buf.gidx.cpu().numpy()[0, 0, 0]
    offs = g % 8
    # the best offset appears in chunks 0, 1, 2; the fourth slot is chunk 0's
    assert sorted(g // 8).count(0) == 2 and len(set(offs)) == 2


def test_empty_segment_launches_nothing():
    p = hga.Params(B=1, Hq=4, Hkv=1, d=128, T_hist=128, T_seg=0, k_c=2, k_g=4)
    z = torch.zeros(16, device="cuda")
    hga.attn_fwd(p, z, z, z, z.int(), z, z)        # T_seg = 0: a valid no-op
    torch.cuda.synchronize()


# ---- named workloads at full size ------------------------------------------
FULL = [W.TINY_FP32, W.TINY_FP32.with_(name="tiny_fp32_all", k_c=-1, k_g=-1),
        W.QWEN3_T2K_FWD, W.QWEN3_CTX16K_FWD, W.QWEN3_CTX16K_TRAIN]


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name)
def test_full_size_workloads(w):
    x = w.full()
    orc = run_oracle(w, f64(x), backward=w.backward)
    gpu, _ = run_gpu(w, x, gidx_in=orc["gidx"], full_summaries=False)
    errs = compare_all(w, gpu, orc)
    print(w.name, errs)


def test_tiny_fp32_all_routing_equals_dense_on_gpu():
    """k = all reduces to dense causal attention (1e-5 in float32)."""
    w = W.TINY_FP32.with_(k_c=-1, k_g=-1)
    x = w.full()
    gpu, _ = run_gpu(w, x)
    q = torch.from_numpy(x["Q"]).double()
    k = torch.from_numpy(x["K"]).double()
    v = torch.from_numpy(x["V"]).double()
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True)
    assert maxabs(gpu["O"], ref.numpy()) < 1e-5


def test_gpu_routing_end_to_end_matches_oracle_attention():
    """The GPU's own routing feeding its own attention, on rows where the
    routing agrees with the oracle's, gives the oracle's output."""
    w = W.QWEN3_CTX16K_TRAIN
    x = w.full()
    orc = run_oracle(w, f64(x), backward=False)
    gpu, _ = run_gpu(w, x)
    same = (gpu["gidx"] == orc["gidx"]).all(axis=-1)          # [B, Hkv, nQB]
    assert same.mean() > 0.95
    G = w.G
    mask = np.repeat(same, G, axis=1)                          # [B, Hq, nQB]
    mask = np.repeat(mask, 64, axis=2)                         # [B, Hq, T_seg]
    assert maxabs(gpu["O"][mask], orc["O"][mask]) <= TOL["bf16"]


# ---- scale sweep: sampled units ------------------------------------------------
SWEEP_CASES = [W.sweep_point(32768, 16, 64), W.sweep_point(131072, 8, 32)]


@pytest.mark.parametrize("w", SWEEP_CASES, ids=lambda w: w.name)
def test_sweep_sampled_units(w):
    x = w.full()
    p = hga.Params.from_workload(w)
    buf = hga.Buffers(p)
    Q, K, V, dO = (to_dev(x[k], "bf16") for k in ("Q", "K", "V", "dO"))
    buf.summaries(K, 0, w.T_hist)               # summaries kept from earlier segments
    buf.step(Q, K, V, dO)                       # the GPU's own routing end to end
    torch.cuda.synchronize()
    for (b, g) in [(0, 0), (w.B - 1, w.Hkv - 1)]:
        wu, xu = unit_slice(w, x, b, g)
        orc = run_oracle(wu, f64(xu), backward=True)
        G = w.G
        got_c = buf.cidx[b:b + 1, g:g + 1].cpu().numpy()
        got_g = buf.gidx[b:b + 1, g:g + 1].cpu().numpy()
        check_block_routing(wu, got_c, got_g, orc)
        # Attention with the oracle's routing, on this unit only.
        pu = hga.Params.from_workload(wu)
        bu = hga.Buffers(pu)
        Qu, Ku, Vu, dOu = (to_dev(xu[k], "bf16") for k in ("Q", "K", "V", "dO"))
        gi = torch.from_numpy(orc["gidx"]).to("cuda")
        bu.forward(Qu, Ku, Vu, gidx=gi)
        bu.backward(Qu, Ku, Vu, dOu, gidx=gi)
        torch.cuda.synchronize()
        for k, t in (("O", bu.O), ("lse", bu.lse), ("dQ", bu.dQ), ("dK", bu.dK), ("dV", bu.dV)):
            assert maxabs(t.cpu().numpy(), orc[k]) <= TOL["bf16"], (w.name, b, g, k)
        # The whole-problem launch gives the same attention for this unit
        # wherever its routing matched.
        if (got_g == orc["gidx"]).all():
            assert maxabs(buf.O[b:b + 1, g * G:(g + 1) * G].cpu().numpy(), orc["O"]) <= TOL["bf16"]


@pytest.mark.parametrize("w", [SMALL[0], SMALL[3], W.QWEN3_CTX16K_FWD], ids=lambda w: w.name)
def test_fused_router_equals_separate_calls(w):
    """hga_route gives bit for bit the outputs of hga_route_chunks followed by
    hga_route_groups."""
    x = w.full()
    p = hga.Params.from_workload(w)
    Q, K = to_dev(x["Q"], w.dtype), to_dev(x["K"], w.dtype)
    a, b = hga.Buffers(p), hga.Buffers(p)
    a.summaries(K, 0, w.T)
    b.summaries(K, 0, w.T)
    a.route(Q, fused=True)
    b.route(Q, fused=False)
    torch.cuda.synchronize()
    assert torch.equal(a.qbar, b.qbar)
    assert torch.equal(a.cidx, b.cidx)
    assert torch.equal(a.gidx, b.gidx)


# ---- whole-problem launches whose backward deals items round-robin --------------
# The persistent backward ranks items by cost only when a CTA takes at most 4
# of them; beyond that it deals them round-robin, and beyond 64 items a CTA
# it reads its items from global memory instead of its prologue table.  The
# gradients of those very launches are checked here on sampled (batch,
# kv-head) units against the oracle's backward fed the launch's own routing
# (once that routing has passed the index gate).
ROUND_ROBIN = [
    W.sweep_point(32768, 16, 64),                                         # 2048 items, 14 a CTA
    Workload("bwd_items_beyond_table", B=10, Hq=32, Hkv=8, d=128, T_hist=0, T_seg=4096, k_c=8,
             k_g=32, keys="clustered", backward=True, seed=51),           # 10240 items, 70 a CTA
]


@pytest.mark.parametrize("w", ROUND_ROBIN, ids=lambda w: w.name)
def test_round_robin_backward_whole_launch(w):
    import oracle
    from parity_util import dims_of
    n_items = w.B * w.Hkv * (w.T_seg // 64) * ((w.G + 1) // 2)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert n_items > 4 * sms
    x = w.full()
    p = hga.Params.from_workload(w)
    buf = hga.Buffers(p)
    Q, K, V, dO = (to_dev(x[k], "bf16") for k in ("Q", "K", "V", "dO"))
    buf.summaries(K, 0, w.T)
    buf.step(Q, K, V, dO)                       # routing, forward, backward: one problem
    torch.cuda.synchronize()
    assert hga.device_status() == 0
    units = [(0, 0), (w.B // 2, 3), (w.B - 1, w.Hkv - 1)]
    for (b, g) in units:
        wu, xu = unit_slice(w, x, b, g)
        x64 = f64(xu)
        dims = dims_of(wu)
        orc = oracle.route(dims, x64["Q"], x64["K"])
        got_c = buf.cidx[b:b + 1, g:g + 1].cpu().numpy()
        got_g = buf.gidx[b:b + 1, g:g + 1].cpu().numpy()
        check_block_routing(wu, got_c, got_g, orc)
        O, lse = oracle.attn_fwd(dims, x64["Q"], x64["K"], x64["V"], got_g)
        dQ, dK, dV = oracle.attn_bwd(dims, x64["Q"], x64["K"], x64["V"], x64["dO"], got_g)
        hs = slice(g * w.G, (g + 1) * w.G)
        for k, got, want in (("O", buf.O[b:b + 1, hs], O), ("lse", buf.lse[b:b + 1, hs], lse),
                             ("dQ", buf.dQ[b:b + 1, hs], dQ), ("dK", buf.dK[b:b + 1, g:g + 1], dK),
                             ("dV", buf.dV[b:b + 1, g:g + 1], dV)):
            err = maxabs(got.cpu().numpy(), want)
            assert err <= TOL["bf16"], (w.name, b, g, k, err)
