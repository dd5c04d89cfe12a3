"""Pins of the CPU oracle against facts outside the oracle itself.

The oracle (``oracle/hga_oracle.c``) is the parity reference of the CUDA
path, so before it is trusted every stage is checked here against
something it does not contain: library routines (numpy means, torch's
scaled-dot-product attention and autograd in float64), closed forms,
brute-force selection on tiny inputs, constructed cases with a known
answer, invariances and central finite differences.

Method source: the article "BMW's 16 GB GPU just did what needs an A100"
(seventnews.com), section "What HGA does differently" (64-token chunks,
8-token groups, top-k chunks then top-k groups, exact-token attention,
weight-free router) and the segment-wise backward described in the same
section.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from hierarchical_routed_sparse_b200.workloads import Workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _inputs(w: Workload):
    x = w.full()
    return {k: v.astype(np.float64) for k, v in x.items()}


def _dims(oracle, w: Workload, **kw):
    return oracle.Dims(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, T_hist=w.T_hist, T_seg=w.T_seg,
                       k_c=kw.pop("k_c", w.k_c), k_g=kw.pop("k_g", w.k_g), **kw)


# ----------------------------------------------------------- summaries ----
def test_summaries_match_numpy_mean(oracle_mod):
    w = Workload("t", B=2, Hq=2, Hkv=2, d=16, T_hist=128, T_seg=128, k_c=2, k_g=4, dtype="fp32")
    x = _inputs(w)
    dims = _dims(oracle_mod, w)
    csum, gsum = oracle_mod.build_summaries(dims, x["K"])
    K = x["K"]
    np.testing.assert_allclose(csum, K.reshape(2, 2, w.T // 64, 64, 16).mean(axis=3), rtol=0, atol=1e-14)
    np.testing.assert_allclose(gsum, K.reshape(2, 2, w.T // 8, 8, 16).mean(axis=3), rtol=0, atol=1e-14)


def test_summaries_closed_forms(oracle_mod):
    # Constant keys per chunk -> the summaries are that constant.
    dims = oracle_mod.Dims(B=1, Hq=1, Hkv=1, d=4, T_hist=0, T_seg=256, k_c=1, k_g=1)
    vals = np.array([3.0, -1.5, 0.25, 7.0])
    K = np.repeat(vals, 64)[None, None, :, None] * np.ones((1, 1, 1, 4))
    csum, gsum = oracle_mod.build_summaries(dims, K)
    np.testing.assert_array_equal(csum[0, 0, :, 0], vals)
    np.testing.assert_array_equal(gsum[0, 0, :, 0], np.repeat(vals, 8))
    # A linear ramp K[t] = a + b t: the mean of a run is its midpoint.
    t = np.arange(256, dtype=np.float64)
    K = (2.0 + 0.5 * t)[None, None, :, None] * np.ones((1, 1, 1, 4))
    csum, gsum = oracle_mod.build_summaries(dims, K)
    np.testing.assert_allclose(csum[0, 0, :, 0], 2.0 + 0.5 * (64 * np.arange(4) + 31.5), rtol=1e-15)
    np.testing.assert_allclose(gsum[0, 0, :, 0], 2.0 + 0.5 * (8 * np.arange(32) + 3.5), rtol=1e-15)


def test_summaries_partial_range_leaves_rest(oracle_mod):
    w = Workload("t", B=1, Hq=1, Hkv=1, d=8, T_hist=128, T_seg=128, k_c=2, k_g=4, dtype="fp32")
    x = _inputs(w)
    dims = _dims(oracle_mod, w)
    full_c, full_g = oracle_mod.build_summaries(dims, x["K"])
    c0 = np.full_like(full_c, 9.0)
    g0 = np.full_like(full_g, 9.0)
    c1, g1 = oracle_mod.build_summaries(dims, x["K"], 128, 256, c0, g0)
    np.testing.assert_array_equal(c1[:, :, :2], 9.0)
    np.testing.assert_array_equal(g1[:, :, :16], 9.0)
    np.testing.assert_array_equal(c1[:, :, 2:], full_c[:, :, 2:])
    np.testing.assert_array_equal(g1[:, :, 16:], full_g[:, :, 16:])


# --------------------------------------------------------- block query ----
def test_block_query_is_mean_over_gqa_heads_and_block(oracle_mod):
    w = Workload("t", B=2, Hq=4, Hkv=2, d=8, T_hist=0, T_seg=192, k_c=1, k_g=1, dtype="fp32")
    x = _inputs(w)
    qbar = oracle_mod.block_query(_dims(oracle_mod, w), x["Q"])
    ref = x["Q"].reshape(2, 2, 2, 3, 64, 8).mean(axis=(2, 4))
    np.testing.assert_allclose(qbar, ref, rtol=0, atol=1e-14)


# ------------------------------------------------------------- routing ----
def _brute_topk(scores: dict, k: int):
    """Rank by counting how many candidates beat each one (no sorting)."""
    chosen = []
    for i, s in scores.items():
        beaten_by = sum(1 for j, t in scores.items() if t > s or (t == s and j < i))
        if k <= 0 or beaten_by < k:
            chosen.append(i)
    return sorted(chosen)


@pytest.mark.parametrize("T_hist,T_seg,k_c,k_g,G", [(0, 512, 3, 5, 1), (256, 256, 2, 7, 2),
                                                     (128, 192, 4, 40, 2), (448, 64, -1, 12, 1),
                                                     (64, 256, 2, -1, 4)])
def test_routing_brute_force(oracle_mod, T_hist, T_seg, k_c, k_g, G):
    w = Workload("t", B=2, Hq=2 * G, Hkv=2, d=8, T_hist=T_hist, T_seg=T_seg, k_c=k_c, k_g=k_g,
                 dtype="fp32", seed=3)
    x = _inputs(w)
    dims = _dims(oracle_mod, w)
    r = oracle_mod.route(dims, x["Q"], x["K"])
    K, Q = x["K"], x["Q"]
    for b in range(2):
        for g in range(2):
            for qb in range(T_seg // 64):
                qv = Q[b, g * G:(g + 1) * G, qb * 64:(qb + 1) * 64].mean(axis=(0, 1))
                c0 = T_hist // 64 + qb
                cs = {c: float(qv @ K[b, g, 64 * c:64 * c + 64].mean(axis=0)) for c in range(c0)}
                want_c = _brute_topk(cs, k_c)
                got_c = [c for c in r["cidx"][b, g, qb] if c >= 0]
                assert got_c == want_c
                assert all(c == -1 for c in r["cidx"][b, g, qb][len(want_c):])
                gs = {8 * c + i: float(qv @ K[b, g, 64 * c + 8 * i:64 * c + 8 * i + 8].mean(axis=0))
                      for c in want_c for i in range(8)}
                want_g = _brute_topk(gs, k_g)
                got_g = [j for j in r["gidx"][b, g, qb] if j >= 0]
                assert got_g == want_g
                assert all(j == -1 for j in r["gidx"][b, g, qb][len(want_g):])


def test_routing_constructed_known_answer(oracle_mod):
    # 8 history chunks; chunk c holds keys w_c * e_c (+ tiny noise); the single
    # query block is sum_c v_c e_c, so the chunk scores are w_c v_c exactly
    # up to the noise: ranking by hand gives the expected choice.
    d = 16
    w_c = np.array([1.0, 2.0, 0.5, 3.0, 1.5, 0.1, 2.5, 0.2])
    v_c = np.array([1.0, 1.0, 4.0, 1.0, 1.0, 9.0, 0.2, 1.0])
    # scores = [1, 2, 2, 3.875, 1.5, 0.9, 0.5, 0.2]: chunks 1 and 2 tie
    # exactly (2.0 * 1.0 == 0.5 * 4.0 in binary floating point).
    K = np.zeros((1, 1, 9 * 64, d))
    for c in range(8):
        K[0, 0, 64 * c:64 * c + 64, c] = w_c[c]
    # groups of chunk 3: make group 3*8+5 stand out, then 3*8+1.
    K[0, 0, 3 * 64 + 40:3 * 64 + 48, 8] = 5.0
    K[0, 0, 3 * 64 + 8:3 * 64 + 16, 8] = 2.0
    Q = np.zeros((1, 1, 64, d))
    Q[0, 0, :, :8] = v_c
    Q[0, 0, :, 8] = 1.0
    dims = oracle_mod.Dims(B=1, Hq=1, Hkv=1, d=d, T_hist=512, T_seg=64, k_c=3, k_g=2)
    r = oracle_mod.route(dims, Q, K)
    # chunk 3 scores 3 + (8*5 + 8*2)/64 = 3.875; chunks 1 and 2 tie at 2 and
    # fill the other two slots.
    assert list(r["cidx"][0, 0, 0]) == [1, 2, 3]
    assert list(r["gidx"][0, 0, 0]) == [3 * 8 + 1, 3 * 8 + 5]
    # with k_c = 2 the tie between chunks 1 and 2 goes to the lower index.
    dims2 = oracle_mod.Dims(B=1, Hq=1, Hkv=1, d=d, T_hist=512, T_seg=64, k_c=2, k_g=2)
    r2 = oracle_mod.route(dims2, Q, K)
    assert list(r2["cidx"][0, 0, 0]) == [1, 3]


def test_routing_exact_ties_take_lowest_index(oracle_mod):
    # Every history chunk is a copy of the same 64 keys: all scores tie
    # exactly, so the lowest indices win at both levels.
    rng = np.random.default_rng(1)
    base = rng.standard_normal((64, 8))
    K = np.concatenate([np.tile(base, (6, 1)), rng.standard_normal((64, 8))])[None, None]
    Q = rng.standard_normal((1, 1, 64, 8))
    dims = oracle_mod.Dims(B=1, Hq=1, Hkv=1, d=8, T_hist=384, T_seg=64, k_c=3, k_g=4)
    r = oracle_mod.route(dims, Q, K)
    assert list(r["cidx"][0, 0, 0]) == [0, 1, 2]
    gs = {j: float(Q[0, 0].mean(0) @ base[8 * j:8 * j + 8].mean(0)) for j in range(8)}
    o1, o2 = sorted(gs, key=lambda j: (-gs[j], j))[:2]
    # The best in-chunk offset o1 ties across the three chosen chunks, so
    # its three copies come first (lowest chunk first); the fourth slot is
    # the second-best offset in the lowest chunk.
    assert list(r["gidx"][0, 0, 0]) == sorted([o1, 8 + o1, 16 + o1, o2])
    assert r["cgap"][0, 0, 0] == 0.0


def test_routing_invariances(oracle_mod):
    w = Workload("t", B=1, Hq=4, Hkv=1, d=16, T_hist=512, T_seg=256, k_c=3, k_g=9, dtype="fp32",
                 keys="clustered", seed=7)
    x = _inputs(w)
    dims = _dims(oracle_mod, w)
    r = oracle_mod.route(dims, x["Q"], x["K"])
    # Scaling K by a positive constant keeps every choice.
    r2 = oracle_mod.route(dims, x["Q"], 2.5 * x["K"])
    np.testing.assert_array_equal(r["cidx"], r2["cidx"])
    np.testing.assert_array_equal(r["gidx"], r2["gidx"])
    # Permuting the q-heads that share a kv-head keeps every choice.
    r3 = oracle_mod.route(dims, x["Q"][:, [2, 0, 3, 1]], x["K"])
    np.testing.assert_array_equal(r["cidx"], r3["cidx"])
    np.testing.assert_array_equal(r["gidx"], r3["gidx"])
    # The own chunk (and anything later) is never routed; groups come only
    # from chosen chunks.
    for qb in range(4):
        c0 = 512 // 64 + qb
        cs = [c for c in r["cidx"][0, 0, qb] if c >= 0]
        assert len(cs) == min(3, c0) and all(c < c0 for c in cs)
        assert all(j // 8 in cs for j in r["gidx"][0, 0, qb] if j >= 0)


def test_routing_gap_definition(oracle_mod):
    # Chunk scores constructed as exactly 5, 4, 3.9, 1 -> k=2 gap is
    # (4 - 3.9) / max(4, 3.9, 1e-3 rms) = 0.025.
    K = np.zeros((1, 1, 5 * 64, 4))
    for c, s in enumerate([5.0, 4.0, 3.9, 1.0]):
        K[0, 0, 64 * c:64 * c + 64, 0] = s
    Q = np.zeros((1, 1, 64, 4))
    Q[..., 0] = 1.0
    dims = oracle_mod.Dims(B=1, Hq=1, Hkv=1, d=4, T_hist=256, T_seg=64, k_c=2, k_g=1)
    r = oracle_mod.route(dims, Q, K)
    assert list(r["cidx"][0, 0, 0]) == [0, 1]
    assert r["cgap"][0, 0, 0] == pytest.approx(0.1 / 4.0, rel=1e-12)
    # k_c covering every candidate: no (k+1)-th score, gap is infinite.
    dims = oracle_mod.Dims(B=1, Hq=1, Hkv=1, d=4, T_hist=256, T_seg=64, k_c=4, k_g=1)
    assert math.isinf(oracle_mod.route(dims, Q, K)["cgap"][0, 0, 0])


def test_routing_gap_floor_decides_near_zero_scores(oracle_mod):
    # Chunk scores 10, 2e-6, 1e-6, -30 with k_c 2: the k-th and (k+1)-th
    # scores are near zero, so the floor tau = 1e-3 * rms of ALL four
    # eligible scores sets the denominator:
    #   rms = sqrt((100 + 4e-12 + 1e-12 + 900) / 4) = sqrt(250.00000000000125)
    #   gap = (2e-6 - 1e-6) / (1e-3 * rms) = 6.32455532e-5  (exempt: < 1e-4).
    # Plausible slips give other values: no floor -> 0.5; rms over the kept
    # scores only -> 1.414e-4 (not exempt); no square root -> 4e-6; a floor
    # factor of 1e-4 -> 6.3e-4.
    K = np.zeros((1, 1, 5 * 64, 4))
    for c, s in enumerate([10.0, 2e-6, 1e-6, -30.0]):
        K[0, 0, 64 * c:64 * c + 64, 0] = s
    Q = np.zeros((1, 1, 64, 4))
    Q[..., 0] = 1.0
    dims = oracle_mod.Dims(B=1, Hq=1, Hkv=1, d=4, T_hist=256, T_seg=64, k_c=2, k_g=1)
    r = oracle_mod.route(dims, Q, K)
    assert list(r["cidx"][0, 0, 0]) == [0, 1]
    want = 1e-6 / (1e-3 * math.sqrt((100.0 + 4e-12 + 1e-12 + 900.0) / 4.0))
    assert want == pytest.approx(6.32455532e-5, rel=1e-8)
    assert r["cgap"][0, 0, 0] == pytest.approx(want, rel=1e-6)
    assert r["cgap"][0, 0, 0] < 1e-4
    # The same floor at group level: the one eligible chunk's eight groups
    # score 10, 2e-6, 1e-6, -30, 0, 0, 0, 0 (k_g 2); rms over the eight
    # candidates is sqrt(1000 / 8) = sqrt(125), so the gap is
    # 1e-6 / (1e-3 * sqrt(125)) = 8.94427191e-5.
    K = np.zeros((1, 1, 128, 4))
    for j, s in enumerate([10.0, 2e-6, 1e-6, -30.0, 0.0, 0.0, 0.0, 0.0]):
        K[0, 0, 8 * j:8 * j + 8, 0] = s
    dims = oracle_mod.Dims(B=1, Hq=1, Hkv=1, d=4, T_hist=64, T_seg=64, k_c=1, k_g=2)
    r = oracle_mod.route(dims, Q, K)
    assert list(r["gidx"][0, 0, 0]) == [0, 1]
    want = 1e-6 / (1e-3 * math.sqrt((100.0 + 4e-12 + 1e-12 + 900.0) / 8.0))
    assert want == pytest.approx(8.94427191e-5, rel=1e-8)
    assert r["ggap"][0, 0, 0] == pytest.approx(want, rel=1e-6)


def test_hand_worked_example(oracle_mod):
    """Tiny example worked by hand (chunk 4, group 2, d 2); see the fixture."""
    with open(os.path.join(GOLDEN, "hand_worked_example.json")) as f:
        ex = json.load(f)
    K = np.array(ex["K"], dtype=np.float64)[None, None]
    V = np.array(ex["V"], dtype=np.float64)[None, None]
    Q = np.array(ex["Q"], dtype=np.float64)[None, None]
    dims = oracle_mod.Dims(B=1, Hq=1, Hkv=1, d=2, T_hist=ex["T_hist"], T_seg=ex["T_seg"],
                           k_c=ex["k_c"], k_g=ex["k_g"], chunk=ex["chunk"], group=ex["group"])
    r = oracle_mod.route(dims, Q, K)
    np.testing.assert_array_equal(r["csum"][0, 0], ex["csum"])
    np.testing.assert_array_equal(r["gsum"][0, 0], ex["gsum"])
    assert list(r["cidx"][0, 0, 0]) == ex["cidx"]
    assert list(r["gidx"][0, 0, 0]) == ex["gidx"]
    O, lse = oracle_mod.attn_fwd(dims, Q, K, V, r["gidx"])
    # Closed forms of the fixture's derivation: query i sees tokens 6, 7
    # (score q.k = 2 each, scaled by 1/sqrt 2) and own tokens 8..8+i
    # (score 0); V6 = (1, 0), V7 = (0, 1), own V = 0.
    a = math.exp(2.0 / math.sqrt(2.0))
    for i in range(4):
        den = 2 * a + (i + 1)
        np.testing.assert_allclose(O[0, 0, i], [a / den, a / den], rtol=1e-14)
        assert lse[0, 0, i] == pytest.approx(math.log(den), rel=1e-14)
    # Backward closed forms of the fixture's backward derivation (dO_i = (1, 0)).
    dO = np.array(ex["dO"], dtype=np.float64)[None, None]
    dQ, dK, dV = oracle_mod.attn_bwd(dims, Q, K, V, dO, r["gidx"])
    s = 1.0 / math.sqrt(2.0)
    Z = [2 * a + (i + 1) for i in range(4)]
    for i in range(4):
        np.testing.assert_allclose(dQ[0, 0, i], [0.0, s * 2 * (a / Z[i]) * (1 - 2 * a / Z[i])],
                                   rtol=1e-13, atol=1e-15)
    for m in range(4):
        k_m = -s * sum(a / Z[i] ** 2 for i in range(m, 4))
        v_m = sum(1.0 / Z[i] for i in range(m, 4))
        np.testing.assert_allclose(dK[0, 0, m], [k_m, k_m], rtol=1e-13)
        np.testing.assert_allclose(dV[0, 0, m], [v_m, 0.0], rtol=1e-13, atol=1e-15)


# ----------------------------------------------------- attention forward --
def _dense_sdpa(Q, K, V, T_hist, scale, keep=None):
    """torch SDPA (float64) with the token-causal mask of the segment."""
    B, Hq, Ts, d = Q.shape
    Hkv, T = K.shape[1], K.shape[2]
    G = Hq // Hkv
    Kt = torch.from_numpy(K).repeat_interleave(G, dim=1)
    Vt = torch.from_numpy(V).repeat_interleave(G, dim=1)
    pos = T_hist + torch.arange(Ts)[:, None]
    mask = torch.arange(T)[None, :] <= pos
    if keep is not None:
        mask = mask[None, None] & torch.from_numpy(keep)
    O = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(Q), Kt, Vt,
                                                         attn_mask=mask, scale=scale)
    S = torch.einsum("bhid,bhjd->bhij", torch.from_numpy(Q), Kt) * scale
    lse = torch.logsumexp(S.masked_fill(~mask, -math.inf), dim=-1)
    return O.numpy(), lse.numpy()


@pytest.mark.parametrize("T_hist,G", [(0, 1), (320, 2), (128, 4)])
def test_all_routing_equals_dense_causal(oracle_mod, T_hist, G):
    w = Workload("t", B=2, Hq=2 * G, Hkv=2, d=16, T_hist=T_hist, T_seg=256, k_c=-1, k_g=-1,
                 dtype="fp32", seed=2)
    x = _inputs(w)
    dims = _dims(oracle_mod, w)
    r = oracle_mod.route(dims, x["Q"], x["K"])
    O, lse = oracle_mod.attn_fwd(dims, x["Q"], x["K"], x["V"], r["gidx"])
    O_ref, lse_ref = _dense_sdpa(x["Q"], x["K"], x["V"], T_hist, dims.scale)
    np.testing.assert_allclose(O, O_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


def test_tiny_fp32_all_equals_dense(oracle_mod):
    """The tiny fp32 workload (d 64, T 1024) with k = all is dense causal."""
    from hierarchical_routed_sparse_b200.workloads import TINY_FP32
    w = TINY_FP32.with_(k_c=-1, k_g=-1)
    x = _inputs(w)
    dims = _dims(oracle_mod, w)
    r = oracle_mod.route(dims, x["Q"], x["K"])
    O, lse = oracle_mod.attn_fwd(dims, x["Q"], x["K"], x["V"], r["gidx"])
    O_ref, lse_ref = _dense_sdpa(x["Q"], x["K"], x["V"], 0, dims.scale)
    np.testing.assert_allclose(O, O_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


def test_chunk_level_when_all_groups_of_chosen_chunks(oracle_mod):
    # k_g = 8 k_c keeps every group of each chosen chunk: the key set is the
    # chosen chunks plus the own causal chunk.
    w = Workload("t", B=1, Hq=2, Hkv=1, d=16, T_hist=384, T_seg=192, k_c=2, k_g=16,
                 dtype="fp32", keys="clustered", seed=4)
    x = _inputs(w)
    dims = _dims(oracle_mod, w)
    r = oracle_mod.route(dims, x["Q"], x["K"])
    O, lse = oracle_mod.attn_fwd(dims, x["Q"], x["K"], x["V"], r["gidx"])
    keep = np.zeros((1, 2, 192, w.T), dtype=bool)
    for qb in range(3):
        for c in r["cidx"][0, 0, qb]:
            keep[:, :, 64 * qb:64 * qb + 64, 64 * c:64 * c + 64] = True
        own = 384 + 64 * qb
        keep[:, :, 64 * qb:64 * qb + 64, own:own + 64] = True
    O_ref, lse_ref = _dense_sdpa(x["Q"], x["K"], x["V"], 384, dims.scale, keep)
    np.testing.assert_allclose(O, O_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


def test_single_block_no_history_is_plain_causal(oracle_mod):
    w = Workload("t", B=1, Hq=3, Hkv=1, d=32, T_hist=0, T_seg=64, k_c=4, k_g=16, dtype="fp32",
                 seed=9)
    x = _inputs(w)
    dims = _dims(oracle_mod, w)
    r = oracle_mod.route(dims, x["Q"], x["K"])
    assert (r["cidx"] == -1).all() and (r["gidx"] == -1).all()
    O, _ = oracle_mod.attn_fwd(dims, x["Q"], x["K"], x["V"], r["gidx"])
    O_ref, _ = _dense_sdpa(x["Q"], x["K"], x["V"], 0, dims.scale)
    np.testing.assert_allclose(O, O_ref, rtol=0, atol=1e-12)


def test_identical_group_keys_give_mean_of_values(oracle_mod):
    # History: 8 identical groups; the single chosen group is the lowest one
    # (tie) and its 8 equal scores weight its values equally.  Own-chunk
    # keys point away from the queries, so they carry negligible weight.
    d = 8
    kstar = np.zeros(d)
    kstar[0] = 1.0
    K = np.zeros((1, 1, 128, d))
    K[0, 0, :64] = kstar
    K[0, 0, 64:] = -kstar
    rng = np.random.default_rng(11)
    V = rng.standard_normal((1, 1, 128, d))
    Q = np.zeros((1, 1, 64, d))
    Q[..., 0] = 100.0
    dims = oracle_mod.Dims(B=1, Hq=1, Hkv=1, d=d, T_hist=64, T_seg=64, k_c=1, k_g=1)
    r = oracle_mod.route(dims, Q, K)
    assert list(r["gidx"][0, 0, 0]) == [0]
    O, lse = oracle_mod.attn_fwd(dims, Q, K, V, r["gidx"])
    np.testing.assert_allclose(O[0, 0], np.broadcast_to(V[0, 0, :8].mean(0), (64, d)),
                               rtol=0, atol=1e-12)
    s = 100.0 / math.sqrt(d)
    np.testing.assert_allclose(lse[0, 0], s + math.log(8.0), rtol=1e-12)


# ---------------------------------------------------- attention backward --
def _fd_case(oracle, seed=0):
    w = Workload("t", B=1, Hq=2, Hkv=1, d=16, T_hist=128, T_seg=256, k_c=2, k_g=4,
                 dtype="fp32", keys="clustered", seed=seed, backward=True)
    x = _inputs(w)
    dims = _dims(oracle, w)
    gidx = oracle.route(dims, x["Q"], x["K"])["gidx"]
    return w, x, dims, gidx


def test_backward_central_finite_differences(oracle_mod):
    w, x, dims, gidx = _fd_case(oracle_mod)
    dQ, dK, dV = oracle_mod.attn_bwd(dims, x["Q"], x["K"], x["V"], x["dO"], gidx)

    def loss(Q, K, V):
        O, _ = oracle_mod.attn_fwd(dims, Q, K, V, gidx)
        return float((O * x["dO"]).sum())

    rng = np.random.default_rng(0)
    h = 1e-6
    for name, grad, sl in (("Q", dQ, None), ("K", dK, w.T_hist), ("V", dV, w.T_hist)):
        for _ in range(12):
            idx = tuple(int(rng.integers(0, n)) for n in grad.shape)
            full_idx = idx if sl is None else (idx[0], idx[1], idx[2] + sl, idx[3])
            args = {k: x[k].copy() for k in ("Q", "K", "V")}
            args[name][full_idx] += h
            up = loss(args["Q"], args["K"], args["V"])
            args[name][full_idx] -= 2 * h
            dn = loss(args["Q"], args["K"], args["V"])
            fd = (up - dn) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(grad[idx])), (name, idx, fd, grad[idx])


def test_backward_all_routing_equals_autograd_dense(oracle_mod):
    w = Workload("t", B=1, Hq=4, Hkv=2, d=16, T_hist=192, T_seg=128, k_c=-1, k_g=-1,
                 dtype="fp32", seed=6, backward=True)
    x = _inputs(w)
    dims = _dims(oracle_mod, w)
    gidx = oracle_mod.route(dims, x["Q"], x["K"])["gidx"]
    dQ, dK, dV = oracle_mod.attn_bwd(dims, x["Q"], x["K"], x["V"], x["dO"], gidx)
    Q = torch.from_numpy(x["Q"]).requires_grad_()
    K = torch.from_numpy(x["K"]).requires_grad_()
    V = torch.from_numpy(x["V"]).requires_grad_()
    pos = 192 + torch.arange(128)[:, None]
    mask = torch.arange(w.T)[None, :] <= pos
    O = torch.nn.functional.scaled_dot_product_attention(
        Q, K.repeat_interleave(2, 1), V.repeat_interleave(2, 1), attn_mask=mask, scale=dims.scale)
    (O * torch.from_numpy(x["dO"])).sum().backward()
    np.testing.assert_allclose(dQ, Q.grad.numpy(), rtol=0, atol=1e-12)
    # The segment part of dK/dV is kept; history is detached (its autograd
    # gradient exists but the method drops it).
    np.testing.assert_allclose(dK, K.grad.numpy()[:, :, 192:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(dV, V.grad.numpy()[:, :, 192:], rtol=0, atol=1e-12)
    assert np.abs(K.grad.numpy()[:, :, :192]).max() > 1e-3


def test_backward_history_receives_nothing(oracle_mod):
    # Only segment tokens have a dK/dV row; the sum over segment rows of
    # dV equals the total probability mass placed on segment keys times dO.
    w, x, dims, gidx = _fd_case(oracle_mod, seed=1)
    dQ, dK, dV = oracle_mod.attn_bwd(dims, x["Q"], x["K"], x["V"], x["dO"], gidx)
    assert dK.shape == (1, 1, w.T_seg, w.d) and dV.shape == (1, 1, w.T_seg, w.d)
    # sum_j dS_j = 0 per query row -> sum of dK over every key (history
    # included) is 0; the segment part alone is not, in general.
    V1 = np.ones_like(x["V"])
    dQ1, dK1, dV1 = oracle_mod.attn_bwd(dims, x["Q"], x["K"], V1, x["dO"], gidx)
    # Constant V: O is constant, so dP - D = 0 and every dS (dQ, dK) vanishes.
    assert np.abs(dQ1).max() < 1e-13 and np.abs(dK1).max() < 1e-13
