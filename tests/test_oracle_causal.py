"""Pins of the oracle's strictly causal variant (article "BMW's 16 GB GPU
just did what needs an A100", section "The one real caveat: causal leakage":
a block's routing depends on several query positions, so an earlier token
sees later tokens through it; a strictly causal variant is in the works).
Reading: every query position routes on its own query, a block of one.

  * Row i equals the decode step at position T_hist + i (the decode oracle is
    pinned against the segment oracle by test_oracle_decode.py).
  * With the 64 queries of every block identical, per-position routing is
    the block routing, so routing, forward and backward equal the block
    oracle (pinned by test_oracle_pins.py).
  * Strict causality: changing Q / K / V at positions after p leaves every
    output at positions <= p unchanged; the same change moves the block
    variant's outputs at p (the leak the variant removes).
  * Full routing is dense causal attention.
  * The backward matches central finite differences of the forward with the
    routing frozen.
"""
import math

import numpy as np
import pytest

import oracle


def _inputs(rng, B, Hq, Hkv, d, T_hist, T_seg, clustered=True):
    T = T_hist + T_seg
    if clustered:
        cent = rng.standard_normal((B, Hkv, 8, d))
        pick = rng.integers(0, 8, size=(B, Hkv, T // 64))
        K = np.repeat(np.take_along_axis(cent, pick[..., None], axis=2), 64, axis=2)
        K = K + 0.3 * rng.standard_normal((B, Hkv, T, d))
    else:
        K = rng.standard_normal((B, Hkv, T, d))
    V = rng.standard_normal((B, Hkv, T, d))
    Q = rng.standard_normal((B, Hq, T_seg, d))
    return Q, K, V


def _dims(B, Hq, Hkv, d, T_hist, T_seg, k_c, k_g):
    return oracle.Dims(B=B, Hq=Hq, Hkv=Hkv, d=d, T_hist=T_hist, T_seg=T_seg, k_c=k_c, k_g=k_g)


def _causal(dims, Q, K, V):
    csum, gsum = oracle.build_summaries(dims, K)
    r = oracle.causal_route(dims, Q, csum, gsum)
    O, lse = oracle.causal_attn_fwd(dims, Q, K, V, r["gidx"])
    return r, O, lse


def test_rows_equal_the_decode_step():
    rng = np.random.default_rng(11)
    B, Hq, Hkv, d, Th, Ts = 2, 4, 2, 16, 192, 128
    dims = _dims(B, Hq, Hkv, d, Th, Ts, 2, 5)
    Q, K, V = _inputs(rng, B, Hq, Hkv, d, Th, Ts)
    csum, gsum = oracle.build_summaries(dims, K)
    r, O, lse = _causal(dims, Q, K, V)
    for i in range(Ts):
        dec = oracle.decode(dims, Th + i, Q[:, :, i], K, V, csum, gsum)
        assert np.array_equal(r["cidx"][:, :, i], dec["cidx"]), i
        assert np.array_equal(r["gidx"][:, :, i], dec["gidx"]), i
        np.testing.assert_allclose(O[:, :, i], dec["O"], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse[:, :, i], dec["lse"], rtol=1e-12, atol=1e-12)
        np.testing.assert_array_equal(r["cgap"][:, :, i], dec["cgap"])


@pytest.mark.parametrize("k_c,k_g", [(2, 7), (3, 24), (-1, -1)])
def test_identical_block_queries_give_the_block_variant(k_c, k_g):
    rng = np.random.default_rng(20 + k_c)
    B, Hq, Hkv, d, Th, Ts = 1, 4, 2, 16, 256, 192
    dims = _dims(B, Hq, Hkv, d, Th, Ts, k_c, k_g)
    Q, K, V = _inputs(rng, B, Hq, Hkv, d, Th, Ts)
    # Every block's 64 queries equal the block's first one (per q-head).
    Q = np.repeat(Q[:, :, ::64], 64, axis=2)
    dO = rng.standard_normal(Q.shape)
    rc, Oc, lc = _causal(dims, Q, K, V)
    rb = oracle.route(dims, Q, K)
    for i in range(Ts):
        assert np.array_equal(rc["cidx"][:, :, i], rb["cidx"][:, :, i // 64])
        assert np.array_equal(rc["gidx"][:, :, i], rb["gidx"][:, :, i // 64])
    Ob, lb = oracle.attn_fwd(dims, Q, K, V, rb["gidx"])
    np.testing.assert_allclose(Oc, Ob, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lc, lb, rtol=1e-12, atol=1e-12)
    gc = oracle.causal_attn_bwd(dims, Q, K, V, dO, rc["gidx"])
    gb = oracle.attn_bwd(dims, Q, K, V, dO, rb["gidx"])
    for a, b in zip(gc, gb):
        np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)


def test_outputs_depend_on_earlier_positions_only():
    rng = np.random.default_rng(5)
    B, Hq, Hkv, d, Th, Ts = 1, 4, 1, 16, 512, 128
    dims = _dims(B, Hq, Hkv, d, Th, Ts, 2, 5)
    Q, K, V = _inputs(rng, B, Hq, Hkv, d, Th, Ts)
    p = 70                                        # inside the segment's second block
    r0, O0, l0 = _causal(dims, Q, K, V)
    # Change everything after position p: later queries (including the rest
    # of p's own block), later keys and values of the segment.
    Q2, K2, V2 = Q.copy(), K.copy(), V.copy()
    Q2[:, :, p + 1:] = 25.0 * rng.standard_normal(Q2[:, :, p + 1:].shape)
    K2[:, :, Th + p + 1:] = rng.standard_normal(K2[:, :, Th + p + 1:].shape)
    V2[:, :, Th + p + 1:] = rng.standard_normal(V2[:, :, Th + p + 1:].shape)
    r1, O1, l1 = _causal(dims, Q2, K2, V2)
    assert np.array_equal(r0["gidx"][:, :, :p + 1], r1["gidx"][:, :, :p + 1])
    assert np.array_equal(O0[:, :, :p + 1], O1[:, :, :p + 1])
    assert np.array_equal(l0[:, :, :p + 1], l1[:, :, :p + 1])
    assert not np.allclose(O0[:, :, p + 1:], O1[:, :, p + 1:])
    # The block variant leaks: only the later queries of p's block change,
    # yet the block's routing and the output at p move.
    Q3 = Q.copy()
    Q3[:, :, p + 1:128] = Q2[:, :, p + 1:128]
    rb0, rb1 = oracle.route(dims, Q, K), oracle.route(dims, Q3, K)
    assert not np.array_equal(rb0["gidx"][:, :, 1], rb1["gidx"][:, :, 1])
    Ob0, _ = oracle.attn_fwd(dims, Q, K, V, rb0["gidx"])
    Ob1, _ = oracle.attn_fwd(dims, Q3, K, V, rb1["gidx"])
    assert np.abs(Ob0[:, :, p] - Ob1[:, :, p]).max() > 1e-3


def test_all_routing_is_dense_causal():
    rng = np.random.default_rng(9)
    B, Hq, Hkv, d, Th, Ts = 1, 2, 1, 16, 128, 128
    dims = _dims(B, Hq, Hkv, d, Th, Ts, -1, -1)
    Q, K, V = _inputs(rng, B, Hq, Hkv, d, Th, Ts, clustered=False)
    _, O, lse = _causal(dims, Q, K, V)
    scale = 1.0 / math.sqrt(d)
    for h in range(Hq):
        for i in range(Ts):
            s = scale * K[0, 0, :Th + i + 1] @ Q[0, h, i]
            w = np.exp(s - s.max())
            np.testing.assert_allclose(O[0, h, i], (w / w.sum()) @ V[0, 0, :Th + i + 1], rtol=1e-11,
                                       atol=1e-12)
            np.testing.assert_allclose(lse[0, h, i], s.max() + np.log(w.sum()), rtol=1e-12)


def test_backward_matches_finite_differences():
    rng = np.random.default_rng(3)
    B, Hq, Hkv, d, Th, Ts = 1, 2, 1, 8, 128, 128
    dims = _dims(B, Hq, Hkv, d, Th, Ts, 1, 3)
    Q, K, V = _inputs(rng, B, Hq, Hkv, d, Th, Ts)
    csum, gsum = oracle.build_summaries(dims, K)
    gidx = oracle.causal_route(dims, Q, csum, gsum)["gidx"]   # frozen routing
    W = rng.standard_normal((B, Hq, Ts, d))
    dQ, dK, dV = oracle.causal_attn_bwd(dims, Q, K, V, W, gidx)

    def loss(Q_, K_, V_):
        return float((oracle.causal_attn_fwd(dims, Q_, K_, V_, gidx)[0] * W).sum())

    h = 1e-6
    for _ in range(12):
        b, hq, i, e = 0, rng.integers(Hq), rng.integers(Ts), rng.integers(d)
        Qp, Qm = Q.copy(), Q.copy()
        Qp[b, hq, i, e] += h
        Qm[b, hq, i, e] -= h
        np.testing.assert_allclose((loss(Qp, K, V) - loss(Qm, K, V)) / (2 * h), dQ[b, hq, i, e], rtol=1e-5,
                                   atol=1e-7)
        t = rng.integers(Ts)
        for X, dX, which in ((K, dK, 0), (V, dV, 1)):
            Xp, Xm = X.copy(), X.copy()
            Xp[b, 0, Th + t, e] += h
            Xm[b, 0, Th + t, e] -= h
            args_p = (Q, Xp, V) if which == 0 else (Q, K, Xp)
            args_m = (Q, Xm, V) if which == 0 else (Q, K, Xm)
            fd = (loss(*args_p) - loss(*args_m)) / (2 * h)
            np.testing.assert_allclose(fd, dX[b, 0, t, e], rtol=1e-5, atol=1e-7)
