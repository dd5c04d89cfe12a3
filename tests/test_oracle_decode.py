"""Pins of the oracle's decode step (a query block of one token; article
section "Retrieval: no degradation in the dense baseline": HGA itself can
also do generation).

  * It equals the segment oracle on a block whose 64 queries are all the
    decode token's query: the block query is then that query (mean over G
    heads), the eligible chunks are the same (c < pos / 64), and row
    i = pos mod 64 attends the same keys.  The segment oracle is pinned by
    test_oracle_pins.py, so this pins routing and attention of the decode.
  * With every chunk and group routed it is dense causal attention of the
    token over positions 0..pos (a direct numpy softmax, written here).
  * At pos 0 it is V[0] exactly, with lse = scale * q . k_0.
"""
import math

import numpy as np
import pytest

import oracle


def _inputs(rng, B, Hq, Hkv, d, T, clustered=True):
    if clustered:
        cent = rng.standard_normal((B, Hkv, 8, d))
        pick = rng.integers(0, 8, size=(B, Hkv, T // 64))
        K = np.repeat(np.take_along_axis(cent, pick[..., None], axis=2), 64, axis=2)
        K = K + 0.3 * rng.standard_normal((B, Hkv, T, d))
    else:
        K = rng.standard_normal((B, Hkv, T, d))
    V = rng.standard_normal((B, Hkv, T, d))
    q = rng.standard_normal((B, Hq, d))
    return q, K, V


@pytest.mark.parametrize("pos", [0, 5, 63, 64, 100, 127, 128, 200, 383])
def test_decode_equals_block_of_identical_queries(pos):
    rng = np.random.default_rng(pos + 1)
    B, Hq, Hkv, d, T = 2, 4, 2, 16, 384
    k_c, k_g = 2, 5
    q, K, V = _inputs(rng, B, Hq, Hkv, d, T)
    dd = oracle.Dims(B=B, Hq=Hq, Hkv=Hkv, d=d, T_hist=T - 64, T_seg=64, k_c=k_c, k_g=k_g)
    dd.wc, dd.wg = k_c, k_g
    csum, gsum = oracle.build_summaries(dd, K)
    dec = oracle.decode(dd, pos, q, K, V, csum, gsum)

    c0, i = pos // 64, pos % 64
    T_tr = 64 * c0 + 64
    dt = oracle.Dims(B=B, Hq=Hq, Hkv=Hkv, d=d, T_hist=64 * c0, T_seg=64, k_c=k_c, k_g=k_g)
    dt.wc, dt.wg = k_c, k_g
    Q = np.repeat(q[:, :, None, :], 64, axis=2)
    Kt, Vt = K[:, :, :T_tr], V[:, :, :T_tr]
    r = oracle.route(dt, Q, Kt)
    O, lse = oracle.attn_fwd(dt, Q, Kt, Vt, r["gidx"])
    assert np.array_equal(dec["cidx"], r["cidx"][:, :, 0])
    assert np.array_equal(dec["gidx"], r["gidx"][:, :, 0])
    np.testing.assert_allclose(dec["O"], O[:, :, i], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dec["lse"], lse[:, :, i], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("pos", [0, 31, 64, 190, 255])
def test_decode_all_routing_is_dense_causal(pos):
    rng = np.random.default_rng(100 + pos)
    B, Hq, Hkv, d, T = 1, 4, 1, 32, 256
    q, K, V = _inputs(rng, B, Hq, Hkv, d, T, clustered=False)
    dd = oracle.Dims(B=B, Hq=Hq, Hkv=Hkv, d=d, T_hist=T - 64, T_seg=64, k_c=-1, k_g=-1)
    csum, gsum = oracle.build_summaries(dd, K)
    dec = oracle.decode(dd, pos, q, K, V, csum, gsum)
    scale = 1.0 / math.sqrt(d)
    for h in range(Hq):
        s = scale * K[0, 0, :pos + 1] @ q[0, h]
        w = np.exp(s - s.max())
        np.testing.assert_allclose(dec["O"][0, h], (w / w.sum()) @ V[0, 0, :pos + 1], rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(dec["lse"][0, h], s.max() + np.log(w.sum()), rtol=1e-12)


def test_decode_first_token():
    rng = np.random.default_rng(7)
    B, Hq, Hkv, d, T = 2, 2, 2, 8, 128
    q, K, V = _inputs(rng, B, Hq, Hkv, d, T, clustered=False)
    dd = oracle.Dims(B=B, Hq=Hq, Hkv=Hkv, d=d, T_hist=64, T_seg=64, k_c=3, k_g=4)
    csum, gsum = oracle.build_summaries(dd, K)
    dec = oracle.decode(dd, 0, q, K, V, csum, gsum)
    assert (dec["cidx"] == -1).all() and (dec["gidx"] == -1).all()
    for b in range(B):
        for h in range(Hq):
            np.testing.assert_array_equal(dec["O"][b, h], V[b, h, 0])
            np.testing.assert_allclose(dec["lse"][b, h], (K[b, h, 0] @ q[b, h]) / math.sqrt(d), rtol=1e-14)
