"""The routing gate of the parity tests, checked on the CPU.

The GPU parity tests accept a routing row that differs from the oracle's
only where the oracle's k-th / (k+1)-th score gap is below 1e-4 (relative),
and only if the row is still a valid top-k (article "BMW's 16 GB GPU just
did what needs an A100", section "What HGA does differently": top-k chunks
by summary score, then top-k groups of those chunks).  Here "GPU" rows are
plain arrays built from the oracle's routing with one planted change each;
the checker must pass the valid ones and reject every planted mistake.
"""
import numpy as np
import pytest

from hierarchical_routed_sparse_b200.workloads import Workload

from parity_util import check_block_routing, check_decode_routing


def _problem(oracle_mod):
    """Four history chunks whose scores against the block query are 5, 4,
    4 - 1e-4 and 1 (a near-tie between chunks 1 and 2, relative gap 2.5e-5),
    with distinct group scores inside each chunk (k_c 2, k_g 3)."""
    d = 4
    K = np.zeros((1, 1, 5 * 64, d))
    chunk_val = [5.0, 4.0, 4.0 - 1e-4, 1.0, 0.0]
    offs = [1.0, -1.0, 2.0, -2.0, 3.0, -3.0, 0.5, -0.5]      # mean 0: chunk scores unchanged
    for c, v in enumerate(chunk_val):
        K[0, 0, 64 * c:64 * c + 64, 0] = v
        for r, o in enumerate(offs):
            K[0, 0, 64 * c + 8 * r:64 * c + 8 * r + 8, 1] = o * (1 + 0.1 * c)
    Q = np.zeros((1, 1, 64, d))
    Q[..., 0] = 1.0
    Q[..., 1] = 0.5
    w = Workload("planted", B=1, Hq=1, Hkv=1, d=d, T_hist=256, T_seg=64, k_c=2, k_g=3)
    dims = oracle_mod.Dims(B=1, Hq=1, Hkv=1, d=d, T_hist=256, T_seg=64, k_c=2, k_g=3)
    orc = oracle_mod.route(dims, Q, K)
    return w, dims, orc, Q, K


def test_oracle_rows_pass(oracle_mod):
    w, _, orc, _, _ = _problem(oracle_mod)
    assert orc["cidx"][0, 0, 0].tolist() == [0, 1]
    assert orc["cgap"][0, 0, 0] < 1e-4
    out = check_block_routing(w, orc["cidx"], orc["gidx"], orc)
    assert out == {"cidx_exempt_rows": 0, "gidx_exempt_rows": 0}


def test_other_side_of_a_near_tie_passes_with_its_own_groups(oracle_mod):
    w, dims, orc, _, _ = _problem(oracle_mod)
    cidx = np.array([[[[0, 2]]]], dtype=np.int32)              # chunk 2 instead of 1: a near-tie
    gidx, _ = oracle_mod.route_groups(dims, orc["qbar"], orc["gsum"], cidx)
    out = check_block_routing(w, cidx, gidx, orc)
    assert out["cidx_exempt_rows"] == 1


def test_groups_of_the_oracle_chunk_row_fail_after_a_different_chunk_row(oracle_mod):
    w, _, orc, _, _ = _problem(oracle_mod)
    cidx = np.array([[[[0, 2]]]], dtype=np.int32)
    gidx = orc["gidx"].copy()                                   # built on chunks {0, 1}
    assert (gidx[gidx >= 0] // 8 == 1).any()
    with pytest.raises(AssertionError):
        check_block_routing(w, cidx, gidx, orc)


@pytest.mark.parametrize("row", [[0, 3], [1, 2], [0, 1, 2], [0], [0, 4], [2, 0]],
                         ids=["outside_band", "drops_the_top", "too_many", "too_few",
                              "own_chunk", "not_ascending"])
def test_planted_chunk_rows_fail(oracle_mod, row):
    w, dims, orc, _, _ = _problem(oracle_mod)
    wc = max(len(row), 2)
    cidx = np.full((1, 1, 1, wc), -1, dtype=np.int32)
    cidx[0, 0, 0, :len(row)] = row
    if wc != 2:                                                # widths must match the oracle's
        ref = np.full((1, 1, 1, wc), -1, dtype=np.int32)
        ref[0, 0, 0, :2] = orc["cidx"][0, 0, 0]
        orc = dict(orc, cidx=ref)
    valid = np.sort(cidx[cidx >= 0]).astype(np.int32)
    dims2 = oracle_mod.Dims(B=1, Hq=1, Hkv=1, d=4, T_hist=256, T_seg=64, k_c=2, k_g=3, wc=wc)
    gsel = np.full((1, 1, 1, wc), -1, dtype=np.int32)
    gsel[0, 0, 0, :len(valid)] = [c for c in valid if c < 5]
    gidx, _ = oracle_mod.route_groups(dims2, orc["qbar"], orc["gsum"], gsel)
    with pytest.raises(AssertionError):
        check_block_routing(w, cidx, gidx, orc)


@pytest.mark.parametrize("change", ["outside_band", "wrong_chunk", "too_few", "duplicate"])
def test_planted_group_rows_fail(oracle_mod, change):
    w, _, orc, _, _ = _problem(oracle_mod)
    gidx = orc["gidx"].copy()
    row = gidx[0, 0, 0]
    if change == "outside_band":           # the weakest group of chunk 0 for the best one
        cand = [j for j in range(8) if j not in row]
        s = [orc["qbar"][0, 0, 0] @ orc["gsum"][0, 0, j] for j in cand]
        row[np.argmax([orc["qbar"][0, 0, 0] @ orc["gsum"][0, 0, j] for j in row])] = \
            cand[int(np.argmin(s))]
        row.sort()
    elif change == "wrong_chunk":          # a group of an unchosen chunk
        row[-1] = 8 * 3 + 1
        row.sort()
    elif change == "too_few":
        row[-1] = -1
    else:
        row[1] = row[0]
    with pytest.raises(AssertionError):
        check_block_routing(w, orc["cidx"], gidx, orc)


def test_decode_rows(oracle_mod):
    # A decode step at position 300 (chunks 0..3 eligible) of the same keys.
    w, dims, _, Q, K = _problem(oracle_mod)
    wd = w.with_(T_hist=256, T_seg=64)
    csum, gsum = oracle_mod.build_summaries(dims, K)
    q = Q[:, :, 0]
    orc = oracle_mod.decode(dims, 300, q, K, np.zeros_like(K), csum, gsum)
    check_decode_routing(wd, 300, orc["cidx"], orc["gidx"], q, csum, gsum, orc)
    bad = orc["cidx"].copy()
    bad[0, 0] = [0, 3]
    with pytest.raises(AssertionError):
        check_decode_routing(wd, 300, bad, orc["gidx"], q, csum, gsum, orc)


def test_many_rows_of_real_workloads(oracle_mod):
    # The oracle's own routing of multi-row problems passes as it stands
    # (block path and strictly causal path); one planted row fails.
    from parity_util import check_causal_routing, dims_of
    w = Workload("rows", B=2, Hq=4, Hkv=2, d=16, T_hist=256, T_seg=256, k_c=2, k_g=5,
                 dtype="fp32", keys="clustered", seed=3)
    x = {k: v.astype(np.float64) for k, v in w.full().items()}
    dims = dims_of(w)
    orc = oracle_mod.route(dims, x["Q"], x["K"])
    check_block_routing(w, orc["cidx"], orc["gidx"], orc)
    rc = oracle_mod.causal_route(dims, x["Q"], orc["csum"], orc["gsum"])
    check_causal_routing(w, rc["cidx"], rc["gidx"], x["Q"], orc["csum"], orc["gsum"], rc)
    bad = rc["gidx"].copy()
    bad[1, 1, 200, 0] = bad[1, 1, 200, 1]                  # a duplicate: malformed
    with pytest.raises(AssertionError):
        check_causal_routing(w, rc["cidx"], bad, x["Q"], orc["csum"], orc["gsum"], rc)
