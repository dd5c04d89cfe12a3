"""Helpers of the GPU parity tests: run the CUDA path through the C ABI and
the CPU oracle on the same seeded inputs, and compare under the gates.

Gates (method description: article "BMW's 16 GB GPU just did what needs an
A100", section "What HGA does differently"; gate values are those the
library is specified to):
  * routed chunk / group indices equal to the oracle's, except on rows where
    the oracle's gap between the k-th and (k+1)-th score is below 1e-4
    (relative); there the GPU's row must still be a valid choice;
  * O, LSE, dQ, dK, dV within 2e-3 max-abs for bf16 inputs (float32
    accumulation) and 1e-4 for float32 inputs.
Attention stages are compared with the ORACLE's routing fed to both sides
(the C ABI takes the indices as an input), so a near-tie that the GPU
resolves the other way cannot leak into the attention comparison.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import hierarchical_routed_sparse_b200 as hga
import oracle

GAP_EXEMPT = 1e-4
TOL = {"bf16": 2e-3, "fp32": 1e-4}


def dims_of(w, **kw) -> oracle.Dims:
    return oracle.Dims(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, T_hist=w.T_hist, T_seg=w.T_seg,
                       k_c=w.k_c, k_g=w.k_g, **kw)


def to_dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.to("cuda", torch.bfloat16 if dtype == "bf16" else torch.float32).contiguous()


def f64(x: dict) -> dict:
    return {k: v.astype(np.float64) for k, v in x.items()}


def unit_slice(w, x: dict, b: int, g: int) -> tuple:
    """Inputs of one (batch, kv-head) unit as a B=1, Hkv=1 problem."""
    G = w.G
    sl = dict(Q=x["Q"][b:b + 1, g * G:(g + 1) * G], K=x["K"][b:b + 1, g:g + 1],
              V=x["V"][b:b + 1, g:g + 1])
    if "dO" in x:
        sl["dO"] = x["dO"][b:b + 1, g * G:(g + 1) * G]
    return w.with_(B=1, Hq=G, Hkv=1), sl


def _format_ok(got: np.ndarray, what: str) -> None:
    """Every row ascending, unique and -1 padded."""
    for row in got.reshape(-1, got.shape[-1]):
        v = row[row >= 0]
        n = len(v)
        assert (row[n:] == -1).all() and (np.diff(v) > 0).all(), f"{what}: malformed row {row}"


def check_indices(got: np.ndarray, want: np.ndarray, gap: np.ndarray, what: str) -> int:
    """Exact equality except on rows whose oracle gap is below the exemption.

    Only the format of an exempt row is checked here; check_routing also
    proves that such a row is a valid top-k.  Returns the number of exempt
    rows that differ.
    """
    diff = (got != want).any(axis=-1)
    bad = diff & ~(gap < GAP_EXEMPT)
    assert not bad.any(), (f"{what}: {int(bad.sum())} rows differ outside the gap exemption; "
                           f"first at {np.argwhere(bad)[0].tolist()}: gpu {got[bad][0].tolist()} "
                           f"oracle {want[bad][0].tolist()} gap {gap[bad][0]}")
    _format_ok(got, what)
    return int((diff & (gap < GAP_EXEMPT)).sum())


def _band(s: np.ndarray, cand: np.ndarray, k: int):
    """For candidate scores s (float64) and a requested k (<= 0: all): the
    kept count, the reference top set (score descending, lower index first
    on ties), the k-th and (k+1)-th scores and the relative gap's
    denominator max(|s_k|, |s_k+1|, 1e-3 rms(s))."""
    n = len(cand)
    keep = n if (k <= 0 or k > n) else k
    order = np.lexsort((cand, -s))
    ref = np.sort(cand[order[:keep]])
    if keep == 0 or keep >= n:
        return keep, ref, None, None, None
    a, b = float(s[order[keep - 1]]), float(s[order[keep]])
    den = max(abs(a), abs(b), 1e-3 * math.sqrt(float(np.mean(s * s))))
    return keep, ref, a, b, den


def _valid_topk(row: np.ndarray, cand: np.ndarray, s: np.ndarray, k: int, what: str, where) -> bool:
    """Assert that `row` is one of the valid answers of a top-k among
    `cand` with scores `s`: it holds min(k, n) candidates, and every pick
    and every dropped reference pick lies within 1e-4 (relative, reading R8)
    of the boundary between the k-th and (k+1)-th scores.  Returns whether
    the row equals the reference top set exactly."""
    v = row[row >= 0]
    keep, ref, a, b, den = _band(s, cand, k)
    assert len(v) == keep, f"{what} {where}: {len(v)} entries, want min(k, eligible) = {keep}"
    pos = {int(c): i for i, c in enumerate(cand)}
    assert all(int(c) in pos for c in v), f"{what} {where}: {v.tolist()} not all eligible"
    if np.array_equal(v, ref):
        return True
    assert a is not None, f"{what} {where}: every candidate kept, yet the row differs"
    gap = (a - b) / den if den > 0 else 0.0
    assert gap < GAP_EXEMPT, f"{what} {where}: differs from the top set outside the gap ({gap:.3g})"
    eps = GAP_EXEMPT * den
    picked = np.array([s[pos[int(c)]] for c in v])
    assert picked.min() >= a - eps, f"{what} {where}: a pick scores {picked.min()} < s_k {a} - eps"
    dropped = np.setdiff1d(ref, v)
    if len(dropped):
        ds = np.array([s[pos[int(c)]] for c in dropped])
        assert ds.max() <= b + eps, f"{what} {where}: dropped {ds.max()} > s_k+1 {b} + eps"
    return False


def check_routing(got_c: np.ndarray, got_g: np.ndarray, q: np.ndarray, unit: np.ndarray,
                  csum: np.ndarray, gsum: np.ndarray, n_elig: np.ndarray, k_c: int, k_g: int,
                  what: str,
                  want_c: np.ndarray, cgap: np.ndarray, want_g: np.ndarray | None = None,
                  ggap: np.ndarray | None = None) -> dict:
    """Routing rows of the GPU against the oracle, under the index gate.

    Rows are flattened: got_c [N, wc], got_g [N, wg]; q [N, d] the row's
    block query (float64, the oracle's); unit [N] the row's flat (batch,
    kv-head) index into csum [U, nC, d] and gsum [U, nG, d]; n_elig [N] the
    eligible chunk count (the own chunk's index).
    A chunk row equals the oracle's exactly, or the oracle's gap is below
    1e-4 and the row is a valid top-k_c of the eligible chunks (count, range,
    scores within the tie band).  A group row is judged against the top-k_g
    of the groups of the GPU's OWN chunk row: want_g / ggap when given (the
    oracle's group routing run on the GPU's chunk rows), else recomputed
    from the scores.  Returns the counts of differing (exempt) rows.
    """
    N = int(np.prod(got_c.shape[:-1]))
    got_c, got_g = got_c.reshape(N, -1), got_g.reshape(N, -1)
    want_c, cgap = want_c.reshape(N, -1), cgap.reshape(N)
    _format_ok(got_c, what + " cidx")
    _format_ok(got_g, what + " gidx")
    gpc = 8
    out = {"cidx_exempt_rows": 0, "gidx_exempt_rows": 0}
    for i in range(N):
        crow = got_c[i][got_c[i] >= 0]
        if not np.array_equal(got_c[i], want_c[i]):
            assert cgap[i] < GAP_EXEMPT, (f"{what} cidx row {i}: gpu {got_c[i].tolist()} oracle "
                                          f"{want_c[i].tolist()} gap {cgap[i]}")
            cand = np.arange(int(n_elig[i]))
            s = csum[unit[i]][:len(cand)] @ q[i]
            _valid_topk(crow, cand, s, k_c, what + " cidx", i)
            out["cidx_exempt_rows"] += 1
        if want_g is not None and np.array_equal(got_g[i], want_g.reshape(N, -1)[i]):
            continue
        if want_g is not None:
            assert ggap.reshape(N)[i] < GAP_EXEMPT, (
                f"{what} gidx row {i}: gpu {got_g[i].tolist()} oracle "
                f"{want_g.reshape(N, -1)[i].tolist()} gap {ggap.reshape(N)[i]}")
        gcand = (crow[:, None] * gpc + np.arange(gpc)[None, :]).reshape(-1)
        s = gsum[unit[i]][gcand] @ q[i]
        grow = got_g[i][got_g[i] >= 0]
        if not _valid_topk(grow, gcand, s, k_g, what + " gidx", i):
            out["gidx_exempt_rows"] += 1
    return out


def block_rows(w, orc: dict, gpu_cidx: np.ndarray):
    """Flattened routing rows of the block path: for every (batch, kv-head,
    query block) the oracle's block query, its summaries and eligible chunk
    count, plus the oracle's group routing run on the GPU's chunk rows."""
    nQB = w.T_seg // 64
    N = w.B * w.Hkv * nQB
    q = orc["qbar"].reshape(N, w.d)
    unit = np.repeat(np.arange(w.B * w.Hkv), nQB)
    csum = orc["csum"].reshape(w.B * w.Hkv, -1, w.d)
    gsum = orc["gsum"].reshape(w.B * w.Hkv, -1, w.d)
    n_elig = np.tile(w.T_hist // 64 + np.arange(nQB), w.B * w.Hkv)
    want_g, ggap = oracle.route_groups(dims_of(w), orc["qbar"], orc["gsum"], gpu_cidx)
    return q, unit, csum, gsum, n_elig, want_g, ggap


def check_block_routing(w, gpu_cidx: np.ndarray, gpu_gidx: np.ndarray, orc: dict) -> dict:
    q, unit, csum, gsum, n_elig, want_g, ggap = block_rows(w, orc, gpu_cidx)
    return check_routing(gpu_cidx, gpu_gidx, q, unit, csum, gsum, n_elig, w.k_c, w.k_g, w.name,
                         orc["cidx"], orc["cgap"], want_g, ggap)


def maxabs(a, b) -> float:
    return float(np.abs(np.asarray(a, dtype=np.float64) - np.asarray(b, dtype=np.float64)).max())


def run_gpu(w, x: dict, gidx_in: np.ndarray | None = None, full_summaries: bool = True):
    """Run the hot path on the GPU.  Returns numpy copies of every output.

    gidx_in: routing fed to the attention stages (oracle's); the GPU's own
    routing is still computed and returned.
    """
    p = hga.Params.from_workload(w)
    buf = hga.Buffers(p)
    Q, K, V = to_dev(x["Q"], w.dtype), to_dev(x["K"], w.dtype), to_dev(x["V"], w.dtype)
    if full_summaries:
        buf.summaries(K, 0, w.T)
    else:  # history first, then the segment's own keys appended
        buf.summaries(K, 0, w.T_hist)
        buf.summaries(K, w.T_hist, w.T)
    buf.route(Q)
    gidx = buf.gidx if gidx_in is None else torch.from_numpy(gidx_in).to("cuda")
    buf.forward(Q, K, V, gidx=gidx)
    out = {}
    if "dO" in x:
        dO = to_dev(x["dO"], w.dtype)
        buf.backward(Q, K, V, dO, gidx=gidx)
        out.update(dQ=buf.dQ, dK=buf.dK, dV=buf.dV)
    torch.cuda.synchronize()
    assert hga.device_status() == 0, "a kernel's bounded wait ran out"
    out.update(csum=buf.csum, gsum=buf.gsum, qbar=buf.qbar, cidx=buf.cidx, gidx=buf.gidx,
               O=buf.O, lse=buf.lse)
    return {k: v.cpu().numpy() for k, v in out.items()}, buf


def run_oracle(w, x64: dict, backward: bool):
    dims = dims_of(w)
    r = oracle.route(dims, x64["Q"], x64["K"])
    O, lse = oracle.attn_fwd(dims, x64["Q"], x64["K"], x64["V"], r["gidx"])
    r.update(O=O, lse=lse)
    if backward:
        r["dQ"], r["dK"], r["dV"] = oracle.attn_bwd(dims, x64["Q"], x64["K"], x64["V"], x64["dO"],
                                                    r["gidx"])
    return r


def compare_all(w, gpu: dict, orc: dict, gpu_routed: dict | None = None) -> dict:
    """Assert every gate; returns the measured errors."""
    tol = TOL[w.dtype]
    errs = {}
    errs["csum"] = maxabs(gpu["csum"], orc["csum"])
    errs["gsum"] = maxabs(gpu["gsum"], orc["gsum"])
    errs["qbar"] = maxabs(gpu["qbar"], orc["qbar"])
    assert errs["csum"] < 1e-5 and errs["gsum"] < 1e-5 and errs["qbar"] < 1e-5, errs
    errs.update(check_block_routing(w, gpu["cidx"], gpu["gidx"], orc))
    for k in ("O", "lse", "dQ", "dK", "dV"):
        if k in gpu:
            errs[k] = maxabs(gpu[k], orc[k])
            assert errs[k] <= tol, f"{k}: max-abs error {errs[k]:.3g} > {tol}"
    return errs


def check_causal_routing(w, got_c: np.ndarray, got_g: np.ndarray, Q64: np.ndarray,
                         csum: np.ndarray, gsum: np.ndarray, orc: dict) -> dict:
    """Routing rows of the strictly causal variant (one per query position):
    the row's query is the mean of its G q-heads' queries at that position
    and chunks before the position's own chunk are eligible.  Group rows are
    judged on the GPU's own chunk rows."""
    B, Hkv, Ts, d, G = w.B, w.Hkv, w.T_seg, w.d, w.G
    q = Q64.reshape(B, Hkv, G, Ts, d).mean(axis=2).reshape(-1, d)
    unit = np.repeat(np.arange(B * Hkv), Ts)
    n_elig = np.tile((w.T_hist + np.arange(Ts)) // 64, B * Hkv)
    return check_routing(got_c, got_g, q, unit, csum.reshape(B * Hkv, -1, d),
                         gsum.reshape(B * Hkv, -1, d), n_elig, w.k_c, w.k_g, w.name + " causal",
                         orc["cidx"], orc["cgap"])


def check_decode_routing(w, pos: int, got_c: np.ndarray, got_g: np.ndarray, q64: np.ndarray,
                         csum: np.ndarray, gsum: np.ndarray, orc: dict) -> dict:
    """Routing rows of one decode step (a block of one at position pos)."""
    B, Hkv, d, G = w.B, w.Hkv, w.d, w.G
    q = q64.reshape(B, Hkv, G, d).mean(axis=2).reshape(-1, d)
    unit = np.arange(B * Hkv)
    n_elig = np.full(B * Hkv, pos // 64)
    return check_routing(got_c, got_g, q, unit, csum.reshape(B * Hkv, -1, d),
                         gsum.reshape(B * Hkv, -1, d), n_elig, w.k_c, w.k_g,
                         f"{w.name} decode@{pos}", orc["cidx"], orc["cgap"])
