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


def check_indices(got: np.ndarray, want: np.ndarray, gap: np.ndarray, what: str) -> int:
    """Exact equality except on rows whose oracle gap is below the exemption.

    Returns the number of exempt rows that differ.
    """
    diff = (got != want).any(axis=-1)
    bad = diff & ~(gap < GAP_EXEMPT)
    assert not bad.any(), (f"{what}: {int(bad.sum())} rows differ outside the gap exemption; "
                           f"first at {np.argwhere(bad)[0].tolist()}: gpu {got[bad][0].tolist()} "
                           f"oracle {want[bad][0].tolist()} gap {gap[bad][0]}")
    # Every row, exempt or not, must still be ascending, unique and -1 padded.
    for row in got.reshape(-1, got.shape[-1]):
        v = row[row >= 0]
        n = len(v)
        assert (row[n:] == -1).all() and (np.diff(v) > 0).all(), f"{what}: malformed row {row}"
    return int((diff & (gap < GAP_EXEMPT)).sum())


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
    errs["cidx_exempt_rows"] = check_indices(gpu["cidx"], orc["cidx"], orc["cgap"], "cidx")
    # Group routing is compared on the rows whose chunk choice agrees (a
    # different, exempt chunk choice gives different candidates).
    same_c = (gpu["cidx"] == orc["cidx"]).all(axis=-1)
    ggap = np.where(same_c, orc["ggap"], 0.0)
    errs["gidx_exempt_rows"] = check_indices(gpu["gidx"], orc["gidx"], ggap, "gidx")
    for k in ("O", "lse", "dQ", "dK", "dV"):
        if k in gpu:
            errs[k] = maxabs(gpu[k], orc[k])
            assert errs[k] <= tol, f"{k}: max-abs error {errs[k]:.3g} > {tol}"
    return errs
