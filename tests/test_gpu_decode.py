"""Decode step on the GPU (hga_decode) against the oracle's decode
(article "BMW's 16 GB GPU just did what needs an A100", section
"Retrieval: no degradation in the dense baseline": HGA can generate too; the
token is a query block of one).

Gates as for the segment path: chunk / group indices equal to the oracle's
except on units whose oracle gap is below 1e-4; O and lse within 2e-3
(bf16) / 1e-4 (float32) max-abs.  On a unit whose routing differs inside
the exemption the GPU's O is checked against a direct float64 softmax over
the keys the GPU chose.

Rows of K / V after pos and summaries of chunks from pos // 64 on are NaN on
the GPU side: the kernel must never read them.
"""
import math

import numpy as np
import pytest
import torch

import hierarchical_routed_sparse_b200 as hga
from hierarchical_routed_sparse_b200 import workloads as W
from hierarchical_routed_sparse_b200.workloads import Workload

import oracle
from parity_util import GAP_EXEMPT, TOL, check_decode_routing, dims_of, maxabs, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup(oracle_mod):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_routed_sparse_b200 import build
    build.build()
    hga.load()


CASES = [
    Workload("dec_gqa4_bf16", B=2, Hq=8, Hkv=2, d=128, T_hist=448, T_seg=64, k_c=3, k_g=13,
             keys="clustered", seed=31),
    Workload("dec_fp32_d64", B=1, Hq=4, Hkv=2, d=64, T_hist=320, T_seg=64, k_c=2, k_g=9,
             dtype="fp32", keys="clustered", seed=32),
    Workload("dec_all_routing", B=1, Hq=4, Hkv=1, d=128, T_hist=192, T_seg=64, k_c=-1, k_g=-1, seed=33),
    Workload("dec_gqa8_bf16", B=1, Hq=16, Hkv=2, d=128, T_hist=256, T_seg=64, k_c=2, k_g=6,
             keys="clustered", seed=34),
    Workload("dec_mha_bf16_d64", B=1, Hq=3, Hkv=3, d=64, T_hist=192, T_seg=64, k_c=4, k_g=40, seed=35),
    Workload("dec_fp32_d128_k1", B=1, Hq=8, Hkv=2, d=128, T_hist=256, T_seg=64, k_c=1, k_g=1, dtype="fp32",
             keys="clustered", seed=36),
]
POSITIONS = [0, 5, 63, 64, 100, 127, 128, 250]


def _attend(q, K, V, grow, pos, scale):
    """float64 softmax attention of q [G][d] over the routed groups' tokens
    and the own chunk's tokens up to pos."""
    c0 = pos // 64
    keys = [8 * g + t for g in grow if g >= 0 for t in range(8)] + list(range(64 * c0, pos + 1))
    s = scale * (q @ K[keys].T)
    m = s.max(axis=1, keepdims=True)
    w = np.exp(s - m)
    l = w.sum(axis=1, keepdims=True)
    return (w / l) @ V[keys], (m + np.log(l))[:, 0]


def _run_decode(w, x, pos, nan_fill=True):
    p = hga.Params.from_workload(w)
    c0 = pos // 64
    K, V = to_dev(x["K"], w.dtype), to_dev(x["V"], w.dtype)
    st = hga.DecodeState(p)
    hga.build_summaries(p, K, 0, 64 * c0, st.csum, st.gsum)
    st.K.copy_(K)
    st.V.copy_(V)
    if nan_fill:
        st.K[:, :, pos + 1:] = float("nan")
        st.V[:, :, pos + 1:] = float("nan")
        st.csum[:, :, c0:] = float("nan")
        st.gsum[:, :, 8 * c0:] = float("nan")
    q = to_dev(np.ascontiguousarray(x["Q"][:, :, pos % w.T_seg]), w.dtype)
    hga.decode(p, pos, q, st.K, st.V, st.csum, st.gsum, st.O, st.lse, st.cidx, st.gidx)
    torch.cuda.synchronize()
    assert hga.device_status() == 0
    return {k: getattr(st, k).cpu().numpy() for k in ("O", "lse", "cidx", "gidx")}, q


def _compare(w, x, pos, got):
    dims = dims_of(w)
    K64, V64 = x["K"].astype(np.float64), x["V"].astype(np.float64)
    q64 = x["Q"][:, :, pos % w.T_seg].astype(np.float64)
    csum, gsum = oracle.build_summaries(dims, K64)
    orc = oracle.decode(dims, pos, q64, K64, V64, csum, gsum)
    check_decode_routing(w, pos, got["cidx"], got["gidx"], q64, csum, gsum, orc)
    tol = TOL[w.dtype]
    G, scale = w.G, 1.0 / math.sqrt(w.d)
    for b in range(w.B):
        for g in range(w.Hkv):
            hs = slice(g * G, (g + 1) * G)
            if np.array_equal(got["gidx"][b, g], orc["gidx"][b, g]):
                O_ref, lse_ref = orc["O"][b, hs], orc["lse"][b, hs]
            else:                                   # an exempt near-tie: the GPU's own choice
                O_ref, lse_ref = _attend(q64[b, hs], K64[b, g], V64[b, g], got["gidx"][b, g], pos, scale)
            assert maxabs(got["O"][b, hs], O_ref) <= tol, (b, g, maxabs(got["O"][b, hs], O_ref))
            assert maxabs(got["lse"][b, hs], lse_ref) <= tol, (b, g)
    return orc


@pytest.mark.parametrize("pos", POSITIONS)
@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_decode_matches_oracle(w, pos):
    x = w.full()
    got, _ = _run_decode(w, x, pos)
    orc = _compare(w, x, pos, got)
    if pos < 64:                                    # the first chunk: nothing to route
        assert (got["cidx"] == -1).all() and (got["gidx"] == -1).all()
    if pos == 0:                                    # one key: O is V[0] itself
        G = w.G
        for g in range(w.Hkv):
            np.testing.assert_array_equal(got["O"][:, g * G:(g + 1) * G],
                                          np.repeat(x["V"][:, g:g + 1, 0], G, axis=1))
    assert np.isfinite(got["O"]).all() and np.isfinite(orc["O"]).all()


def test_decode_last_position_of_the_cache():
    w = CASES[0]
    x = w.full()
    pos = w.T - 1
    got, _ = _run_decode(w, x, pos)
    _compare(w, x, pos, got)


@pytest.mark.parametrize("pos", [16383, 16320, 9000])
def test_decode_full_size_context(pos):
    # The 16K-context Qwen3-8B layer (32 q-heads, 8 kv-heads, d 128, k_c 8,
    # k_g 32): every (batch, kv-head) unit against the oracle.
    w = W.QWEN3_CTX16K_FWD
    x = w.full()
    got, _ = _run_decode(w, x, pos)
    _compare(w, x, pos, got)


def test_generation_appends_summaries():
    # DecodeState: prefill 100 rows, then generate 120 tokens; every step
    # equals the oracle's decode on the cache as it stands.  Crosses the
    # chunk boundaries at 128 and 192 (summaries appended by the state).
    w = CASES[0]
    x = w.full()
    p = hga.Params.from_workload(w)
    dims = dims_of(w)
    K64, V64 = x["K"].astype(np.float64), x["V"].astype(np.float64)
    csum, gsum = oracle.build_summaries(dims, K64)
    st = hga.DecodeState(p)
    n0 = 100
    st.prefill(to_dev(np.ascontiguousarray(x["K"][:, :, :n0]), w.dtype),
               to_dev(np.ascontiguousarray(x["V"][:, :, :n0]), w.dtype))
    rng = np.random.default_rng(5)
    Kd, Vd = to_dev(x["K"], w.dtype), to_dev(x["V"], w.dtype)
    for pos in range(n0, n0 + 120):
        q64 = rng.standard_normal((w.B, w.Hq, w.d))
        if w.dtype == "bf16":
            q64 = W.round_bf16(q64.astype(np.float32)).astype(np.float64)
        q = torch.from_numpy(q64.astype(np.float32)).to("cuda", p.torch_dtype)
        O = st.step(q, Kd[:, :, pos], Vd[:, :, pos]).cpu().numpy()
        orc = oracle.decode(dims, pos, q64, K64, V64, csum, gsum)
        cg = st.cidx.cpu().numpy()
        gg = st.gidx.cpu().numpy()
        check_decode_routing(w, pos, cg, gg, q64, csum, gsum, orc)
        if np.array_equal(gg, orc["gidx"]):
            assert maxabs(O, orc["O"]) <= TOL[w.dtype], pos
    assert st.pos == n0 + 120
    # The state's summaries of the complete chunks are those of the prefix.
    ref = hga.DecodeState(p)
    ref.prefill(Kd[:, :, :st.pos], Vd[:, :, :st.pos])
    torch.cuda.synchronize()
    full = 64 * (st.pos // 64)
    assert torch.equal(st.csum[:, :, :full // 64], ref.csum[:, :, :full // 64])
    assert torch.equal(st.gsum[:, :, :full // 8], ref.gsum[:, :, :full // 8])


def test_decode_rejects_bad_arguments():
    w = CASES[0]
    p = hga.Params.from_workload(w)
    st = hga.DecodeState(p)
    q = torch.zeros(w.B, w.Hq, w.d, device="cuda", dtype=p.torch_dtype)
    for pos in (-1, w.T):
        with pytest.raises(hga.HGAError) as e:
            hga.decode(p, pos, q, st.K, st.V, st.csum, st.gsum, st.O, st.lse, st.cidx, st.gidx)
        assert e.value.code == hga.HGA_ERR_INVALID_ARG
    # More than 8 q-heads per kv-head is refused before any launch.
    p9 = hga.Params(B=1, Hq=9, Hkv=1, d=128, T_hist=64, T_seg=64, k_c=2, k_g=4, dtype=hga.HGA_BF16)
    s9 = hga.DecodeState(p9)
    q9 = torch.zeros(1, 9, 128, device="cuda", dtype=torch.bfloat16)
    with pytest.raises(hga.HGAError) as e:
        hga.decode(p9, 10, q9, s9.K, s9.V, s9.csum, s9.gsum, s9.O, s9.lse, s9.cidx, s9.gidx)
    assert e.value.code == hga.HGA_ERR_UNSUPPORTED


@pytest.mark.parametrize("pos", [131071, 70000])
def test_decode_long_context_sampled_units(pos):
    # 128K context (2047 eligible chunks at the end: chunk selection over
    # shared memory, not registers), k_c 16, k_g 64; two (batch, kv-head)
    # units against the oracle.
    from parity_util import unit_slice
    w = W.sweep_point(131072, 16, 64).with_(B=1, backward=False)
    x = w.full()
    got, _ = _run_decode(w, x, pos)
    for g in (0, w.Hkv - 1):
        wu, xu = unit_slice(w, x, 0, g)
        _compare(wu, xu, pos, {k: v[:, g:g + 1] if k in ("cidx", "gidx") else v[:, g * w.G:(g + 1) * w.G]
                               for k, v in got.items()})
