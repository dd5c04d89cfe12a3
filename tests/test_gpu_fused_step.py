"""The fused segment step's routing and forward (hga_route_attn_fwd), on the GPU.

One persistent launch routes each query block and runs the forward of its
q-head pairs (article "BMW's 16 GB GPU just did what needs an A100",
section "What HGA does differently": HGA as a drop-in module run segment by
segment).  Its results must equal those of hga_route followed by
hga_attn_fwd bit for bit: the routing runs the router's own steps, and the
forward's tile is the same code on the same routing row.  One case is also
compared with the oracle under the parity gates.
"""
import numpy as np
import pytest
import torch

import hierarchical_routed_sparse_b200 as hga
from hierarchical_routed_sparse_b200 import workloads as W
from hierarchical_routed_sparse_b200.workloads import Workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_routed_sparse_b200 import build
    build.build()
    hga.load()


CASES = [
    W.QWEN3_CTX16K_TRAIN,                                              # 256 blocks, 2 head pairs each
    Workload("fused_odd_heads", B=2, Hq=6, Hkv=2, d=128, T_hist=1024, T_seg=640, k_c=4, k_g=17,
             keys="clustered", seed=61),                                 # G 3: a pair with one head
    Workload("fused_d64", B=1, Hq=8, Hkv=2, d=64, T_hist=512, T_seg=384, k_c=3, k_g=13,
             keys="clustered", seed=62),
    Workload("fused_no_history", B=1, Hq=4, Hkv=1, d=128, T_hist=0, T_seg=512, k_c=2, k_g=9, seed=63),
    Workload("fused_all_routing", B=1, Hq=4, Hkv=2, d=128, T_hist=256, T_seg=256, k_c=-1, k_g=-1,
             seed=64),
    Workload("fused_more_blocks_than_ctas", B=2, Hq=32, Hkv=8, d=128, T_hist=2048, T_seg=2048, k_c=4,
             k_g=16, keys="clustered", seed=65),                         # 512 blocks: CTAs take several
    Workload("fused_fp32", B=1, Hq=4, Hkv=2, d=64, T_hist=256, T_seg=192, k_c=2, k_g=9, dtype="fp32",
             seed=66),                                                   # two launches
]


def _run(w, fused: bool):
    x = w.full()
    p = hga.Params.from_workload(w)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    Q, K, V = (torch.from_numpy(x[k]).to("cuda", dt) for k in ("Q", "K", "V"))
    buf = hga.Buffers(p)
    for t in (buf.qbar, buf.O, buf.lse):
        t.fill_(float("nan"))
    buf.cidx.fill_(-7)
    buf.gidx.fill_(-7)
    buf.summaries(K, 0, w.T)
    if fused:
        buf.route_forward(Q, K, V)
    else:
        buf.route(Q)
        buf.forward(Q, K, V)
    torch.cuda.synchronize()
    assert hga.device_status() == 0
    return {k: getattr(buf, k).cpu().numpy() for k in ("qbar", "cidx", "gidx", "O", "lse")}


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_fused_equals_separate_launches(w):
    a, b = _run(w, True), _run(w, False)
    for k in ("cidx", "gidx"):
        assert np.array_equal(a[k], b[k]), k
    for k in ("qbar", "O", "lse"):
        assert np.array_equal(a[k].view(np.uint32), b[k].view(np.uint32)), k


def test_fused_matches_oracle():
    import oracle
    from parity_util import TOL, dims_of, f64, maxabs
    w = CASES[1]
    x = w.full()
    got = _run(w, True)
    x64 = f64(x)
    dims = dims_of(w)
    from parity_util import check_block_routing
    check_block_routing(w, got["cidx"], got["gidx"], oracle.route(dims, x64["Q"], x64["K"]))
    # The attention on the GPU's routing against the oracle's on the same rows.
    O, lse = oracle.attn_fwd(dims, x64["Q"], x64["K"], x64["V"], got["gidx"])
    assert maxabs(got["O"], O) <= TOL[w.dtype]
    assert maxabs(got["lse"], lse) <= TOL[w.dtype]
