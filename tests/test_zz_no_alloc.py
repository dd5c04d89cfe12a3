"""hga_attn_bwd_noalloc against hga_attn_bwd, on the GPU.

hga_attn_bwd_noalloc serves callers that cannot hand the library scratch
memory (plugin interfaces that pass an operator only its inputs and outputs,
hosts whose memory pool owns all device memory, loops that must not call
cudaMalloc / cudaFree).  It keeps its scratch in a fixed array inside the
library.  Its results must match the workspace entry point's within the
parity tolerance, call after call: the array keeps the previous call's
contents, so between the two compared calls another problem (a different
upstream gradient, then another head layout whose item schedule sits at a
different offset) leaves different row sums and a different schedule in it,
and the second call must overwrite every entry it reads.

The file name sorts last so that a run stopping at the first failure has
already run every other test.
"""
import numpy as np
import pytest
import torch

import hierarchical_routed_sparse_b200 as hga
from hierarchical_routed_sparse_b200 import workloads as W
from hierarchical_routed_sparse_b200.workloads import Workload

pytestmark = pytest.mark.gpu

TOL = {"bf16": 2e-3, "fp32": 1e-4}


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_routed_sparse_b200 import build
    build.build()
    hga.load()


def _dev(x, dtype):
    return torch.from_numpy(x).to("cuda", torch.bfloat16 if dtype == "bf16" else torch.float32)


CASES = [
    Workload("noalloc_gqa_bf16", B=2, Hq=8, Hkv=2, d=128, T_hist=512, T_seg=512, k_c=3, k_g=13,
             keys="clustered", backward=True, seed=21),
    Workload("noalloc_fp32_d64", B=1, Hq=4, Hkv=2, d=64, T_hist=256, T_seg=256, k_c=2, k_g=9,
             dtype="fp32", backward=True, seed=22),
    W.QWEN3_CTX16K_TRAIN,
    # 2048 backward items, 14 a CTA: the round-robin schedule (262144 rows)
    Workload("noalloc_round_robin", B=2, Hq=32, Hkv=8, d=128, T_hist=2048, T_seg=4096, k_c=4,
             k_g=16, keys="clustered", backward=True, seed=23),
]

# The problem run between the two compared calls: G = 3 (a pair with one
# head) and another row count, so its row sums and schedule land elsewhere.
OTHER = Workload("noalloc_other", B=1, Hq=6, Hkv=2, d=128, T_hist=1024, T_seg=640, k_c=4, k_g=17,
                 keys="clustered", backward=True, seed=24)


def _other_problem_call():
    x = OTHER.full()
    p = hga.Params.from_workload(OTHER)
    Q, K, V, dO = (_dev(x[k], OTHER.dtype) for k in ("Q", "K", "V", "dO"))
    b = hga.Buffers(p)
    b.summaries(K, 0, OTHER.T)
    b.route(Q)
    b.forward(Q, K, V)
    hga.attn_bwd_noalloc(p, Q, K, V, b.O, b.lse, dO, b.gidx, b.dQ, b.dK, b.dV)
    torch.cuda.synchronize()


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_matches_workspace_backward_twice(w):
    x = w.full()
    p = hga.Params.from_workload(w)
    Q, K, V, dO = (_dev(x[k], w.dtype) for k in ("Q", "K", "V", "dO"))
    buf = hga.Buffers(p)
    buf.summaries(K, 0, w.T)
    buf.route(Q)
    buf.forward(Q, K, V)
    buf.backward(Q, K, V, dO)            # the entry point with a caller workspace
    torch.cuda.synchronize()
    ref = [t.cpu().numpy() for t in (buf.dQ, buf.dK, buf.dV)]
    for call in range(2):
        if call == 1:
            # Same problem, another dO: different row sums in the same slots.
            dO2 = _dev(np.ascontiguousarray(x["dO"][..., ::-1]), w.dtype)
            junk = [torch.empty_like(t) for t in (buf.dQ, buf.dK, buf.dV)]
            hga.attn_bwd_noalloc(p, Q, K, V, buf.O, buf.lse, dO2, buf.gidx, *junk)
            _other_problem_call()
        outs = [torch.full_like(t, float("nan")) for t in (buf.dQ, buf.dK, buf.dV)]
        hga.attn_bwd_noalloc(p, Q, K, V, buf.O, buf.lse, dO, buf.gidx, *outs)
        torch.cuda.synchronize()
        for name, got, want in zip(("dQ", "dK", "dV"), outs, ref):
            err = float(np.abs(got.cpu().numpy() - want).max())
            assert err <= TOL[w.dtype], (w.name, call, name, err)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # B*Hq*T_seg = 2 * 32 * 32768 = 2^21 rows: refused on the host, nothing
    # launched (the pointers below are never dereferenced).
    p = hga.Params(B=2, Hq=32, Hkv=8, d=128, T_hist=0, T_seg=32768, k_c=8, k_g=32)
    assert p.B * p.Hq * p.T_seg > hga.NOALLOC_MAX_ROWS
    z = torch.zeros(64, device="cuda")
    with pytest.raises(hga.HGAError) as ei:
        hga.attn_bwd_noalloc(p, z, z, z, z, z, z, z.int(), z, z, z)
    assert ei.value.code == hga.HGA_ERR_INVALID_ARG
    assert "built-in scratch" in str(ei.value)
