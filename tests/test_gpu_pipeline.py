"""StepPipeline: segment steps from host memory with the copies overlapped
(uploads of step i+1 and downloads of step i-1 on their own streams while
step i computes, two device buffer sets).  Every step's host results must be
those of a plain Buffers.step on the same inputs: dQ bit for bit (same
kernels, same order), dK / dV up to the order of their float32 atomics.
"""
import numpy as np
import pytest
import torch

import hierarchical_routed_sparse_b200 as hga
from hierarchical_routed_sparse_b200.workloads import Workload

from parity_util import maxabs, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup(oracle_mod):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from hierarchical_routed_sparse_b200 import build
    build.build()
    hga.load()


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_pipeline_equals_plain_steps(dtype):
    base = Workload("pipe", B=2, Hq=8, Hkv=2, d=128 if dtype == "bf16" else 64, T_hist=512, T_seg=256, k_c=3,
                    k_g=13, dtype=dtype, keys="clustered", backward=True, seed=51)
    p = hga.Params.from_workload(base)
    tdt = p.torch_dtype
    # Five steps over three different segments (same history).
    inputs = [base.with_(seed=51 + k).full() for k in range(3)]
    hist = inputs[0]
    Kd = to_dev(hist["K"], dtype)
    Vd = to_dev(hist["V"], dtype)
    pipe = hga.StepPipeline(p, Kd[:, :, :base.T_hist], Vd[:, :, :base.T_hist])
    order = [0, 1, 2, 1, 0]
    host_in, host_out = [], []
    for k in order:
        x = inputs[k]
        seg = slice(base.T_hist, base.T)
        hi = [torch.from_numpy(np.ascontiguousarray(a)).to(tdt).pin_memory()
              for a in (x["Q"], x["K"][:, :, seg], x["V"][:, :, seg], x["dO"])]
        ho = [torch.empty(s, dtype=torch.float32).pin_memory() for s in
              ((p.B, p.Hq, p.T_seg, p.d), (p.B, p.Hkv, p.T_seg, p.d), (p.B, p.Hkv, p.T_seg, p.d))]
        host_in.append(hi)
        host_out.append(ho)
        pipe.submit(*hi, ho)
    pipe.synchronize()
    torch.cuda.synchronize()
    assert hga.device_status() == 0
    for (hi, ho) in zip(host_in, host_out):
        Q, Ks, Vs, dO = (t.cuda() for t in hi)
        K, V = Kd.clone(), Vd.clone()
        K[:, :, base.T_hist:] = Ks
        V[:, :, base.T_hist:] = Vs
        buf = hga.Buffers(p)
        buf.summaries(K, 0, base.T_hist)
        buf.step(Q, K, V, dO)
        torch.cuda.synchronize()
        assert torch.equal(ho[0], buf.dQ.cpu())
        assert maxabs(ho[1], buf.dK.cpu()) <= 1e-5
        assert maxabs(ho[2], buf.dV.cpu()) <= 1e-5
