"""The backward's item schedule (bf16 tensor-core path, d 64 and 128), on the GPU.

The row-dot launch of hga_attn_bwd writes, after the row sums in the
workspace, the order in which the persistent backward's G CTAs take the
work items (one per batch, kv-head, query block and pair of q-heads):
CTA c's k-th item is sched[k * G + c].  Checked here from the workspace
after a backward call, against the routing the call used:
  * the schedule is a permutation of the items and CTA c takes as many
    items as round-robin would give it (ceil((n - c) / G));
  * when a CTA takes at most 4 items (R <= 4), items are ranked by
    estimated cost (key tiles plus segment tiles of their index row) and the
    heaviest go to the CTAs that take one item fewer: no item of a CTA with
    R items costs more than any item of a CTA with R - 1 items;
  * with more items a CTA, the schedule is round-robin (the identity).
The gradients themselves are the parity tests' subject.
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
    W.QWEN3_CTX16K_TRAIN,                                            # 512 items on the SMs
    Workload("sched_odd_heads", B=2, Hq=6, Hkv=2, d=128, T_hist=1024, T_seg=640, k_c=4, k_g=17,
             keys="clustered", backward=True, seed=41),                # G 3: a pair with one head
    Workload("sched_few_items", B=1, Hq=4, Hkv=2, d=128, T_hist=256, T_seg=256, k_c=2, k_g=9,
             backward=True, seed=42),                                  # fewer items than SMs
    Workload("sched_wide_rows", B=1, Hq=32, Hkv=8, d=128, T_hist=8192, T_seg=2048, k_c=4, k_g=19,
             keys="clustered", backward=True, seed=43),                # wg not a multiple of 4
    Workload("sched_many_items", B=2, Hq=32, Hkv=8, d=128, T_hist=2048, T_seg=4096, k_c=4, k_g=16,
             keys="clustered", backward=True, seed=44),                # 2048 items: round-robin
    # d = 64 runs on the same tensor-core kernel (only it writes a schedule)
    Workload("sched_d64", B=1, Hq=4, Hkv=2, d=64, T_hist=512, T_seg=256, k_c=3, k_g=13,
             keys="clustered", backward=True, seed=45),
]


def _cost(row: np.ndarray, T_hist: int) -> int:
    """Key tiles plus segment tiles of one index row (ascending groups, -1 padding)."""
    valid = row[row >= 0]
    n_g, c_hist = len(valid), int((valid < T_hist // 8).sum())
    n_rt = (n_g + 7) // 8
    n_seg = n_rt - c_hist // 8 + 1 if c_hist < n_g else 1
    return min(n_rt + 1 + n_seg, 63)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_schedule_is_a_balanced_permutation(w):
    x = w.full()
    p = hga.Params.from_workload(w)
    Q, K, V, dO = (torch.from_numpy(x[k]).to("cuda", torch.bfloat16) for k in ("Q", "K", "V", "dO"))
    buf = hga.Buffers(p)
    buf.summaries(K, 0, w.T)
    buf.route(Q)
    buf.forward(Q, K, V)
    buf.ws.fill_(float("nan"))
    buf.backward(Q, K, V, dO)
    torch.cuda.synchronize()
    assert hga.device_status() == 0
    rows = w.B * w.Hq * w.T_seg
    G_heads = w.Hq // w.Hkv
    n_pairs = (G_heads + 1) // 2
    n = w.B * w.Hkv * (w.T_seg // 64) * n_pairs
    sched = buf.ws.view(torch.int32)[rows:rows + n].cpu().numpy()
    assert sorted(sched.tolist()) == list(range(n))
    G = min(n, torch.cuda.get_device_properties(0).multi_processor_count)
    if (n + G - 1) // G > 4:
        assert np.array_equal(sched, np.arange(n)), w.name
        return
    gidx = buf.gidx.cpu().numpy().reshape(-1, buf.gidx.shape[-1])
    cost = np.array([_cost(gidx[i // n_pairs], w.T_hist) for i in range(n)])
    R = (n + G - 1) // G
    E = n - (R - 1) * G                                   # CTAs 0 .. E-1 take R items
    long_items, short_items = [], []
    for c in range(G):
        n_mine = (n - c + G - 1) // G
        assert n_mine == (R if c < E else R - 1)
        mine = [int(sched[k * G + c]) for k in range(n_mine)]
        (long_items if c < E else short_items).extend(mine)
    assert len(long_items) + len(short_items) == n
    if short_items and long_items:
        assert cost[long_items].max() <= cost[short_items].min(), (w.name, cost[long_items].max(),
                                                                    cost[short_items].min())
