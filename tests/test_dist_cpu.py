"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The hot path shards by independent problems, so the only cross-rank work is
timing: each rank gets its own seeded problem, durations are reduced with a
MAX over ranks, and the whole-job rate is all ranks' tokens over the
slowest rank's time.
"""
import os
import socket

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w_, _ = bench.dist_env()
        assert (r, w_) == (rank, world)
        mine = 10.0 + 5.0 * rank                      # rank 1 is the slow one
        m = bench.max_over_ranks(mine)
        wl = bench.rank_workload(bench.W.QWEN3_CTX16K_TRAIN.with_(T_hist=0, T_seg=128, Hq=4,
                                                                   Hkv=1), rank)
        q = wl.unit(0, 0)["Q"][0, :4, :4].tolist()
        out[rank] = (m, wl.seed, q)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_independent_problems():
    world, port = 2, _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 15.0             # both ranks see the max
    assert res[0][1] != res[1][1]                     # distinct seeds
    assert not np.allclose(res[0][2], res[1][2])      # distinct inputs
    rate = bench.whole_job_rate(2048, steps=10, world=2, max_ms=15.0)
    assert rate == 2 * 10 * 2048 / 0.015


def test_single_process_reduction_is_identity():
    assert bench.max_over_ranks(3.5) == 3.5
