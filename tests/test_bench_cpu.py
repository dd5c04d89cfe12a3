"""CPU checks of the benchmark's algorithmic work per launch, the figures
the roofline fractions divide by.

Expected values are closed forms worked out by hand from the key counts:
query i of a block attends 8 * n_g routed keys plus i + 1 keys of its own
chunk, where n_g = min(k_g, 8 * min(k_c, eligible chunks)); the forward
costs 4 * d FLOPs per (q-head, query, key) and the backward 10 * d.
"""
import importlib.util
import os

import pytest

from hierarchical_routed_sparse_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_16k_training_step(bench):
    a = bench.algorithmic(W.QWEN3_CTX16K_TRAIN)
    # Every block has 224 + qb >= 8 eligible chunks, so n_g = 32 everywhere:
    # per q-head 2048 * 256 routed pairs + 32 blocks * (1 + ... + 64) own-chunk
    # pairs = 524288 + 66560 = 590848.
    pairs = 2048 * 256 + 32 * 2080
    assert a["attn_fwd"]["flops"] == 4 * 128 * 32 * pairs == 9_680_453_632
    assert a["attn_bwd"]["flops"] == 10 * 128 * 32 * pairs
    # Forward bytes: Q (bf16) + K and V gathered once per (kv-head, block),
    # 256 routed + 64 own tokens + O and LSE (float32) + the index rows.
    q = 32 * 2048 * 128 * 2
    kv = 8 * 32 * (256 + 64) * 128 * 2 * 2
    o, lse, gidx = 32 * 2048 * 128 * 4, 32 * 2048 * 4, 8 * 32 * 32 * 4
    assert a["attn_fwd"]["bytes"] == q + kv + o + lse + gidx == 92_569_600
    # Backward: Q, gathered K / V, dO, O, LSE, D written and read, dQ, and
    # the segment keys' dK / dV (float32), plus the index rows.
    seg = 2 * 8 * 2048 * 128 * 4
    assert a["attn_bwd"]["bytes"] == q + kv + q + o + lse + 2 * lse + o + seg + gidx
    # Segment summaries: the 2048 new keys of 8 kv-heads read once, 32 chunk
    # and 256 group rows written.
    assert a["summaries"]["bytes"] == 8 * 2048 * 128 * 2 + 8 * (32 + 256) * 128 * 4


def test_no_history_early_blocks_route_fewer_groups(bench):
    a = bench.algorithmic(W.QWEN3_T2K_FWD)
    # Block qb has qb eligible chunks: n_g = 0, 8, 16, 24 for qb = 0..3 and
    # 32 from qb = 4 on, so the routed groups total 48 + 28 * 32 = 944.
    pairs = 64 * 8 * 944 + 32 * 2080
    assert a["attn_fwd"]["flops"] == 4 * 128 * 32 * pairs == 9_009_364_992
    kv = 8 * (944 * 8 + 32 * 64) * 128 * 2 * 2
    q, o, lse, gidx = 32 * 2048 * 128 * 2, 32 * 2048 * 128 * 4, 32 * 2048 * 4, 8 * 32 * 32 * 4
    assert a["attn_fwd"]["bytes"] == q + kv + o + lse + gidx


@pytest.mark.parametrize("k_g", [32, 64])
def test_sweep_work_is_constant_in_context(bench, k_g):
    # With at least k_c history chunks the routed key count per query does
    # not depend on T: the attention work of the sweep points is equal.
    works = [bench.algorithmic(W.BY_NAME[f"sweep_B4_ctx{T}_kc{8 if k_g == 32 else 16}_kg{k_g}"])
             for T in (32768, 65536, 131072)]
    for stage in ("attn_fwd", "attn_bwd"):
        assert len({(x[stage]["bytes"], x[stage]["flops"]) for x in works}) == 1
    pairs = 2048 * 8 * k_g + 32 * 2080
    assert works[0]["attn_fwd"]["flops"] == 4 * 128 * 4 * 32 * pairs


def test_router_bytes_count_each_byte_once(bench):
    # 16K step: Q (bf16) read once; the 256 chunk summaries of each of the
    # 8 kv-heads read once; per block the 8 groups of each of the 8 chosen
    # chunks gathered; qbar (128 floats) and the index rows written and read
    # back: 16.8 + 1.0 + 8.4 MB plus the small terms, about 26.6 MB.
    a = bench.algorithmic(W.QWEN3_CTX16K_TRAIN)
    q = 32 * 2048 * 128 * 2
    csum = 8 * 256 * 128 * 4
    blocks = 8 * 32
    rc = q + csum + blocks * (128 * 4 + 8 * 4)
    rg = blocks * (128 * 4 + 8 * 4 + 8 * 8 * 128 * 4 + 32 * 4)
    assert a["route_chunks"]["bytes"] == rc
    assert a["route_groups"]["bytes"] == rg
    assert 26.5e6 < rc + rg < 26.7e6
    # Per use, block qb reads its 224 + qb eligible chunk summaries.
    per_use = q + 8 * sum(224 + qb for qb in range(32)) * 128 * 4 + blocks * (128 * 4 + 8 * 4)
    assert a["route_chunks"]["per_use_bytes"] == per_use
