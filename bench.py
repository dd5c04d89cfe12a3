#!/usr/bin/env python
"""Benchmark of the HGA segment training step on B200.

One step is one pass of the whole hot path over one segment: the summaries
of the segment's 2048 new keys (history summaries persist from earlier
segments), block queries + chunk routing, group routing, the routed
attention forward and its backward.  The metric is segment tokens per second
(B * T_seg per step), measured on the device with CUDA events; inputs are
resident in HBM and L2 is flushed (a 256 MiB write) between timed steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the CPU oracle, same metric

Under torchrun each rank runs its own independent problem (weak scaling;
the hot path has no exchange step) and rank 0 prints one JSON line with the
whole-job value: all ranks' tokens over the slowest rank's time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hierarchical_routed_sparse_b200 import workloads as W  # noqa: E402

METRIC = "HGA routed-attention fwd+bwd tokens/s at 16K ctx; % of roofline (TFLOP/s or HBM GB/s)"
DEFAULT_WORKLOAD = W.QWEN3_CTX16K_TRAIN.name
L2_FLUSH_BYTES = 256 << 20
# Kernels of this library launched per step: segment summaries, fused
# chunk+group router, attention forward, and with a backward the row-dot
# (which also zeroes dK/dV) and the attention backward.
LAUNCHES_FWD = 3
LAUNCHES_BWD = 2


def peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        return dict(hbm_gbs=m["hbm_gbs"], bf16_tflops=m["bf16_tflops"],
                    bf16_tflops_sustained=m["bf16_tflops_sustained"], source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                source="fallback")


# ---- algorithmic work (bytes and FLOPs a perfect kernel must move / do) -----
def routed_groups(w, qb: int) -> int:
    """Groups routed for query block qb: min(k_g, 8 * min(k_c, eligible))."""
    c0 = w.T_hist // 64 + qb
    nc = c0 if w.k_c <= 0 else min(w.k_c, c0)
    return 8 * nc if w.k_g <= 0 else min(w.k_g, 8 * nc)


def algorithmic(w) -> dict:
    """Per-launch algorithmic bytes and FLOPs of each stage of one step."""
    el = 2 if w.dtype == "bf16" else 4
    B, Hq, Hkv, d, Ts, G = w.B, w.Hq, w.Hkv, w.d, w.T_seg, w.G
    nQB = Ts // 64
    ng = [routed_groups(w, qb) for qb in range(nQB)]
    # Keys per (q-head, query): 8*n_g routed + (i+1) own-chunk keys.
    key_pairs = sum(64 * 8 * n + 64 * 65 // 2 for n in ng)            # per q-head
    kv_tokens = sum(8 * n + 64 for n in ng)                            # per kv-head
    wc = w.k_c if w.k_c > 0 else w.T // 64
    wg = w.k_g if w.k_g > 0 else 8 * wc
    q_bytes = B * Hq * Ts * d * el
    kv_gather = B * Hkv * kv_tokens * d * el * 2
    o_bytes = B * Hq * Ts * d * 4
    lse_bytes = B * Hq * Ts * 4
    gidx_bytes = B * Hkv * nQB * wg * 4
    fwd_bytes = q_bytes + kv_gather + o_bytes + lse_bytes + gidx_bytes
    bwd_bytes = (q_bytes + kv_gather + q_bytes            # Q, K/V gathered, dO
                 + o_bytes + lse_bytes + 2 * lse_bytes     # O, LSE, D written + read
                 + o_bytes                                 # dQ
                 + 2 * B * Hkv * Ts * d * 4                # dK_seg, dV_seg
                 + gidx_bytes)
    seg_keys = B * Hkv * Ts * d * el
    summ_bytes = seg_keys + B * Hkv * (Ts // 64 + Ts // 8) * d * 4
    # Routers: the block query reads all of Q; chunk routing reads the
    # context's chunk summaries (each once per (batch, kv-head)); group
    # routing gathers the 8 group summaries of each chosen chunk per block;
    # plus qbar and the index rows written and read back.  The per-use
    # figure instead counts every block's own read of its eligible chunk
    # summaries (most of them served by L2).
    n_chunks = w.T // 64
    csum_once = B * Hkv * n_chunks * d * 4
    csum_per_use = B * Hkv * sum(w.T_hist // 64 + qb for qb in range(nQB)) * d * 4
    small = B * Hkv * nQB * (d * 4 + wc * 4)                           # qbar and cidx written
    rc_bytes = q_bytes + csum_once + small
    rg_bytes = B * Hkv * nQB * (d * 4 + wc * 4 + 8 * wc * d * 4 + wg * 4)
    return dict(
        attn_fwd=dict(bytes=fwd_bytes, flops=4.0 * d * B * Hq * key_pairs),
        attn_bwd=dict(bytes=bwd_bytes, flops=10.0 * d * B * Hq * key_pairs),
        summaries=dict(bytes=summ_bytes, flops=0.0),
        route_chunks=dict(bytes=rc_bytes, flops=0.0,
                          per_use_bytes=q_bytes + csum_per_use + small),
        route_groups=dict(bytes=rg_bytes, flops=0.0),
    )


# Source files of each timed kernel: a recorded ncu traffic figure is used
# only while these files are unchanged since the capture.
KERNEL_SOURCES = {
    "attn_fwd": ["attn_tc_fwd.cu", "sm100.cuh", "hga_internal.cuh"],
    "attn_bwd": ["attn_tc_bwd.cu", "sm100.cuh", "hga_internal.cuh"],
    "attn_bwd_causal": ["attn_tc_bwd.cu", "window_union.cuh", "sm100.cuh", "hga_internal.cuh"],
}


def kernel_source_hash(kernel: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "hierarchical_routed_sparse_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def recorded_traffic(kernel: str, w) -> float | None:
    """DRAM bytes per launch from profiles/traffic.json, if still current."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec or rec.get("workload") != w.name or rec.get("source_sha256") != kernel_source_hash(kernel):
        return None
    return float(rec["dram_bytes_per_launch"])


# ---- clocks sampled during the timed region -----------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, out_path: str | None = None):
        self.gpu = gpu_index
        self.proc = None
        self.out_path = out_path

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            out, _ = self.proc.communicate(timeout=10)
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
            if self.out_path:
                with open(self.out_path, "w") as f:
                    f.write("\n".join(self.lines) + "\n")

    def summary(self) -> dict | None:
        if not getattr(self, "lines", None):
            return None
        sm, smax, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            try:
                sm.append(float(f[1]))
                smax = max(smax, float(f[2]))
            except (ValueError, IndexError):
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        loaded = [s for s in sm if s > 0.5 * max(sm)]
        return dict(sm_mhz=statistics.median(loaded), sm_max_mhz=smax, reasons=sorted(reasons),
                    samples=len(sm))


# ---- the CPU oracle, timed on this host ------------------------------------------------------
def oracle_step_rate(w, min_seconds: float = 10.0, max_reps: int = 50, one_thread: bool = False) -> dict:
    """Time the oracle's segment step (same stages as the GPU step) on the host.

    The sample is the whole workload, repeated until min_seconds of CPU work,
    on every core OpenMP uses.  With one_thread, the same step is also timed
    on one thread over one (batch, kv-head) unit (the units are independent
    and equal in work), repeated until a quarter of min_seconds, and scaled
    to the workload's units.
    """
    import oracle
    oracle.build()
    x = {k: v.astype(np.float64) for k, v in w.full().items()}
    dims = oracle.Dims(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, T_hist=w.T_hist, T_seg=w.T_seg,
                       k_c=w.k_c, k_g=w.k_g)
    csum, gsum = oracle.build_summaries(dims, x["K"], 0, w.T_hist)
    reps, t0 = 0, time.perf_counter()
    while True:
        c, g = oracle.build_summaries(dims, x["K"], w.T_hist, w.T, csum, gsum)
        qbar = oracle.block_query(dims, x["Q"])
        cidx, _ = oracle.route_chunks(dims, qbar, c)
        gidx, _ = oracle.route_groups(dims, qbar, g, cidx)
        oracle.attn_fwd(dims, x["Q"], x["K"], x["V"], gidx)
        if w.backward:
            oracle.attn_bwd(dims, x["Q"], x["K"], x["V"], x["dO"], gidx)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or reps >= max_reps:
            break
    out = dict(value=reps * w.B * w.T_seg / el, unit="tokens/s", cores=oracle.num_threads(),
               kind="oracle", seconds=el,
               sample=f"whole {w.name} step (all {w.B * w.Hkv} (batch, kv-head) units) "
                      f"x {reps} repetitions, float64, OpenMP",
               cpu=_cpu_model())
    if one_thread:
        G, units = w.Hq // w.Hkv, w.B * w.Hkv
        x1 = {k: np.ascontiguousarray(v[:1, :G] if k in ("Q", "dO") else v[:1, :1]) for k, v in x.items()}
        d1 = oracle.Dims(B=1, Hq=G, Hkv=1, d=w.d, T_hist=w.T_hist, T_seg=w.T_seg, k_c=w.k_c, k_g=w.k_g)
        n0 = oracle.num_threads()
        oracle.set_num_threads(1)
        try:
            csum1, gsum1 = oracle.build_summaries(d1, x1["K"], 0, w.T_hist)
            reps1, t1 = 0, time.perf_counter()
            while True:
                c, g = oracle.build_summaries(d1, x1["K"], w.T_hist, w.T, csum1, gsum1)
                qbar = oracle.block_query(d1, x1["Q"])
                cidx, _ = oracle.route_chunks(d1, qbar, c)
                gidx, _ = oracle.route_groups(d1, qbar, g, cidx)
                oracle.attn_fwd(d1, x1["Q"], x1["K"], x1["V"], gidx)
                if w.backward:
                    oracle.attn_bwd(d1, x1["Q"], x1["K"], x1["V"], x1["dO"], gidx)
                reps1 += 1
                el1 = time.perf_counter() - t1
                if el1 >= min_seconds / 4 or reps1 >= max_reps:
                    break
        finally:
            oracle.set_num_threads(n0)
        out["one_thread"] = dict(value=reps1 * w.B * w.T_seg / (el1 * units), unit="tokens/s", cores=1,
                                 seconds=el1,
                                 sample=f"one (batch, kv-head) unit of {w.name} x {reps1} repetitions on one "
                                        f"thread, scaled to the workload's {units} units")
    return out


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    return ln.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ---- main ------------------------------------------------------------------------------------
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def rank_workload(w, rank: int):
    """The independent problem of one rank: same shape, its own seed."""
    return w.with_(seed=w.seed + rank)


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank duration over all ranks (1 rank: the value itself)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(tokens_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """All ranks' tokens over the slowest rank's time (weak scaling)."""
    return world * steps * tokens_per_rank_step / (max_ms * 1e-3)


def config_of(w, graph: bool = True) -> dict:
    return dict(workload=w.name, B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, T_hist=w.T_hist,
                T_seg=w.T_seg, T=w.T, k_c=w.k_c, k_g=w.k_g, keys=w.keys,
                l2="flushed between timed steps (256 MiB write)",
                launch=("CUDA graph of the step, events around its replay; stage_ms from a second "
                        "capture with events between the stages") if graph else "eager")


def run_reference(args, w) -> None:
    rank, world, _ = dist_env()
    if rank != 0:
        return
    cb = oracle_step_rate(w, min_seconds=args.ref_seconds)
    steps = args.steps
    line = dict(metric=METRIC, value=cb["value"], unit="tokens/s", n_gpus=args.gpus, steps=steps,
                warmup=args.warmup, ms_per_step=1e3 * w.B * w.T_seg / cb["value"],
                higher_is_better=True, scaling="weak", vs_baseline=None, dtype="f64",
                data="synthetic", impl="reference", config=config_of(w), cpu_baseline=cb,
                e2e=dict(value=cb["value"], unit="tokens/s", h2d_bytes_per_step=0,
                         d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)


def run_gpu(args, w) -> None:
    import torch
    import torch.distributed as dist

    import hierarchical_routed_sparse_b200 as hga

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    wr = rank_workload(w, rank)                      # independent problem per rank
    x = wr.full()
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    Q = torch.from_numpy(x["Q"]).to(dev, tdt)
    K = torch.from_numpy(x["K"]).to(dev, tdt)
    V = torch.from_numpy(x["V"]).to(dev, tdt)
    dO = torch.from_numpy(x["dO"]).to(dev, tdt) if w.backward else None
    p = hga.Params.from_workload(w)
    buf = hga.Buffers(p, device=dev)
    buf.summaries(K, 0, w.T_hist)                    # history summaries persist
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    stages = ["summaries", "route", "attn_fwd", "attn_bwd"]

    def step_on(st, ev=None):
        if ev is not None:
            ev[0].record(st)
        buf.summaries(K, stream=st)
        if ev is not None:
            ev[1].record(st)
        buf.route(Q, st)
        if ev is not None:
            ev[2].record(st)
        buf.forward(Q, K, V, stream=st)
        if ev is not None:
            ev[3].record(st)
        if dO is not None:
            buf.backward(Q, K, V, dO, stream=st)
        if ev is not None:
            ev[4].record(st)

    def step(ev=None):
        step_on(stream, ev)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    # Events recorded inside a captured graph must be "external" to be timed
    # from outside it.
    events = [[torch.cuda.Event(enable_timing=True, external=not args.no_graph) for _ in range(5)]
              for _ in range(args.steps)]
    # Whole-step timing: events on the stream around each step (the L2 flush
    # before the first event).  With graphs, the step is one CUDA graph and
    # the events bracket its replay, graph launch included.
    outer = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(args.steps)]
    run_step = step
    run_plain = step
    if not args.no_graph:
        # Two captures of one segment step: a plain graph, timed from outside
        # for the headline, and one graph per timed step with stage events
        # recorded inside it for the per-stage breakdown (each event node
        # adds a few microseconds between the kernels it separates).
        graphs = []
        cap_stream = torch.cuda.Stream(dev)
        cap_stream.wait_stream(stream)
        with torch.cuda.stream(cap_stream):
            for i in range(args.steps):
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=cap_stream):
                    step_on(cap_stream, events[i])
                graphs.append(g)
            plain = torch.cuda.CUDAGraph()
            with torch.cuda.graph(plain, stream=cap_stream):
                step_on(cap_stream)
        stream.wait_stream(cap_stream)
        torch.cuda.synchronize()
        for _ in range(args.warmup):
            flush.zero_()
            graphs[0].replay()
            flush.zero_()
            plain.replay()
        torch.cuda.synchronize()

        def run_step(ev, i=[0]):
            graphs[i[0] % len(graphs)].replay()
            i[0] += 1

        def run_plain():
            plain.replay()
    clocks_path = args.clocks_csv if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local, clocks_path) as clk:
        for i in range(args.steps):
            flush.zero_()                            # outside the timed events
            outer[i][0].record(stream)
            run_plain()
            outer[i][1].record(stream)
        for i in range(args.steps):
            flush.zero_()
            run_step(events[i])
        # The same step with L2 left warm: plain replays back to back (one
        # untimed replay first), events around each.
        warm = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(args.steps)]
        run_plain()
        for a, b in warm:
            a.record(stream)
            run_plain()
            b.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    warm_ms = [a.elapsed_time(b) for a, b in warm]
    warm_total = max_over_ranks(sum(warm_ms), dev)
    per_stage = {s: [] for s in stages}
    staged_totals = []
    for ev in events:
        for j, s in enumerate(stages):
            per_stage[s].append(ev[j].elapsed_time(ev[j + 1]))
        staged_totals.append(ev[0].elapsed_time(ev[4]))
    totals = [a.elapsed_time(b) for a, b in outer]
    total_ms = max_over_ranks(sum(totals), dev)
    staged_ms = max_over_ranks(sum(staged_totals), dev)
    value = whole_job_rate(w.B * w.T_seg, args.steps, world, total_ms)

    # ---- end to end through the public API with host buffers ----------------------
    Qh = torch.from_numpy(x["Q"]).to(tdt).pin_memory()
    Kh = torch.from_numpy(np.ascontiguousarray(x["K"][:, :, w.T_hist:])).to(tdt).pin_memory()
    Vh = torch.from_numpy(np.ascontiguousarray(x["V"][:, :, w.T_hist:])).to(tdt).pin_memory()
    dOh = torch.from_numpy(x["dO"]).to(tdt).pin_memory() if w.backward else None
    outs_dev = [buf.dQ, buf.dK, buf.dV] if w.backward else [buf.O, buf.lse]
    outs_h = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs_dev]
    h2d = sum(t.numel() * t.element_size() for t in (Qh, Kh, Vh, dOh) if t is not None)
    d2h = sum(t.numel() * t.element_size() for t in outs_h)

    def e2e_step():
        Q.copy_(Qh, non_blocking=True)
        K[:, :, w.T_hist:].copy_(Kh, non_blocking=True)
        V[:, :, w.T_hist:].copy_(Vh, non_blocking=True)
        if dOh is not None:
            dO.copy_(dOh, non_blocking=True)
        step()
        for hst, dv in zip(outs_h, outs_dev):
            hst.copy_(dv, non_blocking=True)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if w.backward:
        # Training steps through hga.StepPipeline: the next step's uploads and
        # the previous step's downloads overlap this step's compute (own
        # streams, two device buffer sets); every step moves all its bytes.
        pipe = hga.StepPipeline(p, K[:, :, :w.T_hist], V[:, :, :w.T_hist], device=dev)
        outs_sets = [outs_h, [torch.empty(o.shape, dtype=o.dtype).pin_memory() for o in outs_dev]]
        for i in range(args.warmup):
            pipe.submit(Qh, Kh, Vh, dOh, outs_sets[i % 2])
        pipe.synchronize()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0.record(pipe.s_in)
        for i in range(args.steps):
            pipe.submit(Qh, Kh, Vh, dOh, outs_sets[i % 2])
        e1.record(pipe.s_out)
        torch.cuda.synchronize()
        e2e_mode = "hga.StepPipeline: uploads, compute and downloads of consecutive steps overlapped"
    else:
        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_mode = "serial: upload, step, download on one stream"
    e2e_value = whole_job_rate(w.B * w.T_seg, args.steps, world,
                               max_over_ranks(e0.elapsed_time(e1), dev))

    # ---- the one-shot summaries of the whole context (not part of a step) ----------
    full_ms = []
    for _ in range(max(args.warmup, 3) + 5):
        flush.zero_()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        buf.summaries(K, 0, w.T, stream)
        s1.record(stream)
        torch.cuda.synchronize()
        full_ms.append(s0.elapsed_time(s1))
    full_ms = statistics.median(full_ms[max(args.warmup, 3):])
    # Context for that figure: a plain device copy moving the same bytes
    # (half read, half written), timed the same way.  A one-shot transfer of
    # tens of MB pays launch, ramp-up and tail, so it does not reach the
    # copy peak measured on gigabytes.
    full_bytes_all = (w.B * w.Hkv * w.T * w.d * (2 if w.dtype == "bf16" else 4)
                      + w.B * w.Hkv * (w.T // 64 + w.T // 8) * w.d * 4)
    cp_src = torch.empty(full_bytes_all // 8, dtype=torch.float32, device=dev)
    cp_dst = torch.empty_like(cp_src)
    copy_ms = []
    for _ in range(max(args.warmup, 3) + 5):
        flush.zero_()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        cp_dst.copy_(cp_src)
        s1.record(stream)
        torch.cuda.synchronize()
        copy_ms.append(s0.elapsed_time(s1))
    copy_ms = statistics.median(copy_ms[max(args.warmup, 3):])
    del cp_src, cp_dst

    # ---- routing + forward: the fused launch against the two launches ---------------
    def eager_ms(fn, n):
        ts = []
        for _ in range(n):
            flush.zero_()
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            fn()
            s1.record(stream)
            torch.cuda.synchronize()
            ts.append(s0.elapsed_time(s1))
        return statistics.median(ts[max(args.warmup, 3):])

    n_rf = max(args.warmup, 3) + 7
    fused_ms = eager_ms(lambda: buf.route_forward(Q, K, V, stream), n_rf)
    separate_ms = eager_ms(lambda: (buf.route(Q, stream), buf.forward(Q, K, V, stream=stream)), n_rf)

    if rank == 0:
        alg = algorithmic(w)
        pk = peaks()
        fwd_ms = statistics.mean(per_stage["attn_fwd"])
        bwd_ms = statistics.mean(per_stage["attn_bwd"]) if w.backward else 0.0
        dom = "attn_bwd" if bwd_ms >= fwd_ms else "attn_fwd"
        dom_ms = bwd_ms if dom == "attn_bwd" else fwd_ms
        a = alg[dom]
        ai = a["flops"] / a["bytes"]
        ridge = pk["bf16_tflops_sustained"] * 1e12 / (pk["hbm_gbs"] * 1e9)
        if ai < ridge:
            achieved = a["bytes"] / (dom_ms * 1e-3) / 1e9
            roof = dict(bound="hbm", achieved=achieved, peak=pk["hbm_gbs"], unit="GB/s")
        else:
            achieved = a["flops"] / (dom_ms * 1e-3) / 1e12
            roof = dict(bound="tensor", achieved=achieved, peak=pk["bf16_tflops_sustained"],
                        unit="TFLOP/s")
        roof.update(frac=roof["achieved"] / roof["peak"],
                    traffic=args.traffic if args.traffic is not None else recorded_traffic(dom, w),
                    kernel=dom, launch_ms=dom_ms, algorithmic_bytes=a["bytes"],
                    algorithmic_flops=a["flops"], peak_source=pk["source"])
        stage_ms = {s: statistics.mean(v) for s, v in per_stage.items()}
        # Every stage against the HBM roofline (algorithmic bytes / stage time;
        # stage times carry the events' own cost of a few microseconds).
        stage_bytes = dict(summaries=alg["summaries"]["bytes"],
                           route=alg["route_chunks"]["bytes"] + alg["route_groups"]["bytes"],
                           attn_fwd=alg["attn_fwd"]["bytes"], attn_bwd=alg["attn_bwd"]["bytes"])
        stage_roof = {}
        for s_, b_ in stage_bytes.items():
            if s_ in stage_ms and stage_ms[s_] > 0:
                gbs = b_ / (stage_ms[s_] * 1e-3) / 1e9
                stage_roof[s_] = dict(ms=stage_ms[s_], algorithmic_bytes=b_, gb_per_s=gbs,
                                      frac=gbs / pk["hbm_gbs"])
        # The routers' roofline counts each byte once (Q, the chunk summaries,
        # the gathered group summaries, index rows); the per-use figure counts
        # every block's read of its eligible chunk summaries.
        if "route" in stage_roof:
            r_ = stage_roof["route"]
            per_use = alg["route_chunks"]["per_use_bytes"] + alg["route_groups"]["bytes"]
            r_["per_use_bytes"] = per_use
            r_["frac_per_use"] = per_use / (r_["ms"] * 1e-3) / 1e9 / pk["hbm_gbs"]
            if r_["frac_per_use"] > 1.0:
                r_["note"] = "per-use bytes above the copy peak: re-reads of the summaries hit L2"
        el = 2 if w.dtype == "bf16" else 4
        full_bytes = w.B * w.Hkv * w.T * w.d * el + w.B * w.Hkv * (w.T // 64 + w.T // 8) * w.d * 4
        stage_roof["summaries_full_history"] = dict(
            ms=full_ms, algorithmic_bytes=full_bytes, gb_per_s=full_bytes / (full_ms * 1e-3) / 1e9,
            frac=full_bytes / (full_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
            copy_same_bytes_ms=copy_ms, frac_of_copy_same_bytes=copy_ms / full_ms,
            note="one-shot build of all chunk / group summaries of the context, timed alone; "
                 "copy_same_bytes_ms: a device copy moving the same bytes, timed the same way")
        rf_bytes = stage_bytes["route"] + stage_bytes["attn_fwd"]
        stage_roof["route_attn_fwd_fused"] = dict(
            ms=fused_ms, separate_ms=separate_ms, algorithmic_bytes=rf_bytes,
            gb_per_s=rf_bytes / (fused_ms * 1e-3) / 1e9, frac=rf_bytes / (fused_ms * 1e-3) / 1e9 / pk["hbm_gbs"],
            note="hga_route_attn_fwd (routing and forward in one persistent launch) against hga_route + "
                 "hga_attn_fwd (separate_ms), each timed alone on eager launches, L2 flushed before each")
        line = dict(metric=METRIC, value=value, unit="tokens/s", n_gpus=world, steps=args.steps,
                    warmup=args.warmup, ms_per_step=total_ms / args.steps, higher_is_better=True,
                    scaling="weak", vs_baseline=None, dtype=w.dtype, data="synthetic",
                    config=config_of(w, not args.no_graph), stage_ms=stage_ms,
                    ms_per_step_with_stage_events=staged_ms / args.steps,
                    ms_per_step_median=statistics.median(totals),
                    l2_warm=dict(ms_per_step=warm_total / args.steps, ms_median=statistics.median(warm_ms),
                                 note="the same graph replayed back to back, L2 not flushed between steps"),
                    roofline=roof,
                    stage_roofline=stage_roof,
                    gpu_launches=(LAUNCHES_FWD + (LAUNCHES_BWD if w.backward else 0)) * args.steps,
                    e2e=dict(value=e2e_value, unit="tokens/s", h2d_bytes_per_step=h2d,
                             d2h_bytes_per_step=d2h, mode=e2e_mode),
                    clocks=clk.summary())
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = oracle_step_rate(w, min_seconds=args.ref_seconds, one_thread=True)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_host_tier(args, w) -> None:
    """The segment step with the history K/V rows in pinned host memory: the
    segment's summaries come from its own rows (hga_build_summaries_rows),
    the routed history groups are staged in device memory over the host link
    after routing (hga_stage_routed), and the attention runs on the staged
    problem.  One JSON line with config.kv_tier = "host"."""
    import torch
    import torch.distributed as dist

    import hierarchical_routed_sparse_b200 as hga

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    wr = rank_workload(w, rank)
    x = wr.full()
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    p = hga.Params.from_workload(w)
    buf = hga.Buffers(p, device=dev)
    # History summaries persist in HBM (built once, from the history rows).
    Kh = torch.from_numpy(np.ascontiguousarray(x["K"][:, :, :w.T_hist])).to(tdt).pin_memory()
    Vh = torch.from_numpy(np.ascontiguousarray(x["V"][:, :, :w.T_hist])).to(tdt).pin_memory()
    hga.build_summaries_rows(p, Kh.to(dev), 0, w.T_hist, buf.csum, buf.gsum)
    Q = torch.from_numpy(x["Q"]).to(dev, tdt)
    Ks = torch.from_numpy(np.ascontiguousarray(x["K"][:, :, w.T_hist:])).to(dev, tdt)
    Vs = torch.from_numpy(np.ascontiguousarray(x["V"][:, :, w.T_hist:])).to(dev, tdt)
    dO = torch.from_numpy(x["dO"]).to(dev, tdt) if w.backward else None
    skv = hga.StagedKV(p, device=dev)
    sbuf = hga.Buffers(skv.ps, device=dev)           # outputs of the staged attention
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    torch.cuda.synchronize()
    stages = ["summaries", "route", "stage", "attn_fwd", "attn_bwd"]

    def step_on(st, ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record(st)
        mark(0)
        hga.build_summaries_rows(p, Ks, w.T_hist, w.T, buf.csum, buf.gsum, st)
        mark(1)
        buf.route(Q, st)
        mark(2)
        skv.stage(Kh, Vh, Ks, Vs, buf.gidx, st)
        mark(3)
        sbuf.forward(Q, skv.K, skv.V, gidx=skv.gidx, stream=st)
        mark(4)
        if dO is not None:
            sbuf.backward(Q, skv.K, skv.V, dO, gidx=skv.gidx, stream=st)
        mark(5)

    for _ in range(args.warmup):
        flush.zero_()
        step_on(stream)
    torch.cuda.synchronize()
    events = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(6)] for _ in range(args.steps)]
    outer = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(args.steps)]
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    graphs = []
    with torch.cuda.stream(cap):
        for i in range(args.steps):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                step_on(cap, events[i])
            graphs.append(g)
        plain = torch.cuda.CUDAGraph()
        with torch.cuda.graph(plain, stream=cap):
            step_on(cap)
    stream.wait_stream(cap)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        flush.zero_()
        plain.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    with ClockSampler(local, None) as clk:
        for i in range(args.steps):
            flush.zero_()
            outer[i][0].record(stream)
            plain.replay()
            outer[i][1].record(stream)
        for i in range(args.steps):
            flush.zero_()
            graphs[i].replay()
        torch.cuda.synchronize()
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in outer), dev)
    stage_ms = {s: statistics.mean(ev[j].elapsed_time(ev[j + 1]) for ev in events) for j, s in enumerate(stages)}
    value = whole_job_rate(w.B * w.T_seg, args.steps, world, total_ms)
    # Host bytes read per step: 8 rows of K and of V per staged history group.
    gidx = buf.gidx.cpu().numpy()
    # Distinct routed history groups per (batch, kv-head): each is staged once.
    fsg = w.T_hist // 8
    n_hist = sum(len(np.unique(gidx[b_, g_][(gidx[b_, g_] >= 0) & (gidx[b_, g_] < fsg)]))
                 for b_ in range(gidx.shape[0]) for g_ in range(gidx.shape[1]))
    host_bytes = n_hist * 8 * w.d * (2 if w.dtype == "bf16" else 4) * 2
    if rank == 0:
        line = dict(metric=METRIC, value=value, unit="tokens/s", n_gpus=world, steps=args.steps,
                    warmup=args.warmup, ms_per_step=total_ms / args.steps, higher_is_better=True,
                    scaling="weak", vs_baseline=None, dtype=w.dtype, data="synthetic",
                    config=dict(config_of(w), kv_tier="host",
                                history="pinned host memory, routed groups staged in HBM per step"),
                    stage_ms=stage_ms,
                    host_link=dict(bytes_per_step=host_bytes,
                                   gb_per_s=host_bytes / (stage_ms["stage"] * 1e-3) / 1e9),
                    gpu_launches=(LAUNCHES_FWD + 1 + (LAUNCHES_BWD if w.backward else 0)) * args.steps,
                    clocks=clk.summary())
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_layer(args, w) -> None:
    """Segment-wise (TBPTT) training of one attention layer with HGA as its
    attention: Q / K / V / O projections of the workload's head layout over
    d_model = Hq * d (bf16 autocast), HGA forward and backward per segment,
    an SGD step per segment.  The sequence is the workload's T tokens in
    T / T_seg segments, so the last segment sees the workload's history.
    One JSON line, config.mode = "layer_tbptt"."""
    import torch

    import hierarchical_routed_sparse_b200 as hga
    from hierarchical_routed_sparse_b200.segment import HGASegmentLayer

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(0)
    d_model = w.Hq * w.d
    layer = HGASegmentLayer(d_model, w.Hq, w.Hkv, w.d, k_c=w.k_c, k_g=w.k_g)
    opt = torch.optim.SGD(layer.parameters(), lr=1e-4)
    x = torch.randn(w.B, w.T, d_model, device=dev, generator=g)
    target = torch.randn(w.B, w.T, d_model, device=dev, generator=g)
    n_seg = w.T // w.T_seg
    stream = torch.cuda.current_stream(dev)

    def sequence():
        layer.cache.reset()
        for s in range(n_seg):
            xs = x[:, s * w.T_seg:(s + 1) * w.T_seg]
            ts = target[:, s * w.T_seg:(s + 1) * w.T_seg]
            with torch.autocast("cuda", dtype=torch.bfloat16):
                out = layer.segment(xs)
                loss = 0.5 * (out.float() - ts).pow(2).mean()
            loss.backward()
            opt.step()
            opt.zero_grad(set_to_none=True)

    for _ in range(args.warmup):
        sequence()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with ClockSampler(0, None) as clk:
        for a, b in ev:
            a.record(stream)
            sequence()
            b.record(stream)
        torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    assert hga.device_status() == 0
    line = dict(metric="HGA attention layer, segment-wise training: tokens/s", value=w.B * w.T / (ms * 1e-3),
                unit="tokens/s", n_gpus=1, steps=args.steps, warmup=args.warmup, ms_per_step=ms,
                higher_is_better=True, scaling="weak", vs_baseline=None, dtype="bf16 (autocast projections)",
                data="synthetic",
                config=dict(config_of(w), mode="layer_tbptt", d_model=d_model, segments=n_seg,
                            l2="not flushed (a pass streams far more than L2)",
                            launch="eager PyTorch autograd, events around each pass",
                            step="one pass over the T tokens: per segment projections, HGA fwd + bwd, SGD"),
                clocks=clk.summary())
    print(json.dumps(line), flush=True)


def causal_algorithmic(w) -> dict:
    """Algorithmic bytes of the causal variant's attention kernels: every
    input row read once (Q, dO, O, lse and the whole K / V context of each
    (batch, kv-head)), every output written once, the per-position routing
    rows read once."""
    el = 2 if w.dtype == "bf16" else 4
    B, Hq, Hkv, d, Ts, T = w.B, w.Hq, w.Hkv, w.d, w.T_seg, w.T
    wc = w.k_c if w.k_c > 0 else T // 64
    wg = w.k_g if w.k_g > 0 else 8 * wc
    q = B * Hq * Ts * d * el
    kv = 2 * B * Hkv * T * d * el
    o = B * Hq * Ts * d * 4
    l_ = B * Hq * Ts * 4
    gi = B * Hkv * Ts * wg * 4
    seg = 2 * B * Hkv * Ts * d * 4
    return dict(attn_fwd_causal=q + kv + o + l_ + gi,
                attn_bwd_causal=q + q + o + l_ + kv + gi + o + seg,
                route_causal=q + B * Hkv * (T // 64 + T // 8) * d * 4 + B * Hkv * Ts * (wc + wg) * 4)


def run_causal(args, w) -> None:
    """The segment training step of the strictly causal variant (every query
    position routes on its own query): segment summaries, per-position
    routing, the causal attention forward and backward.  CUDA graph of the
    step, events around its replay, L2 flushed between steps; stage_ms from a
    second capture with events between the stages.  One JSON line,
    config.mode = "causal"."""
    import torch

    import hierarchical_routed_sparse_b200 as hga

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    x = w.full()
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    p = hga.Params.from_workload(w)
    cb = hga.CausalBuffers(p, device=dev)
    Q, K, V = (torch.from_numpy(x[k]).to(dev, tdt) for k in ("Q", "K", "V"))
    dO = torch.from_numpy(x["dO"]).to(dev, tdt)
    cb.summaries(K, 0, w.T_hist)                     # history summaries persist
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    stages = ["summaries", "route_causal", "attn_fwd_causal", "attn_bwd_causal"]

    def step_on(st, ev=None):
        def mark(i):
            if ev is not None:
                ev[i].record(st)
        mark(0)
        cb.summaries(K, stream=st)
        mark(1)
        cb.route(Q, st)
        mark(2)
        cb.forward(Q, K, V, stream=st)
        mark(3)
        cb.backward(Q, K, V, dO, stream=st)
        mark(4)

    for _ in range(args.warmup):
        flush.zero_()
        step_on(stream)
    torch.cuda.synchronize()
    events = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(5)] for _ in range(args.steps)]
    outer = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(args.steps)]
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    graphs = []
    with torch.cuda.stream(cap):
        for i in range(args.steps):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                step_on(cap, events[i])
            graphs.append(g)
        plain = torch.cuda.CUDAGraph()
        with torch.cuda.graph(plain, stream=cap):
            step_on(cap)
    stream.wait_stream(cap)
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        flush.zero_()
        plain.replay()
    torch.cuda.synchronize()
    with ClockSampler(0, None) as clk:
        for i in range(args.steps):
            flush.zero_()
            outer[i][0].record(stream)
            plain.replay()
            outer[i][1].record(stream)
        for i in range(args.steps):
            flush.zero_()
            graphs[i].replay()
        torch.cuda.synchronize()
    total_ms = sum(a.elapsed_time(b) for a, b in outer)
    stage_ms = {s_: statistics.mean(ev[j].elapsed_time(ev[j + 1]) for ev in events) for j, s_ in enumerate(stages)}
    assert hga.device_status() == 0
    ms = total_ms / args.steps
    alg = causal_algorithmic(w)
    pk = peaks()
    dom = max(("attn_fwd_causal", "attn_bwd_causal"), key=lambda k: stage_ms[k])
    achieved = alg[dom] / (stage_ms[dom] * 1e-3) / 1e9
    # End to end through the public API: Q / K_seg / V_seg / dO from pinned
    # host memory each step, the loss-side dQ read back.
    el = 2 if w.dtype == "bf16" else 4
    seg = slice(w.T_hist, w.T)
    hosts = {k: v.cpu().pin_memory() for k, v in (("Q", Q), ("dO", dO))}
    ks_h = K[:, :, seg].contiguous().cpu().pin_memory()
    vs_h = V[:, :, seg].contiguous().cpu().pin_memory()
    dq_h = torch.empty(cb.dQ.shape, dtype=torch.float32).pin_memory()
    ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        flush.zero_()
        ev2[i][0].record(stream)
        Q.copy_(hosts["Q"], non_blocking=True)
        dO.copy_(hosts["dO"], non_blocking=True)
        K[:, :, seg].copy_(ks_h, non_blocking=True)
        V[:, :, seg].copy_(vs_h, non_blocking=True)
        step_on(stream)
        dq_h.copy_(cb.dQ, non_blocking=True)
        ev2[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = statistics.mean(a.elapsed_time(b) for a, b in ev2)
    h2d = (2 * w.B * w.Hq * w.T_seg + 2 * w.B * w.Hkv * w.T_seg) * w.d * el
    d2h = w.B * w.Hq * w.T_seg * w.d * 4
    line = dict(metric="HGA strictly causal variant, segment fwd+bwd tokens/s at 16K ctx",
                value=w.B * w.T_seg / (ms * 1e-3), unit="tokens/s", n_gpus=1, steps=args.steps,
                warmup=args.warmup, ms_per_step=ms, higher_is_better=True, scaling="weak", vs_baseline=None,
                dtype=w.dtype, data="synthetic",
                config=dict(config_of(w), mode="causal",
                            routing="per query position (a block of one); per-row key sets"),
                stage_ms=stage_ms,
                roofline=dict(bound="hbm", achieved=achieved, peak=pk["hbm_gbs"], unit="GB/s",
                              frac=achieved / pk["hbm_gbs"],
                              traffic=recorded_traffic(dom, w) if dom in KERNEL_SOURCES else None, kernel=dom,
                              algorithmic_bytes_per_launch=alg[dom],
                              peak_source=pk["source"] + " (burst copy)"),
                e2e=dict(value=w.B * w.T_seg / (e2e_ms * 1e-3), unit="tokens/s", h2d_bytes_per_step=h2d,
                         d2h_bytes_per_step=d2h),
                # summaries, routing + the window schedule's two kernels, forward, backward
                gpu_launches=(1 + 3 + 1 + 1) * args.steps, clocks=clk.summary())
    print(json.dumps(line), flush=True)


def decode_algorithmic(w, pos: int) -> dict:
    """Algorithmic bytes of one hga_decode call at position pos: the token's
    queries, the eligible chunk summaries, the group summaries of the routed
    chunks, the routed groups' and the own chunk's K / V rows, and the
    outputs (O, lse, cidx, gidx)."""
    el = 2 if w.dtype == "bf16" else 4
    c0 = pos // 64
    nc = c0 if w.k_c <= 0 else min(w.k_c, c0)
    ng = 8 * nc if w.k_g <= 0 else min(w.k_g, 8 * nc)
    n_keys = 8 * ng + pos - 64 * c0 + 1
    wc = w.k_c if w.k_c > 0 else w.T // 64
    wg = w.k_g if w.k_g > 0 else 8 * wc
    per_unit = (w.G * w.d * el + c0 * w.d * 4 + 8 * nc * w.d * 4 + 2 * n_keys * w.d * el
                + w.G * (w.d + 1) * 4 + (wc + wg) * 4)
    return dict(bytes=w.B * w.Hkv * per_unit, n_keys=n_keys)


def oracle_decode_rate(w, pos0: int, min_seconds: float = 10.0, max_reps: int = 1_000_000) -> dict:
    """The oracle's decode step on the first sequence of the batch, at the
    positions the GPU run decodes, repeated for about min_seconds."""
    import oracle
    oracle.build()
    w1 = w.with_(B=1)
    x = w1.full()
    K, V = x["K"].astype(np.float64), x["V"].astype(np.float64)
    dims = oracle.Dims(B=1, Hq=w.Hq, Hkv=w.Hkv, d=w.d, T_hist=w.T_hist, T_seg=w.T_seg, k_c=w.k_c, k_g=w.k_g)
    csum, gsum = oracle.build_summaries(dims, K)
    q = x["Q"][:, :, 0].astype(np.float64)
    reps, t0 = 0, time.perf_counter()
    while True:
        oracle.decode(dims, pos0 + reps % 64, q, K, V, csum, gsum)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or reps >= max_reps:
            break
    return dict(value=reps / el, unit="tokens/s", cores=oracle.num_threads(), kind="oracle", seconds=el,
                sample=f"{reps} decode steps of one sequence ({w.Hq} q-heads, {w.Hkv} kv-heads, ctx {w.T}), "
                       "float64, OpenMP over kv-heads",
                cpu=_cpu_model())


def run_decode(args, w) -> None:
    """Generation with HGA: one decode step per token (hga_decode) over a
    KV cache of the workload's T rows, for a batch of sequences.  The timed
    steps decode the last 64 positions of the cache (T-64 .. T-1) in order;
    the step that completes the chunk also appends its summaries
    (hga_build_summaries).  Each step is timed alone with CUDA events, L2
    flushed before it.  One JSON line, config.mode = "decode"."""
    import torch

    import hierarchical_routed_sparse_b200 as hga

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    wd = w.with_(B=args.decode_batch, backward=False)
    if args.decode_layers > 1:
        return run_decode_layers(args, wd)
    x = wd.full()
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    p = hga.Params.from_workload(wd)
    st = hga.DecodeState(p, device=dev)
    K = torch.from_numpy(x["K"]).to(dev, tdt)
    V = torch.from_numpy(x["V"]).to(dev, tdt)
    pos0 = wd.T - 64
    st.prefill(K[:, :, :pos0], V[:, :, :pos0])
    st.K.copy_(K)                                   # rows of the timed tokens already in place
    st.V.copy_(V)
    del K, V
    qs = [torch.from_numpy(np.ascontiguousarray(x["Q"][:, :, i])).to(dev, tdt) for i in range(64)]
    del x
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(i, s=None):
        pos = pos0 + i % 64
        hga.decode(p, pos, qs[i % 64], st.K, st.V, st.csum, st.gsum, st.O, st.lse, st.cidx, st.gidx, s)
        if (pos + 1) % 64 == 0:
            hga.build_summaries(p, st.K, pos + 1 - 64, pos + 1, st.csum, st.gsum, s)

    for i in range(max(args.warmup, 3)):
        flush.zero_()
        step(i)
    torch.cuda.synchronize()
    n = max(args.steps, 64)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    launches = 0
    with ClockSampler(0, None) as clk:
        # A decode call is shorter than its host-side launch path (Python
        # marshalling + C-ABI checks): a GPU-side delay first lets the host
        # queue every timed step ahead, so the events time the device work.
        torch.cuda._sleep(int(1e8))
        for i in range(n):
            flush.zero_()
            ev[i][0].record(stream)
            step(i)
            ev[i][1].record(stream)
            launches += 1 + ((pos0 + i % 64 + 1) % 64 == 0)
        torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in ev]
    ms_step = statistics.mean(ms)
    # Decode calls alone (steps that do not append summaries).
    dec_ms = statistics.mean(m for i, m in enumerate(ms) if (pos0 + i % 64 + 1) % 64 != 0)
    # End to end through the public API: q from pinned host memory, O back;
    # no delay ahead, so the host's launch path counts.
    el = 2 if w.dtype == "bf16" else 4
    q_host = [q.cpu().pin_memory() for q in qs]
    o_host = torch.empty(st.O.shape, dtype=torch.float32).pin_memory()
    q_dev = torch.empty_like(qs[0])
    ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for i in range(n):
        flush.zero_()
        ev2[i][0].record(stream)
        q_dev.copy_(q_host[i % 64], non_blocking=True)
        pos = pos0 + i % 64
        hga.decode(p, pos, q_dev, st.K, st.V, st.csum, st.gsum, st.O, st.lse, st.cidx, st.gidx)
        if (pos + 1) % 64 == 0:
            hga.build_summaries(p, st.K, pos + 1 - 64, pos + 1, st.csum, st.gsum)
        o_host.copy_(st.O, non_blocking=True)
        ev2[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = statistics.mean(a.elapsed_time(b) for a, b in ev2)
    assert hga.device_status() == 0
    pk = peaks()
    alg = statistics.mean(decode_algorithmic(wd, pos0 + i)["bytes"] for i in range(63))
    achieved = alg / (dec_ms * 1e-3) / 1e9
    line = dict(metric="HGA decode tokens/s at 16K ctx (one token per sequence per step)",
                value=wd.B / (ms_step * 1e-3), unit="tokens/s", n_gpus=1, steps=n, warmup=args.warmup,
                ms_per_step=ms_step, higher_is_better=True, scaling="weak", vs_baseline=None, dtype=w.dtype,
                data="synthetic",
                config=dict(config_of(wd, graph=False), mode="decode", decode_batch=wd.B,
                            positions=f"{pos0}..{wd.T - 1}, summaries appended at chunk end",
                            l2="flushed before every step (256 MiB write)",
                            launch="eager, CUDA events around each step"),
                decode_call_ms=dec_ms,
                roofline=dict(bound="hbm", achieved=achieved, peak=pk["hbm_gbs"], unit="GB/s",
                              frac=achieved / pk["hbm_gbs"], traffic=None,
                              kernel="decode_kernel", algorithmic_bytes_per_call=alg,
                              peak_source=pk["source"] + " (burst copy)"),
                e2e=dict(value=wd.B / (e2e_ms * 1e-3), unit="tokens/s", h2d_bytes_per_step=wd.B * wd.Hq * wd.d * el,
                         d2h_bytes_per_step=wd.B * wd.Hq * wd.d * 4),
                gpu_launches=launches, clocks=clk.summary())
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_decode_rate(wd, pos0)
    print(json.dumps(line), flush=True)


def run_decode_layers(args, wd) -> None:
    """Decode through a stack of L attention layers per token: L caches (one
    per layer, the workload's 16K context each), one CUDA graph per token
    position holding the L hga_decode calls (and, at a chunk's last token,
    the L summary appends), replayed with events around it; L2 flushed
    before every token.  The decode kernels launch with programmatic
    dependent launch, so each layer's launch overlaps the previous one's
    tail.  One JSON line, config.mode = "decode_layers"."""
    import torch

    import hierarchical_routed_sparse_b200 as hga

    dev = torch.device("cuda", 0)
    L = args.decode_layers
    x = wd.full()
    tdt = torch.bfloat16 if wd.dtype == "bf16" else torch.float32
    p = hga.Params.from_workload(wd)
    K = torch.from_numpy(x["K"]).to(dev, tdt)
    V = torch.from_numpy(x["V"]).to(dev, tdt)
    pos0 = wd.T - 64
    states = []
    for _ in range(L):
        st = hga.DecodeState(p, device=dev)
        st.prefill(K[:, :, :pos0], V[:, :, :pos0])
        st.K.copy_(K)
        st.V.copy_(V)
        states.append(st)
    del K, V
    qs = [torch.from_numpy(np.ascontiguousarray(x["Q"][:, :, i])).to(dev, tdt) for i in range(64)]
    del x
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def token(i, st_):
        pos = pos0 + i
        for l_, sl in enumerate(states):
            hga.decode(p, pos, qs[(i + l_) % 64], sl.K, sl.V, sl.csum, sl.gsum, sl.O, sl.lse, sl.cidx, sl.gidx, st_)
        if (pos + 1) % 64 == 0:
            for sl in states:
                hga.build_summaries(p, sl.K, pos + 1 - 64, pos + 1, sl.csum, sl.gsum, st_)

    for i in range(64):                              # warm-up, eager
        token(i, stream)
    torch.cuda.synchronize()
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    graphs = []
    with torch.cuda.stream(cap):
        for i in range(64):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                token(i, cap)
            graphs.append(g)
    stream.wait_stream(cap)
    torch.cuda.synchronize()
    for i in range(max(args.warmup, 3)):
        flush.zero_()
        graphs[i % 64].replay()
    torch.cuda.synchronize()
    n = max(args.steps, 64)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    with ClockSampler(0, None) as clk:
        for i in range(n):
            flush.zero_()
            ev[i][0].record(stream)
            graphs[i % 64].replay()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in ev]
    ms_tok = statistics.mean(ms)
    assert hga.device_status() == 0
    pk = peaks()
    alg = statistics.mean(decode_algorithmic(wd, pos0 + i)["bytes"] for i in range(63)) * L
    achieved = alg / (ms_tok * 1e-3) / 1e9
    line = dict(metric=f"HGA decode tokens/s at 16K ctx through {L} attention layers per token",
                value=wd.B / (ms_tok * 1e-3), unit="tokens/s", n_gpus=1, steps=n, warmup=args.warmup,
                ms_per_step=ms_tok, higher_is_better=True, scaling="weak", vs_baseline=None, dtype=wd.dtype,
                data="synthetic",
                config=dict(config_of(wd, graph=False), mode="decode_layers", decode_batch=wd.B, layers=L,
                            positions=f"{pos0}..{wd.T - 1}, summaries appended at chunk end",
                            l2="flushed before every token (256 MiB write)",
                            launch="one CUDA graph per token position (L decode calls), events around its replay"),
                us_per_layer=ms_tok * 1e3 / L,
                roofline=dict(bound="hbm", achieved=achieved, peak=pk["hbm_gbs"], unit="GB/s",
                              frac=achieved / pk["hbm_gbs"], traffic=None, kernel="decode_kernel",
                              algorithmic_bytes_per_step=alg, peak_source=pk["source"] + " (burst copy)"),
                gpu_launches=sum(L + (L if (pos0 + i % 64 + 1) % 64 == 0 else 0) for i in range(n)),
                clocks=clk.summary())
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["hga", "reference"], default="hga")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.BY_NAME))
    ap.add_argument("--ref-seconds", type=float, default=10.0,
                    help="seconds of oracle work in the CPU baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="time eager launches instead of a CUDA graph of the step")
    ap.add_argument("--layer", action="store_true",
                    help="segment-wise training of one attention layer with HGA (f4 integration)")
    ap.add_argument("--kv-tier", choices=["hbm", "host"], default="hbm",
                    help="host: history K/V in pinned host memory, routed groups staged per step")
    ap.add_argument("--causal", action="store_true",
                    help="the strictly causal variant: routing per query position (f1)")
    ap.add_argument("--decode", action="store_true",
                    help="generation: one hga_decode step per token over the workload's context (f3)")
    ap.add_argument("--decode-batch", type=int, default=1, help="sequences decoded per step")
    ap.add_argument("--decode-layers", type=int, default=1,
                    help="attention layers per decoded token (one cache each; a CUDA graph per token)")
    ap.add_argument("--clocks-csv", default=None,
                    help="also write the nvidia-smi samples of the timed region to this file")
    ap.add_argument("--traffic", type=float, default=None,
                    help="ncu DRAM bytes per launch of the dominant kernel, if captured")
    args = ap.parse_args()
    w = W.BY_NAME[args.workload]
    if args.impl == "reference":
        run_reference(args, w)
    elif args.causal:
        run_causal(args, w)
    elif args.decode:
        run_decode(args, w)
    elif args.layer:
        run_layer(args, w)
    elif args.kv_tier == "host":
        run_host_tier(args, w)
    else:
        run_gpu(args, w)


if __name__ == "__main__":
    main()
