"""Segment steps fed from host memory, with the copies overlapped.

A training loop that keeps its inputs on the host pays, every step, the
host->device copies of the segment's Q, K, V rows and dO and the
device->host copies of the gradients.  ``StepPipeline`` runs those copies on
their own streams (the GPU's copy engines) and keeps two device buffer sets,
so that while step i computes, the inputs of step i+1 are uploaded and the
gradients of step i-1 are downloaded: in steady state a step costs the
longest of the three instead of their sum.  Every step still moves all its
bytes both ways; only the overlap changes.

The compute of a step is ``Buffers.step`` (segment summaries, routing,
forward and backward of the routed attention) on the library's kernels.
"""
from __future__ import annotations

import torch

from . import binding as B


class StepPipeline:
    """Overlapped host->device, compute and device->host of segment steps.

    p       problem shape (``Params``); history rows ``T_hist`` stay resident.
    K_hist, V_hist  device tensors [B][Hkv][T_hist][d] of the history rows
            (copied into both buffer sets once; their summaries are built once).
    Host tensors given to ``submit`` must be pinned for the copies to be
    asynchronous.
    """

    def __init__(self, p: B.Params, K_hist, V_hist, device="cuda"):
        self.p = p
        dev = torch.device(device)
        dt = p.torch_dtype
        Bn, Hq, Hkv, d, T, Th, Ts = p.B, p.Hq, p.Hkv, p.d, p.T, p.T_hist, p.T_seg
        self.s_in = torch.cuda.Stream(dev)
        self.s_cmp = torch.cuda.Stream(dev)
        self.s_out = torch.cuda.Stream(dev)
        self.sets = []
        for _ in range(2):
            K = torch.empty(Bn, Hkv, T, d, device=dev, dtype=dt)
            V = torch.empty(Bn, Hkv, T, d, device=dev, dtype=dt)
            K[:, :, :Th] = K_hist
            V[:, :, :Th] = V_hist
            buf = B.Buffers(p, device=dev)
            buf.summaries(K, 0, Th)                  # history summaries persist
            self.sets.append(dict(
                Q=torch.empty(Bn, Hq, Ts, d, device=dev, dtype=dt), K=K, V=V,
                Kseg=torch.empty(Bn, Hkv, Ts, d, device=dev, dtype=dt),
                Vseg=torch.empty(Bn, Hkv, Ts, d, device=dev, dtype=dt),
                dO=torch.empty(Bn, Hq, Ts, d, device=dev, dtype=dt), buf=buf,
                in_done=torch.cuda.Event(), cmp_done=torch.cuda.Event(), out_done=torch.cuda.Event(),
                used=False))
        torch.cuda.synchronize(dev)
        self.n = 0

    def submit(self, Qh, Kh_seg, Vh_seg, dOh, outs_h) -> None:
        """Enqueue one step: Qh, dOh [B][Hq][T_seg][d] and Kh_seg, Vh_seg
        [B][Hkv][T_seg][d] on the host (pinned); the step's dQ, dK_seg,
        dV_seg land in outs_h = (dQ, dK, dV) host tensors (pinned, float32).
        Returns at once; ``synchronize`` (or an event) waits for the step."""
        S = self.sets[self.n % 2]
        p = self.p
        Th = p.T_hist
        # Inputs of this set are free once the step two back has computed.
        if S["used"]:
            self.s_in.wait_event(S["cmp_done"])
        with torch.cuda.stream(self.s_in):
            # Four contiguous uploads; the segment rows then move into the
            # caches' strided slots on the device.
            S["Q"].copy_(Qh, non_blocking=True)
            S["dO"].copy_(dOh, non_blocking=True)
            S["Kseg"].copy_(Kh_seg, non_blocking=True)
            S["Vseg"].copy_(Vh_seg, non_blocking=True)
            S["K"][:, :, Th:].copy_(S["Kseg"])
            S["V"][:, :, Th:].copy_(S["Vseg"])
            S["in_done"].record(self.s_in)
        # Outputs of this set are free once the step two back is downloaded.
        self.s_cmp.wait_event(S["in_done"])
        if S["used"]:
            self.s_cmp.wait_event(S["out_done"])
        buf = S["buf"]
        buf.step(S["Q"], S["K"], S["V"], S["dO"], stream=self.s_cmp)
        S["cmp_done"].record(self.s_cmp)
        self.s_out.wait_event(S["cmp_done"])
        with torch.cuda.stream(self.s_out):
            for hst, dv in zip(outs_h, (buf.dQ, buf.dK, buf.dV)):
                hst.copy_(dv, non_blocking=True)
            S["out_done"].record(self.s_out)
        S["used"] = True
        self.n += 1

    def last_done_event(self) -> torch.cuda.Event:
        """Event completed when the last submitted step's outputs are on the host."""
        return self.sets[(self.n - 1) % 2]["out_done"]

    def synchronize(self) -> None:
        self.s_out.synchronize()
