"""HGA as a drop-in attention module trained segment by segment.

Article "BMW's 16 GB GPU just did what needs an A100" (seventnews.com),
section "What HGA does differently": HGA replaces the attention module; a
long sequence is trained in segments, each segment attends the exact tokens
of earlier segments through the router, and older KV is detached -- no
gradient flows into earlier segments.

``HGAAttention`` is the autograd function of one segment: its forward runs
the segment's summaries, the routing and the routed attention forward of
libhga; its backward runs the routed backward with the forward's routing
frozen and returns gradients for the segment's Q, K and V (history gets
none).  ``HGASegmentLayer`` wraps it between real Q / K / V / O projections
and keeps the KV cache and the summaries of the segments seen so far;
``run_tbptt`` trains a sequence segment by segment (truncated
back-propagation through time).
"""
from __future__ import annotations

import math

import torch
from torch import nn

from . import binding as B


class KVCache:
    """History of one layer: K / V rows [B][Hkv][T_hist][d] (no gradient)
    and their chunk / group summaries."""

    def __init__(self):
        self.K = None
        self.V = None
        self.csum = None
        self.gsum = None
        self.pending = None      # summaries including the segment in flight

    @property
    def T_hist(self) -> int:
        return 0 if self.K is None else self.K.shape[2]

    def reset(self):
        self.__init__()


class HGAAttention(torch.autograd.Function):
    """O = routed attention of the segment's queries over the history and the
    segment's own keys (forward of libhga); float32 output."""

    @staticmethod
    def forward(ctx, q, k, v, cache: KVCache, k_c: int, k_g: int):
        Bn, Hq, Ts, d = q.shape
        Hkv = k.shape[1]
        dtype = B.HGA_BF16 if q.dtype == torch.bfloat16 else B.HGA_FP32
        p = B.Params(B=Bn, Hq=Hq, Hkv=Hkv, d=d, T_hist=cache.T_hist, T_seg=Ts, k_c=k_c, k_g=k_g, dtype=dtype)
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        Kall = k if cache.K is None else torch.cat([cache.K, k.detach()], dim=2).contiguous()
        Vall = v if cache.V is None else torch.cat([cache.V, v.detach()], dim=2).contiguous()
        buf = B.Buffers(p, device=q.device)
        if cache.csum is not None:                    # history summaries are kept
            buf.csum[:, :, :cache.csum.shape[2]] = cache.csum
            buf.gsum[:, :, :cache.gsum.shape[2]] = cache.gsum
        B.build_summaries_rows(p, k.detach(), p.T_hist, p.T, buf.csum, buf.gsum)
        buf.route(q)
        buf.forward(q, Kall, Vall)
        ctx.p = p
        ctx.buf = buf
        ctx.save_for_backward(q, Kall, Vall)
        ctx.dtypes = (q.dtype, k.dtype, v.dtype)
        # Summaries of history + segment: the cache takes them when the
        # layer appends the segment.
        cache.pending = (buf.csum, buf.gsum)
        gidx = buf.gidx.clone()
        ctx.mark_non_differentiable(gidx)
        return buf.O.clone(), gidx

    @staticmethod
    def backward(ctx, dO, _dgidx):
        q, Kall, Vall = ctx.saved_tensors
        buf, p = ctx.buf, ctx.p
        dO = dO.to(q.dtype).contiguous()
        buf.backward(q, Kall, Vall, dO)
        tq, tk, tv = ctx.dtypes
        return buf.dQ.to(tq), buf.dK.to(tk), buf.dV.to(tv), None, None, None


class HGASegmentLayer(nn.Module):
    """Attention layer with HGA routed attention: x -> Wq, Wk, Wv (GQA) ->
    HGA -> Wo.  Call ``segment`` once per segment; the layer's KV cache grows
    by the segment's (detached) keys and values after each call."""

    def __init__(self, d_model: int, Hq: int, Hkv: int, d: int, k_c: int = 8, k_g: int = 32,
                 dtype=torch.bfloat16, device="cuda"):
        super().__init__()
        self.Hq, self.Hkv, self.d, self.k_c, self.k_g = Hq, Hkv, d, k_c, k_g
        self.act_dtype = dtype
        kw = dict(bias=False, device=device, dtype=torch.float32)
        self.wq = nn.Linear(d_model, Hq * d, **kw)
        self.wk = nn.Linear(d_model, Hkv * d, **kw)
        self.wv = nn.Linear(d_model, Hkv * d, **kw)
        self.wo = nn.Linear(Hq * d, d_model, **kw)
        for m in (self.wq, self.wk, self.wv, self.wo):
            nn.init.normal_(m.weight, std=1.0 / math.sqrt(m.in_features))
        self.cache = KVCache()
        self.last_gidx = None

    def project(self, x):
        """Q [B][Hq][Ts][d], K, V [B][Hkv][Ts][d] of a segment x [B][Ts][d_model]."""
        Bn, Ts, _ = x.shape
        q = self.wq(x).view(Bn, Ts, self.Hq, self.d).transpose(1, 2)
        k = self.wk(x).view(Bn, Ts, self.Hkv, self.d).transpose(1, 2)
        v = self.wv(x).view(Bn, Ts, self.Hkv, self.d).transpose(1, 2)
        return (q.to(self.act_dtype).contiguous(), k.to(self.act_dtype).contiguous(),
                v.to(self.act_dtype).contiguous())

    def segment(self, x):
        Bn, Ts, _ = x.shape
        q, k, v = self.project(x)
        O, gidx = HGAAttention.apply(q, k, v, self.cache, self.k_c, self.k_g)
        self.last_gidx = gidx
        out = self.wo(O.transpose(1, 2).reshape(Bn, Ts, self.Hq * self.d))
        self._append(k.detach(), v.detach())
        return out

    @torch.no_grad()
    def _append(self, k, v):
        c = self.cache
        c.K = k.clone() if c.K is None else torch.cat([c.K, k], dim=2).contiguous()
        c.V = v.clone() if c.V is None else torch.cat([c.V, v], dim=2).contiguous()
        c.csum, c.gsum = c.pending                    # built by the segment's forward
        c.pending = None


def run_tbptt(layer: HGASegmentLayer, x, target, seg_len: int, optimizer=None):
    """Train over x [B][T][d_model] segment by segment: per segment, the loss
    0.5 * |layer(x_seg) - target_seg|^2 / n is back-propagated (history
    detached); returns the per-segment losses."""
    layer.cache.reset()
    losses = []
    for s in range(0, x.shape[1], seg_len):
        xs, ts = x[:, s:s + seg_len], target[:, s:s + seg_len]
        out = layer.segment(xs)
        loss = 0.5 * (out - ts).pow(2).mean()
        loss.backward()
        if optimizer is not None:
            optimizer.step()
            optimizer.zero_grad(set_to_none=True)
        losses.append(float(loss.detach()))
    return losses
