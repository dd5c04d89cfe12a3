"""HGA as a drop-in attention module trained segment by segment.

Article "BMW's 16 GB GPU just did what needs an A100" (seventnews.com),
section "What HGA does differently": HGA replaces the attention module; a
long sequence is trained in segments, each segment attends the exact tokens
of earlier segments through the router, and older KV is detached -- no
gradient flows into earlier segments.

``HGAAttention`` is the autograd function of one segment: its forward runs
the segment's summaries, then the routing and the routed attention forward
in one persistent launch (hga_route_attn_fwd); its backward runs the routed backward with the forward's routing
frozen and returns gradients for the segment's Q, K and V (history gets
none).  ``HGASegmentLayer`` wraps it between real Q / K / V / O projections
and keeps the KV cache and the summaries of the segments seen so far in
buffers that grow by doubling (the library reads them in place);
``run_tbptt`` trains a sequence segment by segment (truncated
back-propagation through time).
"""
from __future__ import annotations

import math

import torch
from torch import nn

from . import binding as B


class KVCache:
    """History of one layer, kept in preallocated buffers that grow by
    doubling: K / V [B][Hkv][cap][d] (rows 0 .. n-1 in use, no gradient) and
    their chunk / group summaries [B][Hkv][cap/64][d], [B][Hkv][cap/8][d].
    A segment writes only its own rows, and the library reads the buffers in
    place (hga_params.kv_capacity = cap), so a sequence of segments costs no
    copies of the history beyond the occasional doubling."""

    def __init__(self):
        self.K = self.V = self.csum = self.gsum = None
        self.n = 0

    @property
    def T_hist(self) -> int:
        return self.n

    @property
    def cap(self) -> int:
        return 0 if self.K is None else self.K.shape[2]

    def reset(self):
        self.__init__()

    @torch.no_grad()
    def reserve(self, B: int, Hkv: int, d: int, dtype, rows: int, device):
        """Capacity for `rows` rows (a multiple of 64), keeping the rows in use."""
        if self.K is not None and self.K.shape[2] >= rows:
            return
        cap = max(rows, 2 * self.cap)
        K = torch.empty(B, Hkv, cap, d, device=device, dtype=dtype)
        V = torch.empty_like(K)
        csum = torch.zeros(B, Hkv, cap // 64, d, device=device, dtype=torch.float32)
        gsum = torch.zeros(B, Hkv, cap // 8, d, device=device, dtype=torch.float32)
        if self.n:
            K[:, :, :self.n] = self.K[:, :, :self.n]
            V[:, :, :self.n] = self.V[:, :, :self.n]
            csum[:, :, :self.n // 64] = self.csum[:, :, :self.n // 64]
            gsum[:, :, :self.n // 8] = self.gsum[:, :, :self.n // 8]
        self.K, self.V, self.csum, self.gsum = K, V, csum, gsum


class _SegmentBuffers:
    """Per-segment outputs and scratch of one shape, reused segment after
    segment (their sizes depend on the segment length and the routing
    widths, not on the history)."""

    def __init__(self, p: B.Params, device):
        wc, wg = B.route_widths(p)
        Bn, Hq, Hkv, d, Ts, nQB = p.B, p.Hq, p.Hkv, p.d, p.T_seg, p.nQB
        f32 = dict(device=device, dtype=torch.float32)
        i32 = dict(device=device, dtype=torch.int32)
        self.key = (Bn, Hq, Hkv, d, Ts, wc, wg)
        self.qbar = torch.empty(Bn, Hkv, nQB, d, **f32)
        self.cidx = torch.empty(Bn, Hkv, nQB, wc, **i32)
        self.gidx = torch.empty(Bn, Hkv, nQB, wg, **i32)
        self.O = torch.empty(Bn, Hq, Ts, d, **f32)
        self.lse = torch.empty(Bn, Hq, Ts, **f32)
        self.dQ = torch.empty(Bn, Hq, Ts, d, **f32)
        self.dK = torch.empty(Bn, Hkv, Ts, d, **f32)
        self.dV = torch.empty(Bn, Hkv, Ts, d, **f32)
        self.ws = torch.empty(max(1, math.ceil(B.workspace_size(p) / 4)), **f32)


class HGAAttention(torch.autograd.Function):
    """O = routed attention of the segment's queries over the history and the
    segment's own keys (forward of libhga); float32 output.  The segment's
    keys and values are written into the cache (rows T_hist .. T_hist + T_seg)
    before the routing; the caller then advances the cache by T_seg rows."""

    @staticmethod
    def forward(ctx, q, k, v, cache: KVCache, k_c: int, k_g: int, bufs: dict):
        Bn, Hq, Ts, d = q.shape
        Hkv = k.shape[1]
        dtype = B.HGA_BF16 if q.dtype == torch.bfloat16 else B.HGA_FP32
        T_hist = cache.n
        cache.reserve(Bn, Hkv, d, q.dtype, T_hist + Ts, q.device)
        p = B.Params(B=Bn, Hq=Hq, Hkv=Hkv, d=d, T_hist=T_hist, T_seg=Ts, k_c=k_c, k_g=k_g, dtype=dtype,
                     kv_capacity=cache.cap)
        q = q.contiguous()
        with torch.no_grad():
            cache.K[:, :, T_hist:T_hist + Ts] = k
            cache.V[:, :, T_hist:T_hist + Ts] = v
        wc, wg = B.route_widths(p)
        key = (Bn, Hq, Hkv, d, Ts, wc, wg)
        buf = bufs.get(key)
        if buf is None or buf.ws.numel() * 4 < B.workspace_size(p):
            buf = bufs[key] = _SegmentBuffers(p, q.device)
        # The segment's summaries go next to the history's, in the cache.
        B.build_summaries_rows(p, k.detach().contiguous(), T_hist, T_hist + Ts, cache.csum, cache.gsum)
        # Routing and forward in one persistent launch (bf16; the same results as
        # hga_route then hga_attn_fwd, which other shapes run).
        B.route_attn_fwd(p, q, cache.K, cache.V, cache.csum, cache.gsum, buf.qbar, buf.cidx, buf.gidx, buf.O,
                         buf.lse)
        O, lse, gidx = buf.O.clone(), buf.lse.clone(), buf.gidx.clone()
        ctx.p, ctx.buf = p, buf
        ctx.K, ctx.V = cache.K, cache.V          # the buffers this segment's rows live in
        ctx.save_for_backward(q, O, lse, gidx)
        ctx.dtypes = (q.dtype, k.dtype, v.dtype)
        ctx.mark_non_differentiable(gidx)
        return O, gidx

    @staticmethod
    def backward(ctx, dO, _dgidx):
        q, O, lse, gidx = ctx.saved_tensors
        buf, p = ctx.buf, ctx.p
        dO = dO.to(q.dtype).contiguous()
        B.attn_bwd(p, q, ctx.K, ctx.V, O, lse, dO, gidx, buf.dQ, buf.dK, buf.dV, buf.ws)
        tq, tk, tv = ctx.dtypes
        return (buf.dQ.to(tq, copy=True), buf.dK.to(tk, copy=True), buf.dV.to(tv, copy=True),
                None, None, None, None)


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
        self.bufs = {}                                # per-segment buffers, by shape
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
        O, gidx = HGAAttention.apply(q, k, v, self.cache, self.k_c, self.k_g, self.bufs)
        self.cache.n += Ts                            # the segment's rows join the history
        self.last_gidx = gidx
        return self.wo(O.transpose(1, 2).reshape(Bn, Ts, self.Hq * self.d))


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
