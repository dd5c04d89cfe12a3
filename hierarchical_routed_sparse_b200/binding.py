"""Thin ctypes binding of libhga.so (the C ABI declared in include/hga.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libhga.so.  torch provides the device memory (tensors are passed
by data pointer) and the stream (the current torch stream unless one is
given).  There is no fallback: if the library is missing or fails to load,
every call raises.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
import os
from dataclasses import dataclass

import torch

HGA_OK, HGA_ERR_INVALID_ARG, HGA_ERR_UNSUPPORTED, HGA_ERR_CUDA, HGA_ERR_DEVICE_CHECK = 0, 1, 2, 3, 4
HGA_ALL = -1
HGA_BF16, HGA_FP32 = 0, 1

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhga.so")
# The bounds-checked build of the same library (-DHGA_CHECK_BOUNDS).
CHECKED_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhga_checked.so")

EXPORTS = ("hga_route_widths", "hga_workspace_size", "hga_build_summaries", "hga_build_summaries_rows",
           "hga_route_chunks",
           "hga_route_groups", "hga_route", "hga_attn_fwd", "hga_route_attn_fwd", "hga_attn_bwd", "hga_attn_bwd_noalloc",
           "hga_stage_params", "hga_stage_routed", "hga_decode", "hga_route_causal", "hga_causal_sched_size",
           "hga_causal_schedule", "hga_attn_fwd_causal", "hga_attn_bwd_causal", "hga_device_status", "hga_device_check", "hga_checked_build",
           "hga_selftest_wait", "hga_last_error",
           "hga_version")
NOALLOC_MAX_ROWS = 1 << 20     # HGA_NOALLOC_MAX_ROWS


class HGAError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"[hga error {code}] {msg}")
        self.code = code


class _Params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("d", ctypes.c_int), ("T_hist", ctypes.c_int64), ("T_seg", ctypes.c_int64),
                ("chunk", ctypes.c_int), ("group", ctypes.c_int), ("qblock", ctypes.c_int),
                ("k_c", ctypes.c_int), ("k_g", ctypes.c_int), ("scale", ctypes.c_float),
                ("dtype", ctypes.c_int), ("kv_capacity", ctypes.c_int64)]


@dataclass
class Params:
    """Mirror of hga_params.  k_c / k_g may be HGA_ALL (-1)."""
    B: int
    Hq: int
    Hkv: int
    d: int
    T_hist: int
    T_seg: int
    k_c: int
    k_g: int
    dtype: int = HGA_BF16
    scale: float = 0.0
    chunk: int = 64
    group: int = 8
    qblock: int = 64
    kv_capacity: int = 0     # rows per (batch, kv-head) of K / V / summaries; 0 = T

    @staticmethod
    def from_workload(w) -> "Params":
        return Params(B=w.B, Hq=w.Hq, Hkv=w.Hkv, d=w.d, T_hist=w.T_hist, T_seg=w.T_seg,
                      k_c=w.k_c, k_g=w.k_g, dtype=HGA_BF16 if w.dtype == "bf16" else HGA_FP32)

    @property
    def T(self) -> int:
        return self.T_hist + self.T_seg

    @property
    def nQB(self) -> int:
        return self.T_seg // 64

    @property
    def cap(self) -> int:
        """Rows per (batch, kv-head) of the K / V buffers (and 64x / 8x the
        rows of the chunk / group summaries)."""
        return self.kv_capacity or self.T

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == HGA_BF16 else torch.float32

    def c(self) -> _Params:
        return _Params(self.B, self.Hq, self.Hkv, self.d, self.T_hist, self.T_seg, self.chunk,
                       self.group, self.qblock, self.k_c, self.k_g, float(self.scale), self.dtype,
                       self.kv_capacity)


_lib = None


def load() -> ctypes.CDLL:
    """Load libhga.so (built by hierarchical_routed_sparse_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m hierarchical_routed_sparse_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        P, I64 = ctypes.c_void_p, ctypes.c_int64
        PP = ctypes.POINTER(_Params)
        sig = {
            "hga_route_widths": ([PP, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)],
                                 ctypes.c_int),
            "hga_workspace_size": ([PP], ctypes.c_size_t),
            "hga_build_summaries": ([PP, P, I64, I64, P, P, P], ctypes.c_int),
            "hga_build_summaries_rows": ([PP, P, I64, I64, P, P, P], ctypes.c_int),
            "hga_route_chunks": ([PP, P, P, P, P, P], ctypes.c_int),
            "hga_route_groups": ([PP, P, P, P, P, P], ctypes.c_int),
            "hga_route": ([PP, P, P, P, P, P, P, P], ctypes.c_int),
            "hga_attn_fwd": ([PP, P, P, P, P, P, P, P], ctypes.c_int),
            "hga_route_attn_fwd": ([PP, P, P, P, P, P, P, P, P, P, P, P], ctypes.c_int),
            "hga_attn_bwd": ([PP, P, P, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P],
                             ctypes.c_int),
            "hga_attn_bwd_noalloc": ([PP, P, P, P, P, P, P, P, P, P, P, P], ctypes.c_int),
            "hga_stage_params": ([PP, PP], ctypes.c_int),
            "hga_stage_routed": ([PP, P, P, P, P, P, P, P, P, P], ctypes.c_int),
            "hga_decode": ([PP, I64, P, P, P, P, P, P, P, P, P, P], ctypes.c_int),
            "hga_route_causal": ([PP, P, P, P, P, P, P], ctypes.c_int),
            "hga_causal_sched_size": ([PP], ctypes.c_size_t),
            "hga_causal_schedule": ([PP, P, P, P], ctypes.c_int),
            "hga_attn_fwd_causal": ([PP, P, P, P, P, P, P, P, P], ctypes.c_int),
            "hga_attn_bwd_causal": ([PP, P, P, P, P, P, P, P, P, P, P, P, P], ctypes.c_int),
            "hga_device_status": ([ctypes.POINTER(ctypes.c_int), ctypes.c_int], ctypes.c_int),
            "hga_selftest_wait": ([ctypes.c_int, ctypes.POINTER(ctypes.c_int), P], ctypes.c_int),
            "hga_device_check": ([ctypes.POINTER(ctypes.c_int), ctypes.c_int], ctypes.c_int),
            "hga_checked_build": ([], ctypes.c_int),
            "hga_last_error": ([], ctypes.c_char_p),
            "hga_version": ([], ctypes.c_char_p),
        }
        for name, (args, res) in sig.items():
            f = getattr(lib, name)
            f.argtypes, f.restype = args, res
        _lib = lib
    return _lib


def _check(code: int) -> None:
    if code != HGA_OK:
        raise HGAError(code, load().hga_last_error().decode())


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libhga takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libhga takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def version() -> str:
    return load().hga_version().decode()


def device_status(clear: bool = False) -> int:
    """Status word of the kernels' bounded waits (0: none ran out).  Syncs."""
    v = ctypes.c_int()
    _check(load().hga_device_status(ctypes.byref(v), int(clear)))
    return v.value


def use_library(path: str) -> None:
    """Route every later call through the library at `path` (for instance
    CHECKED_LIB_PATH, the bounds-checked build); the next call loads it."""
    global _lib, LIB_PATH
    LIB_PATH = path
    _lib = None


def checked_build() -> bool:
    """Whether the loaded library checks index rows on the device."""
    return bool(load().hga_checked_build())


def device_check(clear: bool = False) -> int:
    """First failed device bounds check's site code (0: none).  Syncs."""
    v = ctypes.c_int()
    _check(load().hga_device_check(ctypes.byref(v), int(clear)))
    return v.value


def selftest_wait(limit_us: int, stream=None) -> int:
    """Launch the failure-path self-test (a bounded wait that runs out after
    limit_us); returns the code it records in the status word."""
    site = ctypes.c_int()
    _check(load().hga_selftest_wait(int(limit_us), ctypes.byref(site), _stream(stream)))
    return site.value


def route_widths(p: Params) -> tuple[int, int]:
    wc, wg = ctypes.c_int(), ctypes.c_int()
    _check(load().hga_route_widths(ctypes.byref(p.c()), ctypes.byref(wc), ctypes.byref(wg)))
    return wc.value, wg.value


def workspace_size(p: Params) -> int:
    return int(load().hga_workspace_size(ctypes.byref(p.c())))


def build_summaries(p: Params, K, t_begin: int, t_end: int, csum, gsum, stream=None) -> None:
    _check(load().hga_build_summaries(ctypes.byref(p.c()), _ptr(K), t_begin, t_end, _ptr(csum),
                                      _ptr(gsum), _stream(stream)))


def build_summaries_rows(p: Params, K_rows, t_begin: int, t_end: int, csum, gsum, stream=None) -> None:
    """Summaries of tokens [t_begin, t_end) from a K holding only those rows."""
    _check(load().hga_build_summaries_rows(ctypes.byref(p.c()), _ptr(K_rows), t_begin, t_end, _ptr(csum),
                                           _ptr(gsum), _stream(stream)))


def route_chunks(p: Params, Q, csum, qbar, cidx, stream=None) -> None:
    _check(load().hga_route_chunks(ctypes.byref(p.c()), _ptr(Q), _ptr(csum), _ptr(qbar), _ptr(cidx),
                                   _stream(stream)))


def route_groups(p: Params, qbar, gsum, cidx, gidx, stream=None) -> None:
    _check(load().hga_route_groups(ctypes.byref(p.c()), _ptr(qbar), _ptr(gsum), _ptr(cidx),
                                   _ptr(gidx), _stream(stream)))


def route(p: Params, Q, csum, gsum, qbar, cidx, gidx, stream=None) -> None:
    """Block queries, chunk routing and group routing in one launch."""
    _check(load().hga_route(ctypes.byref(p.c()), _ptr(Q), _ptr(csum), _ptr(gsum), _ptr(qbar), _ptr(cidx),
                            _ptr(gidx), _stream(stream)))


def attn_fwd(p: Params, Q, K, V, gidx, O, lse, stream=None) -> None:
    _check(load().hga_attn_fwd(ctypes.byref(p.c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(gidx), _ptr(O),
                               _ptr(lse), _stream(stream)))


def route_attn_fwd(p: Params, Q, K, V, csum, gsum, qbar, cidx, gidx, O, lse, stream=None) -> None:
    """hga_route followed by hga_attn_fwd, as one persistent launch (bf16)."""
    _check(load().hga_route_attn_fwd(ctypes.byref(p.c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(csum), _ptr(gsum),
                                     _ptr(qbar), _ptr(cidx), _ptr(gidx), _ptr(O), _ptr(lse), _stream(stream)))


def attn_bwd(p: Params, Q, K, V, O, lse, dO, gidx, dQ, dK_seg, dV_seg, workspace,
             stream=None) -> None:
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(load().hga_attn_bwd(ctypes.byref(p.c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse),
                               _ptr(dO), _ptr(gidx), _ptr(dQ), _ptr(dK_seg), _ptr(dV_seg),
                               _ptr(workspace), ws_bytes, _stream(stream)))


def attn_bwd_noalloc(p: Params, Q, K, V, O, lse, dO, gidx, dQ, dK_seg, dV_seg,
                     stream=None) -> None:
    """hga_attn_bwd with the library's built-in scratch instead of a workspace.

    For callers that cannot pass scratch memory (plugin interfaces that give
    an operator only its inputs and outputs, hosts whose pool owns all device
    memory, loops that must not call cudaMalloc / cudaFree).  Limited to
    B*Hq*T_seg <= NOALLOC_MAX_ROWS; calls that overlap on the GPU share one
    scratch array and race, so keep them on one stream.
    """
    _check(load().hga_attn_bwd_noalloc(ctypes.byref(p.c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                                       _ptr(lse), _ptr(dO), _ptr(gidx), _ptr(dQ), _ptr(dK_seg),
                                       _ptr(dV_seg), _stream(stream)))


def stage_params(p: Params) -> Params:
    """The parameter block of the staged problem (host-RAM KV tier): p with
    T_hist replaced by the staged history rows round_up_64(nQB * wg * 8) and
    k_c, k_g by p's index-row widths (so HGA_ALL keeps the same widths)."""
    out = _Params()
    _check(load().hga_stage_params(ctypes.byref(p.c()), ctypes.byref(out)))
    return dataclasses.replace(p, T_hist=int(out.T_hist), k_c=int(out.k_c), k_g=int(out.k_g))


def _hist_ptr(t: torch.Tensor | None):
    """History rows may be a device tensor or a pinned host tensor."""
    if t is None or t.numel() == 0:                  # no history rows (T_hist = 0)
        return None
    if not t.is_contiguous():
        raise ValueError("libhga takes contiguous tensors")
    if not t.is_cuda and not t.is_pinned():
        raise ValueError("host-resident history must be in pinned memory")
    return ctypes.c_void_p(t.data_ptr())


def stage_routed(p: Params, K_hist, V_hist, K_seg, V_seg, gidx, K_stage, V_stage, gidx_stage,
                 stream=None) -> None:
    """Gather the routed history groups into K_stage / V_stage and remap gidx."""
    _check(load().hga_stage_routed(ctypes.byref(p.c()), _hist_ptr(K_hist), _hist_ptr(V_hist), _ptr(K_seg),
                                   _ptr(V_seg), _ptr(gidx), _ptr(K_stage), _ptr(V_stage), _ptr(gidx_stage),
                                   _stream(stream)))


def decode(p: Params, pos: int, q, K, V, csum, gsum, O, lse, cidx, gidx, stream=None) -> None:
    """One decode step of the token at position ``pos`` (rows 0..pos of K / V
    valid, summaries of the chunks before pos // 64 built)."""
    _check(load().hga_decode(ctypes.byref(p.c()), int(pos), _ptr(q), _ptr(K), _ptr(V), _ptr(csum), _ptr(gsum),
                             _ptr(O), _ptr(lse), _ptr(cidx), _ptr(gidx), _stream(stream)))


def route_causal(p: Params, Q, csum, gsum, cidx, gidx, stream=None) -> None:
    """Strictly causal routing: one routing row per query position
    (cidx [B][Hkv][T_seg][wc], gidx [B][Hkv][T_seg][wg])."""
    _check(load().hga_route_causal(ctypes.byref(p.c()), _ptr(Q), _ptr(csum), _ptr(gsum), _ptr(cidx), _ptr(gidx),
                                   _stream(stream)))


def causal_sched_size(p: Params) -> int:
    """Bytes of the causal window schedule (int32 [2 * n_items])."""
    return int(load().hga_causal_sched_size(ctypes.byref(p.c())))


def causal_schedule(p: Params, gidx, sched, stream=None) -> None:
    """Order the causal attention's window items heaviest first (sched[:n]),
    their costs in sched[n:]."""
    _check(load().hga_causal_schedule(ctypes.byref(p.c()), _ptr(gidx), _ptr(sched), _stream(stream)))


def attn_fwd_causal(p: Params, Q, K, V, gidx, O, lse, stream=None, sched=None) -> None:
    _check(load().hga_attn_fwd_causal(ctypes.byref(p.c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(gidx), _ptr(sched),
                                      _ptr(O), _ptr(lse), _stream(stream)))


def attn_bwd_causal(p: Params, Q, K, V, O, lse, dO, gidx, dQ, dK_seg, dV_seg, stream=None, sched=None) -> None:
    _check(load().hga_attn_bwd_causal(ctypes.byref(p.c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(O), _ptr(lse),
                                      _ptr(dO), _ptr(gidx), _ptr(sched), _ptr(dQ), _ptr(dK_seg), _ptr(dV_seg),
                                      _stream(stream)))


class CausalBuffers:
    """Device buffers of the strictly causal variant for one problem shape:
    routing rows per query position and the attention's window schedule
    (built with the routing, ordering the window items heaviest first);
    ``step`` runs summaries, routing, forward and (with dO) backward."""

    def __init__(self, p: Params, device="cuda"):
        self.p = p
        wc, wg = route_widths(p)
        B, Hq, Hkv, d, T, Ts = p.B, p.Hq, p.Hkv, p.d, p.T, p.T_seg
        f32 = dict(device=device, dtype=torch.float32)
        i32 = dict(device=device, dtype=torch.int32)
        self.csum = torch.zeros(B, Hkv, p.cap // 64, d, **f32)
        self.gsum = torch.zeros(B, Hkv, p.cap // 8, d, **f32)
        self.cidx = torch.empty(B, Hkv, Ts, wc, **i32)
        self.gidx = torch.empty(B, Hkv, Ts, wg, **i32)
        self.O = torch.empty(B, Hq, Ts, d, **f32)
        self.lse = torch.empty(B, Hq, Ts, **f32)
        self.dQ = torch.empty(B, Hq, Ts, d, **f32)
        self.dK = torch.empty(B, Hkv, Ts, d, **f32)
        self.dV = torch.empty(B, Hkv, Ts, d, **f32)
        self.sched = torch.empty(max(1, causal_sched_size(p) // 4), **i32)
        self.sched_of = None          # the index rows the schedule was built from

    def summaries(self, K, t_begin=None, t_end=None, stream=None):
        t_begin = self.p.T_hist if t_begin is None else t_begin
        t_end = self.p.T if t_end is None else t_end
        build_summaries(self.p, K, t_begin, t_end, self.csum, self.gsum, stream)

    def route(self, Q, stream=None):
        route_causal(self.p, Q, self.csum, self.gsum, self.cidx, self.gidx, stream)
        self.schedule(self.gidx, stream)

    def schedule(self, gidx, stream=None):
        """The window schedule of index rows `gidx` (any permutation gives the
        same results; one built from the rows the attention runs on is the
        balanced one)."""
        causal_schedule(self.p, gidx, self.sched, stream)
        self.sched_of = gidx

    def _sched_for(self, gidx):
        return self.sched if self.sched_of is gidx else None

    def forward(self, Q, K, V, gidx=None, stream=None):
        gidx = self.gidx if gidx is None else gidx
        attn_fwd_causal(self.p, Q, K, V, gidx, self.O, self.lse, stream, sched=self._sched_for(gidx))

    def backward(self, Q, K, V, dO, gidx=None, stream=None):
        gidx = self.gidx if gidx is None else gidx
        attn_bwd_causal(self.p, Q, K, V, self.O, self.lse, dO, gidx, self.dQ, self.dK, self.dV, stream,
                        sched=self._sched_for(gidx))

    def step(self, Q, K, V, dO=None, stream=None):
        self.summaries(K, stream=stream)
        self.route(Q, stream)
        self.forward(Q, K, V, stream=stream)
        if dO is not None:
            self.backward(Q, K, V, dO, stream=stream)


class DecodeState:
    """Generation with HGA: a KV cache of ``p.T`` rows and its summaries.

    ``prefill`` fills the first rows; each ``step`` writes the new token's
    K / V row, runs hga_decode for it, and appends the summaries of its chunk
    once the chunk's 64 tokens are in the cache."""

    def __init__(self, p: Params, device="cuda"):
        self.p = p
        wc, wg = route_widths(p)
        B, Hq, Hkv, d, T = p.B, p.Hq, p.Hkv, p.d, p.T
        f32 = dict(device=device, dtype=torch.float32)
        i32 = dict(device=device, dtype=torch.int32)
        self.K = torch.zeros(B, Hkv, p.cap, d, device=device, dtype=p.torch_dtype)
        self.V = torch.zeros(B, Hkv, p.cap, d, device=device, dtype=p.torch_dtype)
        self.csum = torch.zeros(B, Hkv, p.cap // 64, d, **f32)
        self.gsum = torch.zeros(B, Hkv, p.cap // 8, d, **f32)
        self.O = torch.empty(B, Hq, d, **f32)
        self.lse = torch.empty(B, Hq, **f32)
        self.cidx = torch.empty(B, Hkv, wc, **i32)
        self.gidx = torch.empty(B, Hkv, wg, **i32)
        self.pos = 0                               # tokens in the cache

    def prefill(self, K, V, stream=None) -> None:
        """Rows [0, n) of the cache from K, V [B][Hkv][n][d]; summaries of the
        complete chunks among them."""
        n = K.shape[2]
        if n > self.p.T:
            raise ValueError(f"prefill of {n} rows exceeds the cache of {self.p.T}")
        self.K[:, :, :n] = K
        self.V[:, :, :n] = V
        full = n - n % 64
        if full:
            build_summaries(self.p, self.K, 0, full, self.csum, self.gsum, stream)
        self.pos = n

    def step(self, q, k, v, stream=None):
        """Decode the token with queries q [B][Hq][d] and key / value rows
        k, v [B][Hkv][d]; returns O [B][Hq][d] (float32, a view of the
        state's buffer)."""
        pos = self.pos
        if pos >= self.p.T:
            raise ValueError(f"the cache of {self.p.T} rows is full")
        self.K[:, :, pos] = k
        self.V[:, :, pos] = v
        decode(self.p, pos, q, self.K, self.V, self.csum, self.gsum, self.O, self.lse, self.cidx, self.gidx,
               stream)
        if (pos + 1) % 64 == 0:
            build_summaries(self.p, self.K, pos + 1 - 64, pos + 1, self.csum, self.gsum, stream)
        self.pos = pos + 1
        return self.O


class StagedKV:
    """Host-RAM KV tier: history K/V rows stay in (pinned) host memory; after
    routing on the full problem, the routed groups are staged in device
    memory and the attention runs on the staged problem (``ps``), whose
    results equal those of the full problem."""

    def __init__(self, p: Params, device="cuda"):
        self.p = p
        self.ps = stage_params(p)
        _, wg = route_widths(p)
        B, Hkv, d, nQB = p.B, p.Hkv, p.d, p.nQB
        rows = self.ps.T_hist + p.T_seg
        self.K = torch.empty(B, Hkv, rows, d, device=device, dtype=p.torch_dtype)
        self.V = torch.empty(B, Hkv, rows, d, device=device, dtype=p.torch_dtype)
        self.gidx = torch.empty(B, Hkv, nQB, wg, device=device, dtype=torch.int32)

    def stage(self, K_hist, V_hist, K_seg, V_seg, gidx, stream=None) -> None:
        stage_routed(self.p, K_hist, V_hist, K_seg, V_seg, gidx, self.K, self.V, self.gidx, stream)


class Buffers:
    """Device buffers of one problem shape, allocated once with torch.

    ``step`` runs one segment-wise training step of the hot path: the
    summaries of the segment's keys (earlier summaries are kept), chunk and
    group routing, the routed attention forward and its backward.
    """

    def __init__(self, p: Params, device="cuda"):
        self.p = p
        wc, wg = route_widths(p)
        B, Hq, Hkv, d, T, Ts, nQB = p.B, p.Hq, p.Hkv, p.d, p.T, p.T_seg, p.nQB
        f32 = dict(device=device, dtype=torch.float32)
        i32 = dict(device=device, dtype=torch.int32)
        self.csum = torch.zeros(B, Hkv, p.cap // 64, d, **f32)
        self.gsum = torch.zeros(B, Hkv, p.cap // 8, d, **f32)
        self.qbar = torch.empty(B, Hkv, nQB, d, **f32)
        self.cidx = torch.empty(B, Hkv, nQB, wc, **i32)
        self.gidx = torch.empty(B, Hkv, nQB, wg, **i32)
        self.O = torch.empty(B, Hq, Ts, d, **f32)
        self.lse = torch.empty(B, Hq, Ts, **f32)
        self.dQ = torch.empty(B, Hq, Ts, d, **f32)
        self.dK = torch.empty(B, Hkv, Ts, d, **f32)
        self.dV = torch.empty(B, Hkv, Ts, d, **f32)
        self.ws = torch.empty(max(1, math.ceil(workspace_size(p) / 4)), **f32)

    def summaries(self, K, t_begin=None, t_end=None, stream=None):
        t_begin = self.p.T_hist if t_begin is None else t_begin
        t_end = self.p.T if t_end is None else t_end
        build_summaries(self.p, K, t_begin, t_end, self.csum, self.gsum, stream)

    def route(self, Q, stream=None, fused=True):
        if fused:
            route(self.p, Q, self.csum, self.gsum, self.qbar, self.cidx, self.gidx, stream)
        else:
            route_chunks(self.p, Q, self.csum, self.qbar, self.cidx, stream)
            route_groups(self.p, self.qbar, self.gsum, self.cidx, self.gidx, stream)

    def forward(self, Q, K, V, gidx=None, stream=None):
        attn_fwd(self.p, Q, K, V, self.gidx if gidx is None else gidx, self.O, self.lse, stream)

    def route_forward(self, Q, K, V, stream=None):
        """Routing and forward in one launch (hga_route_attn_fwd)."""
        route_attn_fwd(self.p, Q, K, V, self.csum, self.gsum, self.qbar, self.cidx, self.gidx, self.O, self.lse,
                       stream)

    def backward(self, Q, K, V, dO, gidx=None, stream=None):
        attn_bwd(self.p, Q, K, V, self.O, self.lse, dO, self.gidx if gidx is None else gidx,
                 self.dQ, self.dK, self.dV, self.ws, stream)

    def step(self, Q, K, V, dO=None, stream=None):
        self.summaries(K, stream=stream)
        self.route(Q, stream)
        self.forward(Q, K, V, stream=stream)
        if dO is not None:
            self.backward(Q, K, V, dO, stream=stream)
