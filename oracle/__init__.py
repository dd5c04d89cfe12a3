"""CPU oracle for HGA two-level routed sparse attention (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its binding) never touches it.  All arithmetic lives in ``hga_oracle.c``
(double precision, explicit loops); this module only marshals numpy arrays
into it through ctypes and builds it with gcc when asked.

Every function mirrors one call of the CUDA library's C-ABI and follows the
method as described in the article "BMW's 16 GB GPU just did what needs an
A100" (seventnews.com), section "What HGA does differently".
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hga_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (plain -O2, IEEE arithmetic, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-shared", "-fPIC",
               "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


class _Dims(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("d", ctypes.c_int), ("T_hist", ctypes.c_int64), ("T_seg", ctypes.c_int64),
                ("chunk", ctypes.c_int), ("group", ctypes.c_int),
                ("k_c", ctypes.c_int), ("k_g", ctypes.c_int),
                ("wc", ctypes.c_int), ("wg", ctypes.c_int), ("scale", ctypes.c_double)]


@dataclass
class Dims:
    """Problem shape.  k_c / k_g <= 0 mean "keep every eligible candidate".

    wc / wg are the row widths of the chunk / group index tables; by default
    k (or, for "all", every chunk of the context and 8 groups per chunk).
    """
    B: int
    Hq: int
    Hkv: int
    d: int
    T_hist: int
    T_seg: int
    k_c: int
    k_g: int
    chunk: int = 64
    group: int = 8
    scale: float = 0.0
    wc: int = 0
    wg: int = 0

    def __post_init__(self):
        if self.scale == 0.0:
            self.scale = 1.0 / math.sqrt(self.d)
        T = self.T_hist + self.T_seg
        if self.wc == 0:
            self.wc = self.k_c if self.k_c > 0 else T // self.chunk
        if self.wg == 0:
            self.wg = self.k_g if self.k_g > 0 else self.wc * (self.chunk // self.group)

    @property
    def T(self) -> int:
        return self.T_hist + self.T_seg

    @property
    def nQB(self) -> int:
        return self.T_seg // self.chunk

    def _c(self) -> _Dims:
        return _Dims(self.B, self.Hq, self.Hkv, self.d, self.T_hist, self.T_seg,
                     self.chunk, self.group, self.k_c, self.k_g, self.wc, self.wg,
                     float(self.scale))


_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        D = ctypes.POINTER(_Dims)
        lib.oracle_build_summaries.argtypes = [D, P, ctypes.c_int64, ctypes.c_int64, P, P]
        lib.oracle_block_query.argtypes = [D, P, P]
        lib.oracle_route_chunks.argtypes = [D, P, P, P, P]
        lib.oracle_route_groups.argtypes = [D, P, P, P, P, P]
        lib.oracle_attn_fwd.argtypes = [D, P, P, P, P, P, P]
        lib.oracle_attn_bwd.argtypes = [D, P, P, P, P, P, P, P, P]
        lib.oracle_decode.argtypes = [D, ctypes.c_int64, P, P, P, P, P, P, P, P, P, P, P]
        lib.oracle_causal_route.argtypes = [D, P, P, P, P, P, P, P]
        lib.oracle_causal_attn_fwd.argtypes = [D, P, P, P, P, P, P]
        lib.oracle_causal_attn_bwd.argtypes = [D, P, P, P, P, P, P, P, P]
        lib.oracle_num_threads.restype = ctypes.c_int
        lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
        for f in ("oracle_build_summaries", "oracle_block_query", "oracle_route_chunks",
                  "oracle_route_groups", "oracle_attn_fwd", "oracle_attn_bwd", "oracle_decode",
                  "oracle_causal_route", "oracle_causal_attn_fwd", "oracle_causal_attn_bwd",
                  "oracle_set_num_threads"):
            getattr(lib, f).restype = None
        _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def num_threads() -> int:
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> None:
    _load().oracle_set_num_threads(int(n))


def build_summaries(dims: Dims, K, t_begin: int | None = None, t_end: int | None = None,
                    csum=None, gsum=None):
    """Chunk / group mean summaries of keys [t_begin, t_end) (default: all).

    Returns (csum [B,Hkv,T/chunk,d], gsum [B,Hkv,T/group,d]); rows outside the
    range keep the values of the arrays passed in (zeros if none).
    """
    K = _f64(K)
    t_begin = 0 if t_begin is None else t_begin
    t_end = dims.T if t_end is None else t_end
    if csum is None:
        csum = np.zeros((dims.B, dims.Hkv, dims.T // dims.chunk, dims.d))
    if gsum is None:
        gsum = np.zeros((dims.B, dims.Hkv, dims.T // dims.group, dims.d))
    csum, gsum = _f64(csum).copy(), _f64(gsum).copy()
    _load().oracle_build_summaries(ctypes.byref(dims._c()), _ptr(K), t_begin, t_end,
                                   _ptr(csum), _ptr(gsum))
    return csum, gsum


def block_query(dims: Dims, Q):
    Q = _f64(Q)
    qbar = np.zeros((dims.B, dims.Hkv, dims.nQB, dims.d))
    _load().oracle_block_query(ctypes.byref(dims._c()), _ptr(Q), _ptr(qbar))
    return qbar


def route_chunks(dims: Dims, qbar, csum):
    """Returns (cidx [B,Hkv,nQB,wc] int32, gap [B,Hkv,nQB] float64)."""
    qbar, csum = _f64(qbar), _f64(csum)
    cidx = np.full((dims.B, dims.Hkv, dims.nQB, dims.wc), -7, dtype=np.int32)
    gap = np.zeros((dims.B, dims.Hkv, dims.nQB))
    _load().oracle_route_chunks(ctypes.byref(dims._c()), _ptr(qbar), _ptr(csum),
                                _ptr(cidx), _ptr(gap))
    return cidx, gap


def route_groups(dims: Dims, qbar, gsum, cidx):
    """Returns (gidx [B,Hkv,nQB,wg] int32, gap [B,Hkv,nQB] float64)."""
    qbar, gsum, cidx = _f64(qbar), _f64(gsum), _i32(cidx)
    gidx = np.full((dims.B, dims.Hkv, dims.nQB, dims.wg), -7, dtype=np.int32)
    gap = np.zeros((dims.B, dims.Hkv, dims.nQB))
    _load().oracle_route_groups(ctypes.byref(dims._c()), _ptr(qbar), _ptr(gsum),
                                _ptr(cidx), _ptr(gidx), _ptr(gap))
    return gidx, gap


def attn_fwd(dims: Dims, Q, K, V, gidx):
    """Returns (O [B,Hq,T_seg,d], lse [B,Hq,T_seg]) in float64."""
    Q, K, V, gidx = _f64(Q), _f64(K), _f64(V), _i32(gidx)
    O = np.zeros((dims.B, dims.Hq, dims.T_seg, dims.d))
    lse = np.zeros((dims.B, dims.Hq, dims.T_seg))
    _load().oracle_attn_fwd(ctypes.byref(dims._c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(gidx),
                            _ptr(O), _ptr(lse))
    return O, lse


def attn_bwd(dims: Dims, Q, K, V, dO, gidx):
    """Returns (dQ [B,Hq,T_seg,d], dK_seg, dV_seg [B,Hkv,T_seg,d]) in float64."""
    Q, K, V, dO, gidx = _f64(Q), _f64(K), _f64(V), _f64(dO), _i32(gidx)
    dQ = np.zeros((dims.B, dims.Hq, dims.T_seg, dims.d))
    dK = np.zeros((dims.B, dims.Hkv, dims.T_seg, dims.d))
    dV = np.zeros((dims.B, dims.Hkv, dims.T_seg, dims.d))
    _load().oracle_attn_bwd(ctypes.byref(dims._c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(dO),
                            _ptr(gidx), _ptr(dQ), _ptr(dK), _ptr(dV))
    return dQ, dK, dV


def decode(dims: Dims, pos: int, q, K, V, csum, gsum):
    """One generation step for the token at position pos (a query block of
    one): q [B,Hq,d]; K, V [B,Hkv,T,d] with rows 0..pos valid; csum / gsum of
    the complete chunks.  Returns dict(O [B,Hq,d], lse [B,Hq], cidx, gidx
    [B,Hkv,w], cgap, ggap [B,Hkv])."""
    q, K, V, csum, gsum = _f64(q), _f64(K), _f64(V), _f64(csum), _f64(gsum)
    B, Hq, Hkv, d = dims.B, dims.Hq, dims.Hkv, dims.d
    O = np.zeros((B, Hq, d))
    lse = np.zeros((B, Hq))
    cidx = np.full((B, Hkv, dims.wc), -7, dtype=np.int32)
    gidx = np.full((B, Hkv, dims.wg), -7, dtype=np.int32)
    cgap = np.zeros((B, Hkv))
    ggap = np.zeros((B, Hkv))
    _load().oracle_decode(ctypes.byref(dims._c()), int(pos), _ptr(q), _ptr(K), _ptr(V), _ptr(csum),
                          _ptr(gsum), _ptr(O), _ptr(lse), _ptr(cidx), _ptr(gidx), _ptr(cgap), _ptr(ggap))
    return dict(O=O, lse=lse, cidx=cidx, gidx=gidx, cgap=cgap, ggap=ggap)


def causal_route(dims: Dims, Q, csum, gsum):
    """Strictly causal routing: every query position routes on its own query
    (mean over the G q-heads), a block of one.  Returns dict(cidx [B,Hkv,
    T_seg,wc], gidx [B,Hkv,T_seg,wg], cgap, ggap [B,Hkv,T_seg])."""
    Q, csum, gsum = _f64(Q), _f64(csum), _f64(gsum)
    B, Hkv, Ts = dims.B, dims.Hkv, dims.T_seg
    cidx = np.full((B, Hkv, Ts, dims.wc), -7, dtype=np.int32)
    gidx = np.full((B, Hkv, Ts, dims.wg), -7, dtype=np.int32)
    cgap = np.zeros((B, Hkv, Ts))
    ggap = np.zeros((B, Hkv, Ts))
    _load().oracle_causal_route(ctypes.byref(dims._c()), _ptr(Q), _ptr(csum), _ptr(gsum), _ptr(cidx),
                                _ptr(gidx), _ptr(cgap), _ptr(ggap))
    return dict(cidx=cidx, gidx=gidx, cgap=cgap, ggap=ggap)


def causal_attn_fwd(dims: Dims, Q, K, V, gidx):
    """Attention of the causal variant (gidx per position).  Returns (O, lse)."""
    Q, K, V, gidx = _f64(Q), _f64(K), _f64(V), _i32(gidx)
    O = np.zeros((dims.B, dims.Hq, dims.T_seg, dims.d))
    lse = np.zeros((dims.B, dims.Hq, dims.T_seg))
    _load().oracle_causal_attn_fwd(ctypes.byref(dims._c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(gidx),
                                   _ptr(O), _ptr(lse))
    return O, lse


def causal_attn_bwd(dims: Dims, Q, K, V, dO, gidx):
    """Backward of the causal variant (routing frozen).  Returns (dQ, dK_seg, dV_seg)."""
    Q, K, V, dO, gidx = _f64(Q), _f64(K), _f64(V), _f64(dO), _i32(gidx)
    dQ = np.zeros((dims.B, dims.Hq, dims.T_seg, dims.d))
    dK = np.zeros((dims.B, dims.Hkv, dims.T_seg, dims.d))
    dV = np.zeros((dims.B, dims.Hkv, dims.T_seg, dims.d))
    _load().oracle_causal_attn_bwd(ctypes.byref(dims._c()), _ptr(Q), _ptr(K), _ptr(V), _ptr(dO),
                                   _ptr(gidx), _ptr(dQ), _ptr(dK), _ptr(dV))
    return dQ, dK, dV


def route(dims: Dims, Q, K):
    """Convenience: summaries -> block query -> chunk routing -> group routing."""
    csum, gsum = build_summaries(dims, K)
    qbar = block_query(dims, Q)
    cidx, cgap = route_chunks(dims, qbar, csum)
    gidx, ggap = route_groups(dims, qbar, gsum, cidx)
    return dict(csum=csum, gsum=gsum, qbar=qbar, cidx=cidx, cgap=cgap, gidx=gidx, ggap=ggap)
