"""Seeded synthetic inputs for the HGA hot path.

This module only draws random numbers: it holds none of the method's
arithmetic (no summaries, scores, selection or attention), so both the CUDA
path and the CPU oracle may use it.  Every tensor comes from numpy's
counter-based Philox generator, keyed by (seed, tensor id, batch, kv-head),
so any (batch, kv-head) unit can be regenerated on its own and both sides
see identical bytes.  bf16 workloads are rounded to bf16 (round to nearest
even) here and handed out as float32 arrays holding bf16-exact values.

The pages measure end-to-end QLoRA fine-tuning of Qwen3-8B on PG19; neither
the weights nor the dataset exist here, so these synthetic tensors of the
same attention-layer shape (32 q-heads, 8 kv-heads, d=128) stand in for
them.  Recipes:

* ``iid``: Q, K, V (and dO) i.i.d. N(0, 1).
* ``clustered``: per (batch, kv-head) 256 centroids ~ N(0, 1)^d; each
  64-token chunk of keys picks one centroid uniformly and every key is that
  centroid plus N(0, 0.3^2) noise; each query block picks a random subset
  of 8 centroids and every query row (of each q-head of the kv-head) is a
  uniformly chosen member of the subset plus N(0, 0.3^2) noise.  V and dO
  are i.i.d. N(0, 1).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace

import numpy as np

# Tensor ids of the Philox key.
_Q, _K, _V, _DO, _CENT, _ASSIGN, _SUBSET, _PICK = range(8)

N_CENTROIDS = 256
CLUSTER_RUN = 64      # keys share one centroid over runs of this many tokens
QUERY_RUN = 64        # queries share one centroid subset over this many rows
SUBSET = 8
NOISE_STD = 0.3


def _rng(seed: int, tid: int, b: int, g: int) -> np.random.Generator:
    key = np.array([(seed << 8) | tid, (b << 32) | g], dtype=np.uint64)
    return np.random.Generator(np.random.Philox(key=key))


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even), as float32."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)      # finite inputs: the sum below cannot wrap
    u = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return u.view(np.float32)


@dataclass(frozen=True)
class Workload:
    """One synthetic problem: attention-layer shape, routing budget, recipe."""
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    T_hist: int
    T_seg: int
    k_c: int
    k_g: int
    dtype: str = "bf16"          # "bf16" or "fp32" (dtype of Q, K, V, dO)
    keys: str = "iid"            # "iid" or "clustered"
    backward: bool = False
    seed: int = 0
    extra: dict = field(default_factory=dict, compare=False)

    @property
    def T(self) -> int:
        return self.T_hist + self.T_seg

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    # -- generation --------------------------------------------------------
    def _finish(self, x: np.ndarray) -> np.ndarray:
        return round_bf16(x) if self.dtype == "bf16" else x.astype(np.float32)

    def unit(self, b: int, g: int) -> dict:
        """Inputs of one (batch, kv-head) unit.

        Returns float32 arrays Q [G,T_seg,d], K [T,d], V [T,d], dO [G,T_seg,d].
        """
        G, d, T, Ts = self.G, self.d, self.T, self.T_seg
        s = self.seed
        if self.keys == "iid":
            Q = _rng(s, _Q, b, g).standard_normal((G, Ts, d), dtype=np.float32)
            K = _rng(s, _K, b, g).standard_normal((T, d), dtype=np.float32)
        elif self.keys == "clustered":
            cent = _rng(s, _CENT, b, g).standard_normal((N_CENTROIDS, d), dtype=np.float32)
            n_runs = T // CLUSTER_RUN
            assign = _rng(s, _ASSIGN, b, g).integers(0, N_CENTROIDS, size=n_runs)
            K = _rng(s, _K, b, g).standard_normal((T, d), dtype=np.float32)
            K *= np.float32(NOISE_STD)
            K += np.repeat(cent[assign], CLUSTER_RUN, axis=0)
            n_qruns = Ts // QUERY_RUN
            rs = _rng(s, _SUBSET, b, g)
            subsets = np.stack([rs.choice(N_CENTROIDS, SUBSET, replace=False)
                                for _ in range(n_qruns)])                 # [n_qruns, 8]
            pick = _rng(s, _PICK, b, g).integers(0, SUBSET, size=(G, Ts))
            which = subsets[np.arange(Ts)[None, :] // QUERY_RUN, pick]   # [G, Ts]
            Q = _rng(s, _Q, b, g).standard_normal((G, Ts, d), dtype=np.float32)
            Q *= np.float32(NOISE_STD)
            Q += cent[which]
        else:
            raise ValueError(f"unknown key recipe {self.keys!r}")
        V = _rng(s, _V, b, g).standard_normal((T, d), dtype=np.float32)
        out = dict(Q=self._finish(Q), K=self._finish(K), V=self._finish(V))
        if self.backward:
            dO = _rng(s, _DO, b, g).standard_normal((G, Ts, d), dtype=np.float32)
            out["dO"] = self._finish(dO)
        return out

    def full(self) -> dict:
        """All inputs: Q, dO [B,Hq,T_seg,d]; K, V [B,Hkv,T,d] (float32 arrays)."""
        G = self.G
        Q = np.empty((self.B, self.Hq, self.T_seg, self.d), dtype=np.float32)
        K = np.empty((self.B, self.Hkv, self.T, self.d), dtype=np.float32)
        V = np.empty_like(K)
        dO = np.empty_like(Q) if self.backward else None
        def fill(bg):
            b, g = divmod(bg, self.Hkv)
            u = self.unit(b, g)
            Q[b, g * G:(g + 1) * G] = u["Q"]
            K[b, g] = u["K"]
            V[b, g] = u["V"]
            if dO is not None:
                dO[b, g * G:(g + 1) * G] = u["dO"]

        # Units are independent streams: fill them concurrently.
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, range(self.B * self.Hkv)))
        out = dict(Q=Q, K=K, V=V)
        if dO is not None:
            out["dO"] = dO
        return out


# The workloads of the benchmark and the parity suite.  Names state shapes.
TINY_FP32 = Workload("tiny_fp32_d64_T1024", B=1, Hq=1, Hkv=1, d=64, T_hist=0, T_seg=1024,
                     k_c=4, k_g=16, dtype="fp32", keys="iid")
QWEN3_T2K_FWD = Workload("qwen3_8b_layer_T2048_fwd", B=1, Hq=32, Hkv=8, d=128, T_hist=0,
                         T_seg=2048, k_c=8, k_g=32, dtype="bf16", keys="iid")
QWEN3_CTX16K_FWD = Workload("qwen3_8b_layer_ctx16k_fwd", B=1, Hq=32, Hkv=8, d=128,
                            T_hist=14336, T_seg=2048, k_c=8, k_g=32, dtype="bf16",
                            keys="clustered")
QWEN3_CTX16K_TRAIN = QWEN3_CTX16K_FWD.with_(name="qwen3_8b_layer_ctx16k_segment_train",
                                            backward=True)


def sweep_point(T: int, k_c: int, k_g: int) -> Workload:
    """Scale-sweep point: B=4, 2048-token segment over T total tokens."""
    return Workload(f"sweep_B4_ctx{T}_kc{k_c}_kg{k_g}", B=4, Hq=32, Hkv=8, d=128,
                    T_hist=T - 2048, T_seg=2048, k_c=k_c, k_g=k_g, dtype="bf16",
                    keys="clustered", backward=True)


SWEEP = [sweep_point(T, kc, kg) for T in (32768, 65536, 131072)
         for kc in (8, 16) for kg in (32, 64)]

BY_NAME = {w.name: w for w in [TINY_FP32, QWEN3_T2K_FWD, QWEN3_CTX16K_FWD,
                               QWEN3_CTX16K_TRAIN, *SWEEP]}
