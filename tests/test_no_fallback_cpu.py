"""The product path has no CPU fallback: host tensors are refused by the
binding, and a missing libhga.so makes every call raise (checked in a child
process whose binding points at a path that does not exist)."""
import os
import subprocess
import sys

import pytest
import torch

import hierarchical_routed_sparse_b200 as hga

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_host_tensors_are_refused():
    p = hga.Params(B=1, Hq=2, Hkv=1, d=64, T_hist=0, T_seg=64, k_c=1, k_g=8, dtype=hga.HGA_FP32)
    Q = torch.zeros(1, 2, 64, 64)
    K = V = torch.zeros(1, 1, 64, 64)
    gidx = torch.zeros(1, 1, 1, 8, dtype=torch.int32)
    O, lse = torch.zeros(1, 2, 64, 64), torch.zeros(1, 2, 64)

    class Stream:
        cuda_stream = 0

    with pytest.raises(ValueError, match="device tensors"):
        hga.attn_fwd(p, Q, K, V, gidx, O, lse, stream=Stream())


def test_missing_library_raises():
    code = (
        "import hierarchical_routed_sparse_b200.binding as B\n"
        "B.LIB_PATH = '/nonexistent/libhga.so'\n"
        "B._lib = None\n"
        "import hierarchical_routed_sparse_b200 as hga\n"
        "try:\n"
        "    hga.workspace_size(hga.Params(B=1, Hq=1, Hkv=1, d=64, T_hist=0, T_seg=64, k_c=1, k_g=8))\n"
        "except RuntimeError as e:\n"
        "    print('raised:', e)\n"
        "    raise SystemExit(0)\n"
        "raise SystemExit(1)\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "is missing" in r.stdout
