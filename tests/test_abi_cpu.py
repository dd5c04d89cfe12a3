"""CPU checks of the C ABI: the library loads, exports every function that
include/hga.h declares, and rejects bad arguments on the host before any
launch (these calls never reach the GPU)."""
import ctypes
import os
import re

import pytest

import hierarchical_routed_sparse_b200 as hga
from hierarchical_routed_sparse_b200 import build as hbuild
from hierarchical_routed_sparse_b200.binding import _Params

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "hga.h")


@pytest.fixture(scope="module")
def lib():
    hbuild.build()
    return hga.load()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hga_\w+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert "hga_attn_fwd" in names and "hga_attn_bwd" in names
    for n in names:
        assert hasattr(lib, n), n
    assert set(hga.EXPORTS) == set(names)
    assert "sm_100a" in hga.version()


def _p(**kw):
    base = dict(B=1, Hq=32, Hkv=8, d=128, T_hist=14336, T_seg=2048, k_c=8, k_g=32)
    base.update(kw)
    return hga.Params(**base)


def test_route_widths_and_workspace(lib):
    assert hga.route_widths(_p()) == (8, 32)
    assert hga.route_widths(_p(k_c=hga.HGA_ALL, k_g=hga.HGA_ALL)) == (256, 2048)
    assert hga.route_widths(_p(k_c=4, k_g=hga.HGA_ALL)) == (4, 32)
    # Row sums (B*Hq*T_seg floats), then one int per backward item
    # (B*Hkv*nQB*ceil(G/2) = 8 * 32 * 2).
    assert hga.workspace_size(_p()) == 4 * (32 * 2048 + 8 * 32 * 2)
    assert hga.workspace_size(_p(d=96)) == 0
    # G = 3: two q-head pairs per (kv-head, block), the second with one head.
    p3 = _p(B=2, Hq=6, Hkv=2, T_hist=1024, T_seg=640)
    assert hga.workspace_size(p3) == 4 * (2 * 6 * 640 + 2 * 2 * 10 * 2)


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), hga.HGA_ERR_UNSUPPORTED),
    (dict(T_hist=100), hga.HGA_ERR_INVALID_ARG),
    (dict(T_seg=2000), hga.HGA_ERR_INVALID_ARG),
    (dict(Hq=30), hga.HGA_ERR_INVALID_ARG),
    (dict(k_c=0), hga.HGA_ERR_INVALID_ARG),
    (dict(k_g=-5), hga.HGA_ERR_INVALID_ARG),
    (dict(dtype=7), hga.HGA_ERR_INVALID_ARG),
    (dict(chunk=32), hga.HGA_ERR_UNSUPPORTED),
    (dict(B=0), hga.HGA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), hga.HGA_ERR_INVALID_ARG),
])
def test_invalid_params_rejected(lib, kw, code):
    p = _p(**kw).c()
    wc, wg = ctypes.c_int(), ctypes.c_int()
    assert lib.hga_route_widths(ctypes.byref(p), ctypes.byref(wc), ctypes.byref(wg)) == code
    assert lib.hga_last_error().decode()
    # The same validation guards every launching call: nothing is launched.
    P = ctypes.c_void_p(16)
    assert lib.hga_attn_fwd(ctypes.byref(p), P, P, P, P, P, P, None) == code


def test_null_and_misaligned_pointers_rejected(lib):
    p = _p().c()
    good = ctypes.c_void_p(1 << 20)
    assert lib.hga_attn_fwd(ctypes.byref(p), None, good, good, good, good, good, None) == \
        hga.HGA_ERR_INVALID_ARG
    assert "Q is NULL" in lib.hga_last_error().decode()
    bad = ctypes.c_void_p((1 << 20) + 4)
    assert lib.hga_route_chunks(ctypes.byref(p), good, bad, good, good, None) == hga.HGA_ERR_INVALID_ARG
    assert "csum is not 16-byte aligned" in lib.hga_last_error().decode()
    # Summary range must be 64-aligned and inside the context.
    assert lib.hga_build_summaries(ctypes.byref(p), good, 64, 100, good, good, None) == \
        hga.HGA_ERR_INVALID_ARG
    assert lib.hga_build_summaries(ctypes.byref(p), good, 0, 1 << 20, good, good, None) == \
        hga.HGA_ERR_INVALID_ARG
    # Workspace smaller than hga_workspace_size.
    P = ctypes.c_void_p(1 << 20)
    assert lib.hga_attn_bwd(ctypes.byref(p), P, P, P, P, P, P, P, P, P, P, P, 16, None) == \
        hga.HGA_ERR_INVALID_ARG
    assert "workspace" in lib.hga_last_error().decode()
    # The row sums alone (B*Hq*T_seg floats) are not enough: the workspace
    # also holds the backward's item schedule.
    rows_only = 4 * 32 * 2048
    assert lib.hga_attn_bwd(ctypes.byref(p), P, P, P, P, P, P, P, P, P, P, P, rows_only, None) == \
        hga.HGA_ERR_INVALID_ARG
    assert str(hga.workspace_size(_p())) in lib.hga_last_error().decode()
    # The fused routing + forward checks every pointer before any launch.
    args = [good] * 10
    for k, name in enumerate(("Q", "K", "V", "csum", "gsum", "qbar", "cidx", "gidx", "O", "lse")):
        a = list(args)
        a[k] = None
        assert lib.hga_route_attn_fwd(ctypes.byref(p), *a, None) == hga.HGA_ERR_INVALID_ARG, name
        assert f"{name} is NULL" in lib.hga_last_error().decode()


def test_empty_segment_is_a_no_op(lib):
    # T_seg = 0: valid, nothing to do, no pointer is touched.
    p = _p(T_seg=0).c()
    assert lib.hga_route_chunks(ctypes.byref(p), None, None, None, None, None) == hga.HGA_OK
    assert lib.hga_attn_fwd(ctypes.byref(p), None, None, None, None, None, None, None) == hga.HGA_OK
    assert lib.hga_build_summaries(ctypes.byref(p), None, 64, 64, None, None, None) == hga.HGA_OK


def test_params_struct_layout_matches_header(lib, tmp_path):
    # Compare the ctypes mirror with the C compiler's layout of hga_params.
    import subprocess
    fields = [f for f, _ in _Params._fields_]
    prog = "#include <stdio.h>\n#include <stddef.h>\n#include \"hga.h\"\nint main(void){\n"
    prog += 'printf("%zu\\n", sizeof(hga_params));\n'
    prog += "".join(f'printf("%zu\\n", offsetof(hga_params, {f}));\n' for f in fields)
    prog += "return 0;}\n"
    src = tmp_path / "layout.c"
    src.write_text(prog)
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)], check=True)
    out = [int(x) for x in subprocess.run([str(exe)], capture_output=True, text=True,
                                          check=True).stdout.split()]
    assert out[0] == ctypes.sizeof(_Params)
    assert out[1:] == [getattr(_Params, f).offset for f in fields]


def test_stage_params_round_history_to_whole_chunks(lib):
    # T_stage = round_up_64(nQB * wg * 8); every other field unchanged.
    p = _p()
    ps = hga.stage_params(p)
    assert ps.T_hist == 32 * 32 * 8 and (ps.T_seg, ps.k_c, ps.k_g, ps.d) == (p.T_seg, p.k_c, p.k_g, p.d)
    ps = hga.stage_params(_p(T_seg=128, k_g=5))                  # 2 blocks x 5 groups x 8 = 80 -> 128
    assert ps.T_hist == 128
    ps = hga.stage_params(_p(T_hist=0, T_seg=64, k_g=3))          # 24 -> 64
    assert ps.T_hist == 64
    wg = hga.route_widths(_p(k_c=4, k_g=hga.HGA_ALL))[1]          # all groups of the chosen chunks
    assert hga.stage_params(_p(k_c=4, k_g=hga.HGA_ALL)).T_hist == -(-32 * wg * 8 // 64) * 64
    # The staged problem keeps the index-row widths (HGA_ALL would follow T).
    for kw in (dict(), dict(k_c=hga.HGA_ALL, k_g=hga.HGA_ALL), dict(k_c=4, k_g=hga.HGA_ALL),
               dict(T_hist=192, T_seg=256, k_c=hga.HGA_ALL, k_g=hga.HGA_ALL)):
        assert hga.route_widths(hga.stage_params(_p(**kw))) == hga.route_widths(_p(**kw)), kw
    assert lib.hga_stage_params(ctypes.byref(_p(T_hist=100).c()), ctypes.byref(_Params())) == \
        hga.HGA_ERR_INVALID_ARG
    assert lib.hga_stage_params(ctypes.byref(_p().c()), None) == hga.HGA_ERR_INVALID_ARG


def test_stage_routed_rejects_bad_pointers_on_the_host(lib):
    p = _p()
    P = ctypes.c_void_p
    ok, mis = P(0x10000), P(0x10008)
    args = [ok] * 8
    # NULL segment rows and a misaligned staging buffer are refused before
    # any CUDA call (the history pointers are checked first only when set).
    for i, bad in ((2, None), (6, mis)):
        a = list(args)
        a[i] = bad
        assert lib.hga_stage_routed(ctypes.byref(p.c()), *a, None) == hga.HGA_ERR_INVALID_ARG
    assert lib.hga_stage_routed(ctypes.byref(_p(T_seg=0).c()), *([None] * 8), None) == hga.HGA_OK


def test_decode_rejects_bad_arguments_on_the_host(lib):
    p = _p().c()
    P = ctypes.c_void_p
    ok = P(1 << 20)
    T = p.T_hist + p.T_seg
    for pos in (-1, T, T + 5):
        assert lib.hga_decode(ctypes.byref(p), pos, *([ok] * 10), None) == hga.HGA_ERR_INVALID_ARG
        assert "pos" in lib.hga_last_error().decode()
    a = [ok] * 10
    a[0] = None
    assert lib.hga_decode(ctypes.byref(p), 3, *a, None) == hga.HGA_ERR_INVALID_ARG
    assert "q is NULL" in lib.hga_last_error().decode()
    a[0], a[7] = ok, P((1 << 20) + 8)
    assert lib.hga_decode(ctypes.byref(p), 3, *a, None) == hga.HGA_ERR_INVALID_ARG
    assert "cidx is not 16-byte aligned" in lib.hga_last_error().decode()
    # More than 8 q-heads per kv-head: refused before any launch.
    p9 = hga.Params(B=1, Hq=9, Hkv=1, d=128, T_hist=64, T_seg=64, k_c=2, k_g=4, dtype=hga.HGA_BF16).c()
    assert lib.hga_decode(ctypes.byref(p9), 3, *([ok] * 10), None) == hga.HGA_ERR_UNSUPPORTED


def test_causal_calls_reject_bad_arguments_on_the_host(lib):
    ok = ctypes.c_void_p(1 << 20)
    p9 = hga.Params(B=1, Hq=9, Hkv=1, d=128, T_hist=64, T_seg=64, k_c=2, k_g=4, dtype=hga.HGA_BF16).c()
    assert lib.hga_route_causal(ctypes.byref(p9), *([ok] * 5), None) == hga.HGA_ERR_UNSUPPORTED
    assert lib.hga_attn_fwd_causal(ctypes.byref(p9), *([ok] * 7), None) == hga.HGA_ERR_UNSUPPORTED
    assert lib.hga_attn_bwd_causal(ctypes.byref(p9), *([ok] * 11), None) == hga.HGA_ERR_UNSUPPORTED
    assert lib.hga_causal_schedule(ctypes.byref(p9), ok, ok, None) == hga.HGA_ERR_UNSUPPORTED
    assert lib.hga_causal_sched_size(ctypes.byref(p9)) == 0
    p = _p().c()
    a = [ok] * 11
    a[6] = None
    assert lib.hga_attn_bwd_causal(ctypes.byref(p), *a, None) == hga.HGA_ERR_INVALID_ARG
    assert "gidx is NULL" in lib.hga_last_error().decode()
    a = [ok] * 11
    a[7] = ctypes.c_void_p((1 << 20) + 4)            # the schedule is optional, but aligned when given
    assert lib.hga_attn_bwd_causal(ctypes.byref(p), *a, None) == hga.HGA_ERR_INVALID_ARG
    assert "sched is not 16-byte aligned" in lib.hga_last_error().decode()
    assert lib.hga_causal_schedule(ctypes.byref(p), ok, None, None) == hga.HGA_ERR_INVALID_ARG
    assert "sched is NULL" in lib.hga_last_error().decode()
    assert lib.hga_route_causal(ctypes.byref(p), ok, ok, ctypes.c_void_p((1 << 20) + 4), ok, ok, None) == \
        hga.HGA_ERR_INVALID_ARG
    assert "gsum is not 16-byte aligned" in lib.hga_last_error().decode()
    # An empty segment is a no-op.
    p0 = _p(T_seg=0).c()
    assert lib.hga_attn_fwd_causal(ctypes.byref(p0), *([None] * 7), None) == hga.HGA_OK
    assert lib.hga_causal_schedule(ctypes.byref(p0), None, None, None) == hga.HGA_OK


def test_causal_schedule_refuses_contexts_past_its_bitmap(lib):
    # The cost kernel keeps a bitmap of the context's groups in shared memory:
    # a context of 16M tokens (2M groups) is refused on the host.
    ok = ctypes.c_void_p(1 << 20)
    p = _p(T_hist=16 * 1024 * 1024, T_seg=2048).c()
    assert lib.hga_causal_schedule(ctypes.byref(p), ok, ok, None) == hga.HGA_ERR_UNSUPPORTED
    assert "bitmap" in lib.hga_last_error().decode()


def test_causal_schedule_size():
    # int32 order and costs of every window item: B * Hkv * ceil(T_seg / 32) * ceil(G / 4).
    for kw, items in [(dict(B=2, Hq=8, Hkv=2, T_seg=256), 2 * 2 * 8 * 1),
                      (dict(B=1, Hq=16, Hkv=2, T_seg=128), 1 * 2 * 4 * 2),
                      (dict(B=1, Hq=2, Hkv=2, T_seg=64), 1 * 2 * 2 * 1)]:
        assert hga.causal_sched_size(_p(**kw)) == 8 * items

@pytest.mark.parametrize("compiler,suffix", [("gcc", ".c"), ("g++", ".cpp")])
def test_plain_c_and_cpp_callers_link_and_call(lib, tmp_path, compiler, suffix):
    # A caller written against include/hga.h alone, linked to libhga.so:
    # host-only calls (version, workspace size, validation) need no GPU.
    import subprocess
    libdir = os.path.dirname(hga.LIB_PATH)
    prog = r"""
#include <stdio.h>
#include <string.h>
#include "hga.h"
int main(void) {
    hga_params p;
    memset(&p, 0, sizeof p);
    p.B = 1; p.Hq = 32; p.Hkv = 8; p.d = 128; p.T_hist = 14336; p.T_seg = 2048;
    p.chunk = 64; p.group = 8; p.qblock = 64; p.k_c = 8; p.k_g = 32; p.dtype = HGA_BF16;
    int wc = 0, wg = 0;
    if (hga_route_widths(&p, &wc, &wg) != HGA_OK || wc != 8 || wg != 32) return 1;
    if (hga_workspace_size(&p) != 4u * (32u * 2048u + 8u * 32u * 2u)) return 2;
    if (hga_attn_fwd(&p, NULL, NULL, NULL, NULL, NULL, NULL, NULL) != HGA_ERR_INVALID_ARG) return 3;
    if (strstr(hga_last_error(), "NULL") == NULL) return 4;
    p.d = 96;
    if (hga_workspace_size(&p) != 0) return 5;
    puts(hga_version());
    return 0;
}
"""
    src = tmp_path / ("caller" + suffix)
    src.write_text(prog)
    exe = tmp_path / "caller"
    subprocess.run([compiler, "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(src), "-L", libdir,
                    "-lhga", "-Wl,-rpath," + libdir, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stdout, r.stderr)
    assert "sm_100a" in r.stdout


def test_kv_capacity_is_validated_on_the_host(lib):
    import ctypes
    from hierarchical_routed_sparse_b200.binding import Params
    p = Params(B=1, Hq=4, Hkv=2, d=128, T_hist=128, T_seg=128, k_c=2, k_g=8)
    wc, wg = ctypes.c_int(), ctypes.c_int()
    for bad in (192, 256 + 32, -64):          # below T = 256, not a multiple of 64, negative
        p.kv_capacity = bad
        assert lib.hga_route_widths(ctypes.byref(p.c()), ctypes.byref(wc), ctypes.byref(wg)) == 1
        assert b"kv_capacity" in lib.hga_last_error()
    for good in (0, 256, 1024):
        p.kv_capacity = good
        assert lib.hga_route_widths(ctypes.byref(p.c()), ctypes.byref(wc), ctypes.byref(wg)) == 0
