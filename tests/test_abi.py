"""The C-ABI library: it loads, exports every entry point include/*.h declares,
and rejects bad arguments with the documented status codes before launching
anything (these calls return before any CUDA call, so they run without a GPU).
"""
import ctypes
import glob
import os
import re

import pytest

import mixture_experts_ffn_planner_b200 as moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

OK, INVALID, UNSUPPORTED, ALIGNMENT, WORKSPACE = 0, -1, -2, -3, -4


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names |= set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(\w+)\s*\(", src))
    return names


@pytest.fixture(scope="module")
def lib():
    return moe.load()


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert {"moe_align", "fused_moe_bf16", "fused_moe_mxfp8", "pack_scales_blocked"} <= names
    for n in sorted(names):
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_size_queries(lib):
    assert moe.moe_align_capacity(64, 2, 8, 64) == 128 + 8 * 63
    assert moe.moe_align_capacity(-1, 2, 8, 64) == -1
    assert moe.pack_scales_blocked_bytes(2, 129, 5) == 2 * 2 * 2 * 512
    assert moe.pack_scales_blocked_bytes(3, 128, 4) == 3 * 512
    a = moe.moe_workspace_bytes(moe.DTYPE_BF16, 64, 1024, 1024, 8, 2, 64)
    b = moe.moe_workspace_bytes(moe.DTYPE_BF16, 128, 1024, 1024, 8, 2, 64)
    assert 0 < a < b and a % 256 == 0
    assert lib.moe_workspace_bytes(7, 64, 1024, 1024, 8, 2, 64) == -1
    assert lib.moe_workspace_bytes(moe.DTYPE_BF16, 64, 1024, 1024, 8, 2, 100) == -1


def _align(lib, T=4, k=2, E=4, bm=64, cap=None, ptrs=(8, 8, 8, 8)):
    cap = lib.moe_align_capacity(T, k, E, bm) if cap is None else cap
    return lib.moe_align(ptrs[0], T, k, E, bm, ptrs[1], ptrs[2], ptrs[3], cap, None)


def test_moe_align_rejects(lib):
    assert _align(lib, bm=100) == UNSUPPORTED
    assert b"block_m" in lib.moe_last_error() and b"100" in lib.moe_last_error()
    assert _align(lib, E=0) == UNSUPPORTED
    assert _align(lib, E=1025) == UNSUPPORTED
    assert _align(lib, k=0) == INVALID
    assert _align(lib, T=-1) == INVALID
    assert _align(lib, cap=10) == INVALID
    assert _align(lib, ptrs=(8, 0, 8, 8)) == INVALID
    assert _align(lib, ptrs=(0, 8, 8, 8)) == INVALID
    assert _align(lib, T=1 << 30, k=4) == UNSUPPORTED
    assert b"2^31" in lib.moe_last_error()


def _route(lib, T=4, E=8, k=2, bm=64, cap=None, ptrs=(8, 8, 8, 8, 8, 8, 8), bias=None, S=0):
    cap = lib.moe_align_capacity(T, k + S, E + S, bm) if cap is None else cap
    return lib.moe_route_align(ptrs[0], bias, T, E, k, S, bm, ptrs[1], ptrs[2], ptrs[3], ptrs[4], ptrs[5], cap, None)


def test_moe_route_align_rejects(lib):
    assert _route(lib, k=0) == UNSUPPORTED
    assert _route(lib, k=9) == UNSUPPORTED          # more than 8 kept experts
    assert _route(lib, E=4, k=5) == UNSUPPORTED     # top_k > E
    assert _route(lib, E=1025) == UNSUPPORTED
    assert _route(lib, bm=100) == UNSUPPORTED
    assert _route(lib, T=-1) == INVALID
    assert _route(lib, cap=10) == INVALID
    assert _route(lib, ptrs=(0, 8, 8, 8, 8, 8, 8)) == INVALID   # logits
    assert _route(lib, ptrs=(8, 0, 8, 8, 8, 8, 8)) == INVALID   # topk_ids
    assert _route(lib, ptrs=(8, 8, 0, 8, 8, 8, 8)) == INVALID   # topk_weights
    assert _route(lib, ptrs=(8, 8, 8, 0, 8, 8, 8)) == INVALID   # sorted_token_ids
    assert _route(lib, S=-1) == UNSUPPORTED
    assert _route(lib, k=8, E=64, S=25) == UNSUPPORTED       # more than 32 routes per token
    assert _route(lib, E=1020, S=5) == UNSUPPORTED           # more than 1024 experts with the shared ones
    assert _route(lib, S=2, cap=lib.moe_align_capacity(4, 2, 8, 64)) == INVALID  # capacity without the shared
    assert b"moe_route_align" in lib.moe_last_error()


def test_pack_rejects(lib):
    assert lib.pack_scales_blocked(8, 8, -1, 4, 4, None) == INVALID
    assert lib.pack_scales_blocked(0, 8, 1, 4, 4, None) == INVALID
    assert lib.pack_scales_blocked(8, 9, 1, 4, 4, None) == ALIGNMENT
    assert lib.pack_scales_blocked(0, 0, 0, 4, 4, None) == OK  # nothing to do


def _bf16(lib, T=64, K=1024, N=1024, E=8, k=2, bm=64, cap=None, ws=1 << 30, p=256, wsp=256):
    cap = lib.moe_align_capacity(T, k, E, bm) if cap is None else cap
    return lib.fused_moe_bf16(p, p, p, p, p, p, p, p, T, K, N, E, k, bm, cap, wsp, ws, None, None)


def _mx(lib, T=64, K=1024, N=1024, E=8, k=2, bm=128, p=256, ws=1 << 30):
    cap = lib.moe_align_capacity(T, k, E, bm)
    return lib.fused_moe_mxfp8(p, p, p, p, p, p, p, p, p, p, p, T, K, N, E, k, bm, cap, p, ws, None, None)


def _mx4(lib, T=64, K=1024, N=1024, E=8, k=2, bm=128, p=256, w=256, ws=1 << 30):
    cap = lib.moe_align_capacity(T, k, E, bm)
    return lib.fused_moe_mxfp4(p, p, w, p, w, p, p, p, p, p, p, T, K, N, E, k, bm, cap, p, ws, None, None)


def test_mxfp4_rejects(lib):
    assert _mx4(lib, K=1152) == UNSUPPORTED
    assert _mx4(lib, N=640) == UNSUPPORTED
    assert _mx4(lib, p=0) == INVALID
    assert _mx4(lib, w=256 + 16) == ALIGNMENT      # packed e2m1 weights need 32-byte alignment
    assert _mx4(lib, ws=4096) == WORKSPACE
    assert b"fused_moe_mxfp4" in lib.moe_last_error()
    assert lib.moe_workspace_bytes(moe.DTYPE_MXFP4, 64, 1024, 1024, 8, 2, 128) == \
        lib.moe_workspace_bytes(moe.DTYPE_MXFP8, 64, 1024, 1024, 8, 2, 128)


def test_fused_rejects(lib):
    assert _bf16(lib, K=1000) == UNSUPPORTED
    assert _bf16(lib, N=1000) == UNSUPPORTED
    assert _bf16(lib, bm=48) == UNSUPPORTED
    assert _bf16(lib, E=0) == INVALID
    assert _bf16(lib, cap=10) == INVALID
    assert _bf16(lib, p=0) == INVALID
    assert _bf16(lib, p=258) == ALIGNMENT
    assert _bf16(lib, wsp=512 + 16) == ALIGNMENT
    assert _bf16(lib, ws=1024) == WORKSPACE
    assert _bf16(lib, T=0) == OK  # empty batch: nothing to launch
    assert _mx(lib, K=1152) == UNSUPPORTED
    assert _mx(lib, N=640) == UNSUPPORTED
    assert _mx(lib, p=0) == INVALID
    assert _mx(lib, ws=4096) == WORKSPACE
    msg = lib.moe_last_error()
    assert isinstance(msg, bytes) and b"workspace" in msg


def _noalloc(lib, T=64, K=1024, N=1024, E=8, k=2, bm=64, cap=None, p=256):
    cap = lib.moe_align_capacity(T, k, E, bm) if cap is None else cap
    return lib.fused_moe_bf16_noalloc(p, p, p, p, p, p, p, p, T, K, N, E, k, bm, cap, None, None)


def test_noalloc_rejects_like_fused_bf16(lib):
    """Bad sizes give the no-allocation call the same status as fused_moe_bf16."""
    for kw, code in ((dict(bm=48), UNSUPPORTED), (dict(T=-1), INVALID), (dict(E=0), INVALID),
                     (dict(k=0), INVALID), (dict(K=1000), UNSUPPORTED), (dict(N=1000), UNSUPPORTED),
                     (dict(cap=10), INVALID), (dict(p=0), INVALID), (dict(p=258), ALIGNMENT)):
        assert _noalloc(lib, **kw) == code, kw
        assert _bf16(lib, **kw) == code, kw
    assert _noalloc(lib, T=0) == OK


def test_tuning_struct_layout_matches_the_header(tmp_path):
    """The binding's ctypes moe_tuning has the C struct's size and field offsets (compiled from
    include/moe_ffn.h with the host C compiler)."""
    import shutil
    import subprocess

    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no host C compiler")
    fields = [f[0] for f in moe.Tuning._fields_]
    prog = tmp_path / "layout.c"
    prog.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "moe_ffn.h"\nint main(void) {\n'
                    '  printf("size %zu\\n", sizeof(moe_tuning));\n'
                    + "".join(f'  printf("{f} %zu\\n", offsetof(moe_tuning, {f}));\n' for f in fields)
                    + "  return 0;\n}\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-std=c99", "-I", os.path.join(ROOT, "include"), str(prog), "-o", str(exe)], check=True)
    got = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True,
                                                        check=True).stdout.splitlines())
    assert int(got["size"]) == ctypes.sizeof(moe.Tuning)
    for f in fields:
        assert int(got[f]) == getattr(moe.Tuning, f).offset, f
