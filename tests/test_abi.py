"""The C-ABI library loads without a GPU, exports every symbol include/sge.h
declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re
import subprocess

import pytest

import activation_sparse_gated_epilogue_b200 as sge
from activation_sparse_gated_epilogue_b200 import build as sge_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sge.h")


SELFTEST_HEADER = os.path.join(ROOT, "include", "sge_selftest.h")


def declared_functions(header=HEADER):
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M)
    return sorted(set(n for n in names if n not in ("defined",)))


@pytest.fixture(scope="module")
def lib():
    sge_build.build()
    return sge.library()


def test_header_declares_entry_points():
    names = declared_functions()
    for want in ("twell_gate_pack", "twell_fused_up_down", "dense_ffn_fwd", "sge_last_error"):
        assert want in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", sge.library_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    for name in declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_every_header_is_covered():
    """include/ holds the product library's header and the self-test
    library's; the tests below check both."""
    headers = sorted(os.listdir(os.path.join(ROOT, "include")))
    assert headers == ["sge.h", "sge_selftest.h"], headers


def test_selftest_library_exports_its_declared_symbols(lib):
    path = sge_build.SELFTEST_LIB
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True,
                         check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    names = declared_functions(SELFTEST_HEADER)
    assert names == ["sge_selftest_wait_timeout"]
    st = ctypes.CDLL(path)
    for name in names:
        assert name in exported, name
        assert getattr(st, name) is not None


def test_debug_library_exports_the_same_symbols(lib):
    """libsge_debug.so (the index-checking build) exports every symbol of
    the header, like the release library; the release build's
    sge_debug_flags answers -1 without touching the device."""
    path = sge_build.build_debug()
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True,
                         check=True).stdout
    exported = set(line.split()[-1] for line in out.splitlines() if line.strip())
    for name in declared_functions():
        assert name in exported, name
    lib.sge_debug_flags.restype = ctypes.c_int
    lib.sge_debug_flags.argtypes = [ctypes.c_int]
    assert lib.sge_debug_flags(0) == -1


def test_selftest_rejects_bad_arguments(lib):
    st = ctypes.CDLL(sge_build.SELFTEST_LIB)
    P = ctypes.c_void_p
    st.sge_selftest_wait_timeout.argtypes = [ctypes.c_int, P, P, ctypes.c_int64, ctypes.c_int64,
                                             ctypes.c_int64, P, P, P]
    p = P(4096)
    assert st.sge_selftest_wait_timeout(0, None, p, 256, 256, 256, p, p, None) == 1
    assert st.sge_selftest_wait_timeout(1, p, p, 256, 256, 32, p, p, None) == 1    # k < 64


def test_version_and_error_string(lib):
    assert lib.sge_version() >= 100
    assert isinstance(lib.sge_last_error(), bytes)


def _gate(lib, **kw):
    a = dict(x=None, w=None, n=8, d=64, f=256, dt=sge.SGE_BF16, tile=128, cap=128,
             count=None, idx=None, val=None, diag=None, stream=None)
    a.update(kw)
    return lib.twell_gate_pack(a["x"], a["w"], a["n"], a["d"], a["f"], a["dt"], a["tile"], a["cap"],
                               a["count"], a["idx"], a["val"], a["diag"], a["stream"])


def test_bad_arguments_are_rejected_on_host(lib):
    assert _gate(lib, d=60) == 1                  # d % 8
    assert _gate(lib, tile=48) == 2               # unsupported tile
    assert _gate(lib, f=200, tile=64) == 1        # T does not divide F
    assert _gate(lib, cap=0) == 1
    assert _gate(lib, cap=129) == 1
    assert _gate(lib, n=-1) == 1
    assert _gate(lib) == 1                        # null pointers
    assert b"null" in lib.sge_last_error()
    assert _gate(lib, dt=7, x=ctypes.c_void_p(16), w=ctypes.c_void_p(16), count=ctypes.c_void_p(16),
                 idx=ctypes.c_void_p(16), val=ctypes.c_void_p(16)) == 2
    assert _gate(lib, x=ctypes.c_void_p(17), w=ctypes.c_void_p(16), count=ctypes.c_void_p(16),
                 idx=ctypes.c_void_p(16), val=ctypes.c_void_p(16)) == 1   # misaligned
    assert b"aligned" in lib.sge_last_error()


def test_empty_input_is_a_no_op(lib):
    assert _gate(lib, n=0) == 0
    assert lib.twell_fused_up_down(None, None, None, None, None, None, 64, None, 0, 64, 256,
                                   sge.SGE_BF16, 128, 128, None, 0, None, None) == 0
    assert lib.dense_ffn_fwd(None, None, None, None, None, None, 0, 64, 256, None, None) == 0


def test_fused_rejects_bad_arguments(lib):
    assert lib.twell_fused_up_down(None, None, None, None, None, None, 12, None, 8, 12, 256,
                                   sge.SGE_BF16, 128, 128, None, 0, None, None) == 1
    assert lib.twell_fused_up_down(None, None, None, None, None, None, 64, None, 8, 64, 256,
                                   sge.SGE_BF16, 128, 128, None, 0, None, None) == 1
    p = ctypes.c_void_p(16)
    # a workspace smaller than the query's answer is rejected
    assert lib.twell_fused_up_down(p, p, p, p, p, p, 64, p, 1000, 64, 256, sge.SGE_BF16, 128, 128,
                                   p, 64, None, None) == 1
    assert b"workspace" in lib.sge_last_error()
    assert lib.twell_fused_up_down_workspace_bytes(1000, 64) >= 16 + 5 * 1000
    assert lib.twell_fused_up_down_workspace_bytes(1000, 64) % 256 == 0
    # the workspace must be 256-byte aligned
    ws = lib.twell_fused_up_down_workspace_bytes(1000, 64)
    assert lib.twell_fused_up_down(p, p, p, p, p, p, 64, p, 1000, 64, 256, sge.SGE_BF16, 128, 128,
                                   ctypes.c_void_p(4096 + 16), ws, None, None) == 1
    assert b"aligned" in lib.sge_last_error()
    # the weights' row stride: at least d_model, a multiple of 8
    for ldw in (32, 60, 68):
        assert lib.twell_fused_up_down(p, p, p, p, p, p, ldw, p, 1000, 64, 256, sge.SGE_BF16, 128,
                                       128, ctypes.c_void_p(4096), ws, None, None) == 1
        assert b"ldw" in lib.sge_last_error()
    assert lib.dense_ffn_fwd(None, None, None, None, None, None, 8, 64, 100, None, None) == 1


def test_interleave_rejects_bad_arguments(lib):
    p = ctypes.c_void_p(4096)
    assert lib.sge_interleave_up_down(None, None, None, 0, 64, sge.SGE_BF16, None) == 0  # F = 0
    assert lib.sge_interleave_up_down(None, p, p, 8, 64, sge.SGE_BF16, None) == 1
    assert b"null" in lib.sge_last_error()
    assert lib.sge_interleave_up_down(p, p, p, 8, 0, sge.SGE_BF16, None) == 1
    assert lib.sge_interleave_up_down(p, p, p, 8, 64, 7, None) == 2
    # the output may not overlap an input
    assert lib.sge_interleave_up_down(ctypes.c_void_p(4096), ctypes.c_void_p(1 << 20),
                                      ctypes.c_void_p(4096 + 512), 8, 64, sge.SGE_BF16, None) == 1
    assert b"overlaps" in lib.sge_last_error()


def test_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        sge.twell_gate_pack(x, torch.zeros(128, 64, dtype=torch.bfloat16), 128, 128)


def _routed(lib, **kw):
    p = ctypes.c_void_p(4096)
    a = dict(x=p, count=p, idx=p, val=p, wu=p, wd=p, ldw=64, wd_t=p, y=p, n=1000, d=64, f=256,
             tile=128, cap=128, k=16, s_max=64, ws=p, ws_bytes=1 << 40, diag=None, stream=None)
    a.update(kw)
    return lib.twell_hybrid_up_down(a["x"], a["count"], a["idx"], a["val"], a["wu"], a["wd"],
                                    a["ldw"], a["wd_t"], a["y"], a["n"], a["d"], a["f"], a["tile"],
                                    a["cap"], a["k"], a["s_max"], a["ws"], a["ws_bytes"], a["diag"],
                                    a["stream"])


def test_routed_rejects_bad_arguments(lib):
    assert _routed(lib, n=0, x=None, ws=None) == 0          # empty input: no-op
    assert _routed(lib, k=-1) == 1
    assert b"capacity" in lib.sge_last_error()
    assert _routed(lib, s_max=-3) == 1
    assert _routed(lib, wd_t=None) == 1                      # the spill needs W_down^T
    assert b"null" in lib.sge_last_error()
    assert _routed(lib, f=260, tile=20, cap=20) == 1         # F % 8
    assert _routed(lib, d=60, ldw=64) == 1                   # d % 8
    need = lib.twell_hybrid_up_down_workspace_bytes(1000, 64, 256, 64)
    assert _routed(lib, ws_bytes=need - 1) == 1
    assert b"workspace" in lib.sge_last_error()
    assert _routed(lib, ws=ctypes.c_void_p(4096 + 128), ws_bytes=need) == 1
    assert b"aligned" in lib.sge_last_error()
    # the spill operands grow the workspace with S_max
    small = lib.twell_hybrid_up_down_workspace_bytes(1000, 64, 256, 0)
    assert need >= small + 64 * (64 + 2 * 256) * 2
    assert lib.twell_hybrid_up_down_workspace_bytes(1000, 64, 256, -1) == 0


def test_transpose_up_gate_rejects_bad_arguments(lib):
    p = ctypes.c_void_p(4096)
    assert lib.sge_transpose_up_gate(p, p, p, 100, 64, None) == 1     # F % 8
    assert lib.sge_transpose_up_gate(p, None, p, 128, 64, None) == 1
    assert b"null" in lib.sge_last_error()
    assert lib.sge_transpose_up_gate(ctypes.c_void_p(4100), p, p, 128, 64, None) == 1
    assert b"aligned" in lib.sge_last_error()
