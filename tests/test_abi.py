"""The C ABI without a GPU: libpa.so loads, exports every entry point that
include/pa.h declares, and rejects bad arguments synchronously (before any
launch) with the documented status codes."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_pa_b200 as pa
from block_sparse_attention_pa_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return pa.lib()


def declared_entry_points():
    src = open(os.path.join(ROOT, "include", "pa.h")).read()
    return sorted(set(re.findall(r"PA_API\s+[\w\s\*]*?\b(pa_\w+)\s*\(", src)))


def test_header_declares_the_binding_entry_points():
    assert declared_entry_points() == sorted(pa.ENTRY_POINTS)


def test_library_exports_every_declared_symbol(L):
    for name in declared_entry_points():
        assert hasattr(L, name), name


def test_version_and_status_strings(L):
    assert L.pa_abi_version() == 3
    for code in range(8):
        assert L.pa_status_string(code).decode() not in ("", "unknown status")
    assert L.pa_status_string(99).decode() == "unknown status"


def shape(B=1, N=1024, H=8, Hkv=2, d=64, blk=128, G=1):
    return pa.Shape(B, N, H, Hkv, d, blk, G)


def test_workspace_size_formula(L):
    s = shape(N=1024, H=8, Hkv=2, d=64, G=2)
    nb = 8
    T = nb * (nb + 1) // 2
    a256 = lambda x: (x + 255) // 256 * 256
    dyn = pa.workspace_size(s, pa.make_budget(pa.DYNAMIC, 0.9))
    assert dyn == a256(8 * nb * 128 * 8) + 2 * a256(2 * 1024 * 64 * 2) + a256(2 * T * 4)
    fixed = pa.workspace_size(s, pa.make_budget(pa.FIXED_FRACTION, 0, 100))
    assert fixed == 2 * a256(2 * 1024 * 64 * 2) + a256(2 * T * 4)
    assert pa.workspace_size(shape(N=1000), pa.make_budget()) == 0
    assert pa.workspace_size(s, pa.make_budget(pa.DYNAMIC, 1.5)) == 0
    # a query-row stride r keeps only N/r rows of the q proxy; 0 reads as 1
    for r in (2, 4, 8):
        st = pa.workspace_size(s, pa.make_budget(pa.FIXED_FRACTION, 0, 100, r))
        assert st == a256(2 * (1024 // r) * 64 * 2) + a256(2 * 1024 * 64 * 2) + a256(2 * T * 4)
    assert pa.workspace_size(s, pa.make_budget(pa.FIXED_FRACTION, 0, 100, 0)) == fixed
    for r in (3, 16, -1):
        assert pa.workspace_size(s, pa.make_budget(pa.FIXED_FRACTION, 0, 100, r)) == 0


@pytest.mark.parametrize("bad,code", [
    (dict(N=1000), 2),          # N % 128
    (dict(d=96), 2),            # head_dim
    (dict(blk=64), 2),          # block
    (dict(H=8, Hkv=3), 2),      # H % Hkv
    (dict(H=8, G=3), 2),        # H % G
    (dict(N=128 * 4097), 2),    # too long
    (dict(H=0), 1),             # non-positive
    (dict(B=0), 1),
    (dict(N=0), 1),             # empty sequence
    (dict(N=-128), 1),
    (dict(Hkv=0), 1),
    (dict(G=0), 1),
])
def test_bad_shapes_rejected_before_launch(L, bad, code):
    s = shape(**bad)
    st = pa.Strides(0, 512, 64)
    r = L.pa_pool_heads(ctypes.byref(s), 16, st, 16, st, 16, 16, None)
    assert r == code
    assert L.pa_last_error() != b""


def test_null_and_misaligned_pointers_rejected(L):
    s = shape()
    st = pa.Strides(0, 512, 64)
    assert L.pa_pool_heads(ctypes.byref(s), None, st, 16, st, 16, 16, None) == 1
    assert L.pa_pool_heads(ctypes.byref(s), 8, st, 16, st, 16, 16, None) == 1      # 8-byte aligned only
    assert L.pa_pool_heads(ctypes.byref(s), 16, pa.Strides(0, 512, 60), 16, st, 16, 16, None) == 1
    assert L.pa_block_scores(ctypes.byref(s), 16, 16, None, None) == 1
    assert L.pa_block_scores(None, 16, 16, 16, None) == 1


@pytest.mark.parametrize("r", [0, 3, 16, -2])
def test_bad_score_stride_rejected(L, r):
    s = shape()
    st = pa.Strides(0, 512, 64)
    assert L.pa_pool_heads_strided(ctypes.byref(s), r, 16, st, 16, st, 16, 16, None) == 1
    assert b"score_stride" in L.pa_last_error()
    assert L.pa_block_scores_strided(ctypes.byref(s), r, 16, 16, 16, None) == 1
    if r != 0:  # 0 in pa_budget means "every row"
        m = pa.MaskBufs(16, 16, 16, 16)
        bad = pa.make_budget(pa.FIXED_FRACTION, 0, 100, r)
        assert L.pa_prefill(ctypes.byref(s), ctypes.byref(bad), 16, st, 16, st, 16, st, 16, st, ctypes.byref(m),
                            256, 1 << 30, None) == 1


def test_budget_and_workspace_errors(L):
    s = shape()
    st = pa.Strides(0, 512, 64)
    m = pa.MaskBufs(16, 16, 16, 16)
    for bad in (pa.make_budget(pa.DYNAMIC, 0.0), pa.make_budget(pa.DYNAMIC, 1.01),
                pa.make_budget(pa.FIXED_FRACTION, 0, 0), pa.make_budget(pa.FIXED_FRACTION, 0, 1001),
                pa.make_budget(7, 0.5, 0)):
        assert L.pa_build_mask(ctypes.byref(s), ctypes.byref(bad), 16, 16, st, 16, st, ctypes.byref(m), 256, 1 << 30,
                               None) == 1
    good = pa.make_budget(pa.DYNAMIC, 0.9)
    # dynamic mode needs the mass buffer and a large enough workspace
    m_nomass = pa.MaskBufs(16, 16, 16, None)
    assert L.pa_build_mask(ctypes.byref(s), ctypes.byref(good), 16, 16, st, 16, st, ctypes.byref(m_nomass), 256,
                           1 << 30, None) == 1
    assert L.pa_build_mask(ctypes.byref(s), ctypes.byref(good), 16, 16, st, 16, st, ctypes.byref(m), 256, 16,
                           None) == 3
    need = pa.workspace_size(s, good)
    assert L.pa_prefill(ctypes.byref(s), ctypes.byref(good), 16, st, 16, st, 16, st, 16, st, ctypes.byref(m), 256,
                        need - 1, None) == 3
    assert L.pa_prefill(ctypes.byref(s), ctypes.byref(good), 16, st, 16, st, 16, st, 16, st, ctypes.byref(m), None,
                        need, None) == 3


@pytest.mark.parametrize("lam", [-0.1, 1.5, float("nan")])
def test_bad_skip_threshold_rejected(L, lam):
    s = shape()
    st = pa.Strides(0, 512, 64)
    assert L.pa_block_sparse_attn_skip(ctypes.byref(s), 16, st, 16, st, 16, st, 16, 16, ctypes.c_float(0.125),
                                       ctypes.c_float(lam), 16, st, None, None, None) == 1
    assert b"skip_threshold" in L.pa_last_error()
    assert pa.workspace_size(s, pa.make_budget(pa.ALL, 0, 0, 1, lam)) == 0


def test_xattn_workspace_and_argument_errors(L):
    s = shape(N=1024, H=8)
    for S in (4, 8, 16):
        rows = 1024 // S
        a256 = lambda x: (x + 255) // 256 * 256
        assert L.pa_xattn_workspace_size(ctypes.byref(s), S) == a256(8 * 8 * rows * 4) + a256(8 * ((rows + 127) // 128) * rows * 4)
    assert L.pa_xattn_workspace_size(ctypes.byref(s), 2) == 0
    st = pa.Strides(0, 512, 64)
    for S, tau in ((3, 0.9), (32, 0.9), (8, 0.0), (8, 1.5)):
        assert L.pa_xattn_mask(ctypes.byref(s), S, ctypes.c_float(tau), 16, st, 16, st, 16, 16, None, 256, 1 << 30,
                               None) == 1
    assert L.pa_xattn_mask(ctypes.byref(s), 8, ctypes.c_float(0.9), 16, st, 16, st, 16, 16, None, 256, 16,
                           None) == 3


def test_noncausal_shape_sizes_and_errors(L):
    s = shape(N=1024, H=8, Hkv=2, d=64, G=2)
    s.non_causal = 1
    nb = 8
    a256 = lambda x: (x + 255) // 256 * 256
    fixed = pa.workspace_size(s, pa.make_budget(pa.FIXED_FRACTION, 0, 100))
    assert fixed == 2 * a256(2 * 1024 * 64 * 2) + a256(2 * nb * nb * 4)
    s.non_causal = 2
    assert pa.workspace_size(s, pa.make_budget(pa.FIXED_FRACTION, 0, 100)) == 0
    st = pa.Strides(0, 512, 64)
    assert L.pa_pool_heads(ctypes.byref(s), 16, st, 16, st, 16, 16, None) == 1


def test_varlen_validation_and_workspace(L):
    s = shape(N=2560, H=8, Hkv=2, d=64, G=2)
    b = pa.make_budget(pa.DYNAMIC, 0.9)
    cu = (ctypes.c_int32 * 5)(0, 384, 1408, 1536, 2560)
    longest = shape(N=1024, H=8, Hkv=2, d=64, G=2)
    assert L.pa_workspace_size_varlen(ctypes.byref(s), ctypes.byref(b), 4, cu) == pa.workspace_size(longest, b)
    st = pa.Strides(0, 512, 64)
    m = pa.MaskBufs(16, 16, 16, 16)
    for bad, code in (((0, 384, 1400, 1536, 2560), 2), ((128, 384, 1408, 1536, 2560), 1),
                      ((0, 384, 1408, 1536, 2432), 1), ((0, 384, 384, 1536, 2560), 2)):
        c = (ctypes.c_int32 * 5)(*bad)
        assert L.pa_workspace_size_varlen(ctypes.byref(s), ctypes.byref(b), 4, c) == 0
        assert L.pa_prefill_varlen(ctypes.byref(s), ctypes.byref(b), 4, c, 16, st, 16, st, 16, st, 16, st,
                                   ctypes.byref(m), 256, 1 << 30, None) == code
    s2 = shape(B=2, N=2560, H=8, Hkv=2, d=64, G=2)
    assert L.pa_prefill_varlen(ctypes.byref(s2), ctypes.byref(b), 4, cu, 16, st, 16, st, 16, st, 16, st,
                               ctypes.byref(m), 256, 1 << 30, None) == 1
    assert L.pa_prefill_varlen(ctypes.byref(s), ctypes.byref(b), 4, None, 16, st, 16, st, 16, st, 16, st,
                               ctypes.byref(m), 256, 1 << 30, None) == 1


def test_attention_argument_errors(L):
    s = shape()
    st = pa.Strides(0, 512, 64)
    assert L.pa_block_sparse_attn(ctypes.byref(s), 16, st, 16, st, 16, st, 16, 16, ctypes.c_float(0.0), 16, st, None,
                                  None) == 1
    assert L.pa_block_sparse_attn(ctypes.byref(s), 16, st, 16, st, 16, st, None, 16, ctypes.c_float(0.125), 16, st,
                                  None, None) == 1
    assert L.pa_block_sparse_attn(ctypes.byref(s), 16, st, 16, st, 16, st, 16, 16, ctypes.c_float(0.125), 16, st,
                                  2, None) == 1  # misaligned lse


def test_binding_refuses_cpu_tensors():
    import torch
    q = torch.zeros(1, 128, 2, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        pa.pool_heads(q, q, 1)


def test_header_compiles_and_links_as_plain_c(tmp_path):
    """A C99 program (tests/c/abi_from_c.c) includes pa.h, links libpa.so and
    gets argument errors back without a GPU."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("no C compiler")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    libdir = os.path.dirname(pa.LIB_PATH)
    exe = tmp_path / "abi_from_c"
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(root, "include"),
                         os.path.join(root, "tests", "c", "abi_from_c.c"), "-o", str(exe),
                         "-L", libdir, "-l:libpa.so", f"-Wl,-rpath,{libdir}"], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stdout + run.stderr
