"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point the header declares, and refuses bad shapes and host
pointers before it would touch the device."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from bit_grouped_moe_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib_path():
    return build.build()


@pytest.fixture(scope="module")
def g(lib_path):
    from bit_grouped_moe_b200 import gnf4
    return gnf4


def test_header_symbols_exported(lib_path, g):
    names = g.declared_symbols()
    assert len(names) >= 12, names
    for required in ("gnf4_route_permute", "gnf4_grouped_gemm_nf4", "gnf4_grouped_gemm_mxfp4",
                     "gnf4_grouped_gemv_nf4", "gnf4_grouped_gemv_mxfp4", "gnf4_combine"):
        assert required in names
    lib = ctypes.CDLL(lib_path)
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/gnf4.h but not exported"
    out = subprocess.run(["nm", "-D", "--defined-only", lib_path], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (gnf4_\w+)", out))
    assert set(names) <= exported


def test_version(g):
    assert "sm_100a" in g.version()


def test_route_workspace_size(g):
    assert g.route_workspace_bytes(16, 2, 8) >= (8 + 1) * 4
    assert g.route_workspace_bytes(4096, 8, 384) >= 128 * 384 * 4
    assert g.route_workspace_bytes(0, 2, 8) == 0
    assert g.route_workspace_bytes(4, 0, 8) == 0


def test_binding_sets_argtypes_for_every_call(g):
    """The binding passes pointers as plain ints: each entry point it calls
    must declare its argument types, or a pointer would be cut to a C int."""
    import re
    src = open(g.__file__).read()
    called = set(re.findall(r"_lib\.(gnf4_\w+)", src)) | set(re.findall(r"\"(gnf4_\w+)\"", src))
    assert called
    missing = [n for n in sorted(called) if getattr(g._lib, n).argtypes is None and n not in ("gnf4_last_error",
                                                                                               "gnf4_version")]
    assert not missing, missing


def test_every_entry_point_has_a_same_name_binding(g):
    """The binding exposes each C entry point under its name without the gnf4_ prefix."""
    import re
    hdr = open(g.HEADER_PATH).read()
    names = sorted(set(re.findall(r"\b(gnf4_\w+)\s*\(", hdr)))
    assert len(names) > 20
    missing = [n for n in names if not hasattr(g, n[len("gnf4_"):])]
    assert not missing, missing


def test_mxfp4_workspace_size(g):
    """hi and lo e4m3 codes [M, K] plus hi and lo e8m0 scales [M, K/32], each part 16-byte aligned; 0 where the
    native path does not apply (K % 64 != 0 or K < 128)."""
    for M, K in [(1, 128), (33, 2880), (32768, 7168), (7, 192)]:
        sc = (M * (K // 32) + 15) // 16 * 16
        assert g.mxfp4_workspace_bytes(M, K) == 2 * M * K + 2 * sc
    for M, K in [(0, 256), (8, 96), (8, 64), (8, 160), (-1, 256)]:
        assert g.mxfp4_workspace_bytes(M, K) == 0
    assert g.mxfp4_native_max_rows() == 96


def test_mxfp4_ws_refusals(g):
    f = g._lib.gnf4_grouped_gemm_mxfp4_ws
    one = ctypes.c_void_p(16)
    # the shape rules of the MXFP4 GEMM, before any pointer
    assert f(None, None, None, one, None, 4, 60, 256, 8, None, None, 0, None) == g.ERR_UNSUPPORTED_SHAPE
    assert f(None, None, None, None, None, 4, 64, 256, 8, None, None, 0, None) == g.ERR_INVALID_ARG
    assert f(None, None, None, one, None, 4, 64, 256, 0, None, None, 0, None) == 0  # M == 0: nothing to do


def _raw(g, name, *args):
    return getattr(g._lib, name)(*args)


@pytest.mark.parametrize("E,N,K,fmt,expect", [
    (0, 64, 64, "nf4", 2), (1025, 64, 64, "nf4", 2), (4, 60, 64, "nf4", 2),
    (4, 64, 96, "nf4", 2), (4, 64, 48, "mxfp4", 2), (4, 64, 0, "mxfp4", 2),
])
def test_gemm_shape_refusals(g, E, N, K, fmt, expect):
    fn = g._lib.gnf4_grouped_gemm_nf4 if fmt == "nf4" else g._lib.gnf4_grouped_gemm_mxfp4
    st = fn(None, None, None, ctypes.c_void_p(16), None, E, N, K, 8, None, None)
    assert st == expect, g.last_error()
    assert g.last_error()


def test_exactly_one_group_description(g):
    for fn in (g._lib.gnf4_grouped_gemm_nf4, g._lib.gnf4_grouped_gemv_mxfp4):
        assert fn(None, None, None, None, None, 4, 64, 64, 8, None, None) == g.ERR_INVALID_ARG
        assert fn(None, None, None, ctypes.c_void_p(16), ctypes.c_void_p(16), 4, 64, 64, 8, None, None) \
            == g.ERR_INVALID_ARG


def test_empty_gemm_is_a_no_op(g):
    # M == 0 launches nothing and needs no device pointers
    assert g._lib.gnf4_grouped_gemm_nf4(None, None, None, ctypes.c_void_p(16), None, 4, 64, 64, 0, None, None) == 0


def test_host_pointers_refused(g):
    """A CPU buffer is never computed on: the call refuses it (no CPU fallback)."""
    a = np.zeros((8, 64), np.uint16)
    w = np.zeros((4, 64, 32), np.uint8)
    am = np.ones((4, 64, 1), np.float32)
    off = np.array([0, 2, 4, 6, 8], np.int32)
    y = np.zeros((8, 64), np.uint16)
    p = lambda x: x.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    st = g._lib.gnf4_grouped_gemm_nf4(p(a), p(w), p(am), p(off), None, 4, 64, 64, 8, p(y), None)
    assert st in (g.ERR_INVALID_ARG, g.ERR_CUDA)
    assert "device" in g.last_error() or "CUDA" in g.last_error() or "aligned" in g.last_error()


def test_route_refusals(g):
    f = g._lib.gnf4_route_permute
    assert f(None, None, 4, 0, 8, 64, None, None, None, None, None, 0, None, None) == g.ERR_UNSUPPORTED_SHAPE
    assert f(None, None, 4, 9, 8, 64, None, None, None, None, None, 0, None, None) == g.ERR_UNSUPPORTED_SHAPE
    assert f(None, None, 4, 2, 8, 60, None, None, None, None, None, 0, None, None) == g.ERR_UNSUPPORTED_SHAPE
    assert f(None, None, -1, 2, 8, 64, None, None, None, None, None, 0, None, None) == g.ERR_UNSUPPORTED_SHAPE


def test_combine_refusals(g):
    f = g._lib.gnf4_combine
    assert f(None, None, None, 4, 2, 12, None, None) == g.ERR_UNSUPPORTED_SHAPE
    assert f(None, None, None, 4, 0, 16, None, None) == g.ERR_UNSUPPORTED_SHAPE
    assert f(None, None, None, 0, 2, 16, None, None) == g.OK


def test_product_path_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "bit_grouped_moe_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, fn)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", text, re.M), fn
                assert "gnf4_oracle" not in text and "liboracle" not in text, fn


@pytest.mark.parametrize("name,K", [("gnf4_grouped_gemm_w4a8", 96), ("gnf4_grouped_gemm_w4a8", 64),
                                    ("gnf4_grouped_gemm_w4a8", 2848), ("gnf4_grouped_gemm_w4a4", 192),
                                    ("gnf4_grouped_gemm_w4a4", 320 + 32)])
def test_native_gemm_shape_refusals(g, name, K):
    """K rules of the native modes are checked before any pointer: W4A8 needs a
    multiple of 64 of at least 128, W4A4 a multiple of 64 of at least 256."""
    st = getattr(g._lib, name)(None, None, None, None, ctypes.c_void_p(16), None, 4, 64, K, 8, None, None)
    assert st == g.ERR_UNSUPPORTED_SHAPE, g.last_error()


def test_two_term_gemm_needs_both_terms(g):
    f = g._lib.gnf4_grouped_gemm_w4a8x2
    st = f(None, None, None, None, None, None, ctypes.c_void_p(16), None, 4, 64, 128, 8, None, None)
    assert st == g.ERR_INVALID_ARG and "lo_" in g.last_error()


@pytest.mark.parametrize("name", ["gnf4_quantize_mxfp8", "gnf4_quantize_mxfp4_act"])
def test_quantiser_refusals(g, name):
    f = getattr(g._lib, name)
    assert f(None, 4, 48, None, None, None) == g.ERR_UNSUPPORTED_SHAPE
    assert f(None, -1, 64, None, None, None) == g.ERR_UNSUPPORTED_SHAPE
    assert f(None, 0, 64, None, None, None) == g.OK  # nothing to do


def test_split_quantiser_refusals(g):
    f = g._lib.gnf4_quantize_mxfp8_split
    assert f(None, 4, 16, None, None, None, None, None) == g.ERR_UNSUPPORTED_SHAPE
    assert f(None, 0, 64, None, None, None, None, None) == g.OK


def test_fused_combine_gemv_refusals(g):
    f = g._lib.gnf4_grouped_gemv_nf4_combine
    off = ctypes.c_void_p(16)
    assert f(None, None, None, off, None, 4, 60, 64, 8, None, None, None, None, 2, 4, None, None, None) \
        == g.ERR_UNSUPPORTED_SHAPE  # N % 8
    assert f(None, None, None, off, None, 4, 64, 64, 8, None, None, None, None, 2, 0, None, None, None) \
        == g.ERR_UNSUPPORTED_SHAPE  # k < 1
    assert g.combine_counters_bytes(8, 2048) == 8 * 32 * 4
    assert g.combine_counters_bytes(8, 136) == 8 * 3 * 4


def test_selftest_limit_refusal(g):
    assert g._lib.gnf4_selftest_bounded_wait(0, None) == g.ERR_INVALID_ARG
    assert g._lib.gnf4_selftest_bounded_wait((1 << 32) + 1, None) == g.ERR_INVALID_ARG


DGRAD = ["gnf4_grouped_dgrad_nf4", "gnf4_grouped_dgrad_mxfp4"]


@pytest.mark.parametrize("name", DGRAD)
@pytest.mark.parametrize("E,N,K", [(0, 64, 64), (1025, 64, 64), (4, 60, 64), (4, 64, 0), (4, 64, 16)])
def test_dgrad_shape_refusals(g, name, E, N, K):
    """The data gradient takes the grouped GEMM's shape rules (N = the
    contracted weight rows, K = the output width) before any pointer."""
    st = getattr(g._lib, name)(None, None, None, ctypes.c_void_p(16), None, E, N, K, 8, None, None)
    assert st == g.ERR_UNSUPPORTED_SHAPE, g.last_error()


@pytest.mark.parametrize("name", DGRAD)
def test_dgrad_group_description_and_empty_call(g, name):
    f = getattr(g._lib, name)
    off = ctypes.c_void_p(16)
    assert f(None, None, None, None, None, 4, 64, 64, 8, None, None) == g.ERR_INVALID_ARG
    assert f(None, None, None, off, off, 4, 64, 64, 8, None, None) == g.ERR_INVALID_ARG
    assert f(None, None, None, off, None, 4, 64, 64, 0, None, None) == g.OK  # M == 0 launches nothing


def test_dgrad_host_pointers_refused(g):
    """A CPU buffer is never computed on: the call refuses it (no CPU fallback)."""
    dy = np.zeros((8, 64), np.uint16)
    w = np.zeros((4, 64, 32), np.uint8)
    am = np.ones((4, 64, 1), np.float32)
    off = np.array([0, 2, 4, 6, 8], np.int32)
    dx = np.zeros((8, 64), np.uint16)
    p = lambda x: x.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
    st = g._lib.gnf4_grouped_dgrad_nf4(p(dy), p(w), p(am), p(off), None, 4, 64, 64, 8, p(dx), None)
    assert st in (g.ERR_INVALID_ARG, g.ERR_CUDA)


@pytest.mark.parametrize("name", ["gnf4_grouped_gemm_nf4_swiglu", "gnf4_grouped_gemm_mxfp4_swiglu",
                                  "gnf4_grouped_gemv_nf4_swiglu", "gnf4_grouped_gemv_mxfp4_swiglu"])
def test_swiglu_width_refusals_and_empty_call(g, name):
    """The output width I must be a positive multiple of 64 (a gate_up stack
    of 2I rows, 64 gate + 64 up rows per weight tile)."""
    f = getattr(g._lib, name)
    off = ctypes.c_void_p(16)
    for width in (0, 32, 96, -64):
        assert f(None, None, None, off, None, 4, width, 64, 8, None, None) == g.ERR_UNSUPPORTED_SHAPE, width
    assert f(None, None, None, off, None, 4, 64, 64, 0, None, None) == g.OK  # M == 0 launches nothing


def test_library_needs_no_torch_or_python(lib_path):
    """The boundary is plain C over a self-contained library: libgnf4.so links the C/C++ runtime only (the CUDA
    runtime is static), never torch, c10 or libpython."""
    out = subprocess.run(["readelf", "-d", lib_path], capture_output=True, text=True).stdout
    needed = re.findall(r"\(NEEDED\)\s+Shared library: \[([^\]]+)\]", out)
    assert needed
    allowed = ("libstdc++", "libgcc_s", "libc.", "libm.", "ld-linux", "libdl", "librt", "libpthread")
    extra = [n for n in needed if not n.startswith(allowed)]
    assert not extra, extra
