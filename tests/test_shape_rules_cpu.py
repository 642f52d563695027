"""The shape rules written in include/gnf4.h are the rules the library
enforces: for shapes drawn around every documented bound, a call returns
GNF4_ERR_UNSUPPORTED_SHAPE exactly when a rule of its header comment is
broken ("#324's pre-launch shape refusal", grouped-nf4-gemm status page).

Each predicate below restates the header's "Rules:" text for that call.  Calls
are made with zero rows (or tokens), or with NULL / host data pointers, so an
accepted shape either returns GNF4_OK with nothing enqueued or stops at a
pointer check; no call reaches a device."""
import ctypes

import pytest
from hypothesis import given, settings, strategies as st

from bit_grouped_moe_b200 import build

ONE = ctypes.c_void_p(16)  # a non-NULL group description; never dereferenced on the host
SHAPE = 2
SETTINGS = settings(max_examples=150, deadline=None, derandomize=True)
_G = None  # the binding, set by the fixture (refused() reads its last_error)


@pytest.fixture(scope="module")
def g():
    global _G
    build.build()
    from bit_grouped_moe_b200 import gnf4
    _G = gnf4
    return gnf4


def around(*bounds, lo=-2, hi=70000):
    """Integers near each bound (bound-1, bound, bound+1) mixed with uniform draws."""
    near = sorted({b + d for b in bounds for d in (-1, 0, 1)})
    return st.one_of(st.sampled_from(near), st.integers(lo, hi))


E_ = around(0, 1, 1024, 4096, hi=5000)
N_ = st.one_of(around(0, 1, 8, 64), st.integers(0, 4096).map(lambda n: 8 * n))
K_ = st.one_of(around(0, 8, 32, 64, 128, 256, 65536), st.integers(0, 2100).map(lambda n: 32 * n))
M_ = st.integers(-2, 3)


def grouped_ok(kq, E, N, K, M):
    # "1 <= E <= 1024, N >= 1, N % 8 == 0, K % 64 == 0, 64 <= K <= 65536, M >= 0" (MXFP4: 32 for 64)
    return 1 <= E <= 1024 and N >= 1 and N % 8 == 0 and K % kq == 0 and kq <= K <= 65536 and M >= 0


def refused(status):
    """True for GNF4_ERR_UNSUPPORTED_SHAPE, which must come with a message naming what was wrong."""
    if status == SHAPE and _G is not None:
        msg = _G.last_error()
        assert msg and any(w in msg for w in ("E=", "N=", "K=", "M=", "I=", "T=", "k=", "rows=", "too large", "T*k",
                                              "E*N")), msg
    return status == SHAPE


@SETTINGS
@given(E=E_, N=N_, K=K_, M=M_)
def test_grouped_gemm_gemv_dgrad_and_ws_rules(g, E, N, K, M):
    L = g._lib
    for fmt, kq, calls in (("nf4", 64, (L.gnf4_grouped_gemm_nf4, L.gnf4_grouped_gemv_nf4, L.gnf4_grouped_dgrad_nf4)),
                           ("mxfp4", 32, (L.gnf4_grouped_gemm_mxfp4, L.gnf4_grouped_gemv_mxfp4,
                                          L.gnf4_grouped_dgrad_mxfp4))):
        want = not grouped_ok(kq, E, N, K, M)
        for f in calls:
            assert refused(f(None, None, None, ONE, None, E, N, K, M, None, None)) == want, (fmt, f, g.last_error())
    # the workspace call keeps the MXFP4 GEMM's rules; its native path adds no refusal
    st_ws = L.gnf4_grouped_gemm_mxfp4_ws(None, None, None, ONE, None, E, N, K, M, None, None, 0, None)
    assert refused(st_ws) == (not grouped_ok(32, E, N, K, M)), g.last_error()


@SETTINGS
@given(E=E_, I=st.one_of(around(0, 64, 1 << 29, hi=1 << 30), st.integers(0, 64).map(lambda n: 64 * n)), K=K_, M=M_)
def test_swiglu_rules(g, E, I, K, M):
    L = g._lib
    # "I must be a positive multiple of 64, at most 2^29", the rest as the GEMM with N = 2I
    i_ok = 64 <= I <= (1 << 29) and I % 64 == 0
    for f, kq in ((L.gnf4_grouped_gemm_nf4_swiglu, 64), (L.gnf4_grouped_gemv_nf4_swiglu, 64),
                  (L.gnf4_grouped_gemm_mxfp4_swiglu, 32), (L.gnf4_grouped_gemv_mxfp4_swiglu, 32)):
        want = not (i_ok and grouped_ok(kq, E, 2 * I if i_ok else 8, K, M))
        assert refused(f(None, None, None, ONE, None, E, I, K, M, None, None)) == want, g.last_error()


@SETTINGS
@given(E=E_, N=st.one_of(N_, st.sampled_from([(1 << 21) - 8, 1 << 21, (1 << 21) + 8, 1 << 22])), K=K_, M=M_)
def test_native_mode_rules(g, E, N, K, M):
    L = g._lib
    base = 1 <= E <= 1024 and N >= 1 and N % 8 == 0 and M >= 0 and E * N < (1 << 31)
    # W4A8 and the two-term form: "K must be a multiple of 64 in [128, 65536], and E*N < 2^31"
    w4a8_ok = base and K % 64 == 0 and 128 <= K <= 65536
    assert refused(L.gnf4_grouped_gemm_w4a8(None, None, None, None, ONE, None, E, N, K, M, None, None)) == \
        (not w4a8_ok), g.last_error()
    assert refused(L.gnf4_grouped_gemm_w4a8x2(None, None, ONE, ONE, None, None, ONE, None, E, N, K, M, None,
                                              None)) == (not w4a8_ok), g.last_error()
    # W4A4: "K must be a multiple of 64 in [256, 65536]; other rules as gnf4_grouped_gemm_w4a8"
    w4a4_ok = base and K % 64 == 0 and 256 <= K <= 65536
    assert refused(L.gnf4_grouped_gemm_w4a4(None, None, None, None, ONE, None, E, N, K, M, None, None)) == \
        (not w4a4_ok), g.last_error()


@SETTINGS
@given(M=M_, K=K_)
def test_quantiser_rules(g, M, K):
    L = g._lib
    # "K must be a positive multiple of 32 and M >= 0"
    want = not (M >= 0 and K >= 32 and K % 32 == 0)
    assert refused(L.gnf4_quantize_mxfp8(None, M, K, None, None, None)) == want
    assert refused(L.gnf4_quantize_mxfp8_split(None, M, K, None, None, None, None, None)) == want
    assert refused(L.gnf4_quantize_mxfp4_act(None, M, K, None, None, None)) == want


T_ = st.one_of(st.integers(-2, 3), st.sampled_from([1 << 20, (1 << 27) - 1, 1 << 27, (1 << 28) + 1, 1 << 30]))
k_ = around(0, 1, 8, 32, lo=-1, hi=5000)


@SETTINGS
@given(T=T_, k=k_, E=E_, K=around(0, 8, 7168, lo=-2, hi=20000))
def test_routing_rules(g, T, k, E, K):
    L = g._lib
    # "T >= 0, 1 <= k <= E <= 4096, T*k <= 2^30, K >= 8 and K % 8 == 0"
    ok = T >= 0 and 1 <= k <= E <= 4096 and T * k <= (1 << 30) and K >= 8 and K % 8 == 0
    st_r = L.gnf4_route_permute(None, None, T, k, E, K, None, None, None, None, None, 0, None, None)
    assert refused(st_r) == (not ok), g.last_error()
    # the router epilogue: "1 <= k <= min(E, 32), E <= 4096, other shape rules as gnf4_route_permute"
    st_t = L.gnf4_route_topk_permute(None, None, T, E, k, None, K, None, None, None, None, None, None, None, 0, None)
    assert refused(st_t) == (not (ok and k <= 32)), g.last_error()


@SETTINGS
@given(T=T_, k=k_, N=N_, E=E_, K=K_, M=M_)
def test_combine_rules(g, T, k, N, E, K, M):
    L = g._lib
    # "T >= 0, k >= 1, T*k < 2^31, N >= 8 and N % 8 == 0"
    c_ok = T >= 0 and k >= 1 and T * k < (1 << 31)
    assert refused(L.gnf4_combine(None, None, None, T, k, N, None, None)) == (not (c_ok and N >= 8 and N % 8 == 0))
    # fused forms: the combine's T / k rules and the GEMM's shape rules
    for f, kq in ((L.gnf4_grouped_gemv_nf4_combine, 64), (L.gnf4_grouped_gemm_mxfp4_combine, 32)):
        want = not (c_ok and grouped_ok(kq, E, N, K, M))
        st_f = f(None, None, None, ONE, None, E, N, K, M, None, None, None, None, T, k, None, None, None)
        assert refused(st_f) == want, g.last_error()


@SETTINGS
@given(rows=st.integers(-2, 3), K=K_)
def test_dequant_rules(g, rows, K):
    L = g._lib
    # NF4: "K >= 64 and K % 64 == 0, rows >= 0"; MXFP4: "K >= 32 and K % 32 == 0, rows >= 0"
    assert refused(L.gnf4_dequant_nf4_f32(None, None, rows, K, None, None)) == \
        (not (rows >= 0 and K >= 64 and K % 64 == 0))
    assert refused(L.gnf4_dequant_mxfp4_f32(None, None, rows, K, None, None)) == \
        (not (rows >= 0 and K >= 32 and K % 32 == 0))


@SETTINGS
@given(M=st.integers(-2, 1 << 20), K=K_)
def test_workspace_size_is_zero_exactly_where_the_native_path_does_not_apply(g, M, K):
    n = g.grouped_gemm_mxfp4_workspace_bytes(M, K)
    applies = M >= 1 and K >= 128 and K % 64 == 0 and K <= 65536
    assert (n > 0) == applies
    if applies:
        sc = (M * (K // 32) + 15) // 16 * 16
        assert n == 2 * M * K + 2 * sc
