"""Engagement counters on the host (no GPU): every entry point that enqueues
work is counted under its C name, refusals and no-op calls are told apart from
calls that reached a kernel, a call made on another entry point's behalf
counts once, and the counts stay exact under concurrent callers (grouped-nf4-gemm
releases, v0.2.6 "Honest instrumentation": a patch count is not a call count)."""
import ctypes
import re
import threading

import pytest

from bit_grouped_moe_b200 import build


@pytest.fixture(scope="module")
def g():
    build.build()
    from bit_grouped_moe_b200 import gnf4
    return gnf4


ONE = ctypes.c_void_p(16)  # a non-NULL offsets pointer; never dereferenced by the host checks


def _fresh(g):
    g.call_stats_get(None, reset=True)


def test_every_work_entry_point_is_counted(g):
    hdr = open(g.HEADER_PATH).read()
    status_calls = set(re.findall(r"^gnf4_status\s+(gnf4_\w+)\s*\(", hdr, flags=re.M))
    diagnostics = {"gnf4_device_errors", "gnf4_selftest_bounded_wait", "gnf4_call_stats_get"}
    names = g.call_stats_names()
    assert len(names) == len(set(names))
    assert set(names) == status_calls - diagnostics
    assert g.call_stats_name(-1) is None and g.call_stats_name(len(names)) is None


def test_refusal_and_no_op_are_not_engagement(g):
    _fresh(g)
    f = g._lib.gnf4_grouped_gemm_nf4
    assert f(None, None, None, ONE, None, 0, 64, 64, 8, None, None) == g.ERR_UNSUPPORTED_SHAPE  # E = 0
    assert f(None, None, None, ONE, None, 4, 64, 64, 0, None, None) == g.OK  # M = 0: nothing to enqueue
    s = g.call_stats_get("gnf4_grouped_gemm_nf4")
    assert s == {"calls": 2, "refused": 1, "engaged": 0, "rows": 0, "decode_path": 0, "native_path": 0,
                 "gemv_path": 0}
    # other entry points untouched
    assert g.call_stats_get("gnf4_grouped_gemm_mxfp4")["calls"] == 0
    assert g.call_stats_get(None)["calls"] == 2


def test_each_entry_point_counts_under_its_own_name(g):
    _fresh(g)
    L = g._lib
    L.gnf4_grouped_gemv_mxfp4(None, None, None, ONE, None, 4, 60, 64, 8, None, None)  # N % 8 != 0
    L.gnf4_grouped_gemm_mxfp4_ws(None, None, None, ONE, None, 4, 60, 256, 8, None, None, 0, None)
    L.gnf4_grouped_gemm_mxfp4_ws(None, None, None, ONE, None, 4, 64, 256, 8, None, None, 0, None)  # host pointers
    L.gnf4_combine(None, None, None, -1, 2, 64, None, None)  # T < 0
    L.gnf4_route_permute(None, None, 4, 0, 8, 64, None, None, None, None, None, 0, None, None)  # k = 0
    assert g.call_stats_get("gnf4_grouped_gemv_mxfp4")["refused"] == 1
    ws = g.call_stats_get("gnf4_grouped_gemm_mxfp4_ws")
    assert ws["calls"] == 2 and ws["refused"] == 2 and ws["engaged"] == 0
    assert g.call_stats_get("gnf4_combine")["refused"] == 1
    assert g.call_stats_get("gnf4_route_permute")["refused"] == 1
    total = g.call_stats_get(None)
    assert total["calls"] == 5 and total["refused"] == 5


def test_a_call_made_for_another_entry_point_counts_once(g):
    """gnf4_route_permute_static runs gnf4_route_permute; only the outer call is counted."""
    _fresh(g)
    # over the static array's size: refused before the inner call
    assert g._lib.gnf4_route_permute_static(None, None, 1 << 20, 8, 4096, 64, ONE, None, None, None, None,
                                            None) == g.ERR_UNSUPPORTED_SHAPE
    # a small shape reaches the device lookup (no device here, or host pointers later): refused either way
    assert g._lib.gnf4_route_permute_static(None, None, 4, 2, 8, 64, ONE, None, None, None, None, None) != g.OK
    assert g.call_stats_get("gnf4_route_permute_static")["calls"] == 2
    assert g.call_stats_get("gnf4_route_permute_static")["refused"] == 2
    assert g.call_stats_get("gnf4_route_permute")["calls"] == 0


def test_reset_and_unknown_names(g):
    _fresh(g)
    g._lib.gnf4_grouped_gemm_nf4(None, None, None, ONE, None, 0, 64, 64, 8, None, None)
    assert g.call_stats_get("gnf4_grouped_gemm_nf4", reset=True)["calls"] == 1
    assert g.call_stats_get("gnf4_grouped_gemm_nf4")["calls"] == 0
    with pytest.raises(g.Gnf4Error) as e:
        g.call_stats_get("gnf4_no_such_call")
    assert e.value.status == g.ERR_INVALID_ARG
    with pytest.raises(g.Gnf4Error):
        g.call_stats_get("gnf4_call_stats_get")  # the read-out itself is not counted
    assert g._lib.gnf4_call_stats_get(None, None, 0) == g.ERR_INVALID_ARG


def test_counts_are_exact_under_concurrent_callers(g):
    """ctypes drops the GIL around the call, so the threads really race on the counters."""
    _fresh(g)
    f = g._lib.gnf4_grouped_gemm_nf4
    n_threads, n_calls = 8, 2000

    def worker():
        for _ in range(n_calls):
            f(None, None, None, ONE, None, 0, 64, 64, 8, None, None)

    ts = [threading.Thread(target=worker) for _ in range(n_threads)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    s = g.call_stats_get("gnf4_grouped_gemm_nf4")
    assert s["calls"] == n_threads * n_calls and s["refused"] == n_threads * n_calls
