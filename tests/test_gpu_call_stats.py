"""Engagement counters on the GPU: which kernel family each accepted call
reached (status page, "What is open": a silent fallback made countable).

The MXFP4 GEMM with a workspace is the call with a fallback: groups of at most
96 rows go to the native block-scaled kernel, the others to the decode-path
kernel, and without a workspace (or on a shape the native kernel does not
take) every group goes to the decode path.  The counters tell these apart.
Outputs are checked against the oracle by the parity tests; here only the
counts are."""
import numpy as np
import pytest
import torch

from bit_grouped_moe_b200 import inputs
from tests._util import offsets_from_counts, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    assert torch.cuda.is_available()
    from bit_grouped_moe_b200 import gnf4
    gnf4.device_errors(clear=True)
    return gnf4


def _mx(groups, K, N, seed):
    E = len(groups)
    offsets = offsets_from_counts(groups)
    M = int(offsets[-1])
    w, sc = inputs.mxfp4_random(inputs.rng(seed), E, N, K)
    a = inputs.bf16_normal(inputs.rng(seed + 1), (M, K))
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    return to_dev_bf16(a), to_dev(w), to_dev(sc), y, to_dev(offsets), M


def _ws_stats(g):
    return g.call_stats_get("gnf4_grouped_gemm_mxfp4_ws", reset=True)


@pytest.mark.parametrize("groups,K,with_ws,native,decode", [
    ([3, 5, 0, 17], 512, True, 1, 0),                # M <= 96: the native kernel alone
    ([0, 1, 95, 96, 97, 200, 7], 512, True, 1, 1),   # both kernels
    ([0, 1, 95, 96, 97, 200, 7], 512, False, 0, 1),  # no workspace: the decode path throughout
    ([3, 5, 0, 17], 416, True, 0, 1),                # K % 64 != 0: the decode path
])
def test_mxfp4_ws_reports_the_path_it_took(g, groups, K, with_ws, native, decode):
    g.call_stats_get(None, reset=True)
    a, w, sc, y, off, M = _mx(groups, K, 256, seed=40 + K + len(groups))
    ws = None
    if with_ws:
        n = g.mxfp4_workspace_bytes(M, K)
        ws = torch.empty(max(n, 256), dtype=torch.uint8, device="cuda")
    g.grouped_gemm_mxfp4_ws(a, w, sc, y, ws, offsets=off)
    torch.cuda.synchronize()
    s = _ws_stats(g)
    assert s == {"calls": 1, "refused": 0, "engaged": 1, "rows": M, "decode_path": decode, "native_path": native,
                 "gemv_path": 0}
    assert g.device_errors() == 0


def test_gemm_gemv_and_route_count_their_own_family(g):
    g.call_stats_get(None, reset=True)
    E, k, T, K, N = 8, 2, 16, 256, 128
    # token t picks experts t % E and (t + 3) % E: four rows per expert, inside the GEMV's limit
    ids = np.array([[t % E, (t + 3) % E] for t in range(T)], dtype=np.int32)
    x = torch.randn(T, K, device="cuda").to(torch.bfloat16)
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    s2f = torch.empty(T * k, dtype=torch.int32, device="cuda")
    f2s = torch.empty(T * k, dtype=torch.int32, device="cuda")
    xs = torch.empty(T * k, K, dtype=torch.bfloat16, device="cuda")
    g.route_permute_static(torch.from_numpy(ids).cuda(), x, E, off, s2f, f2s, xs)
    w = inputs.device_random_bytes(5, (E, N, K // 2))
    am = torch.rand(E, N, K // 64, device="cuda") + 0.5
    y = torch.empty(T * k, N, dtype=torch.bfloat16, device="cuda")
    g.grouped_gemm_nf4(xs, w, am, y, offsets=off)
    y2 = torch.empty_like(y)
    g.grouped_gemv_nf4(xs, w, am, y2, offsets=off)
    torch.cuda.synchronize()
    assert int(torch.diff(off).max()) == 4
    st = g.call_stats_get("gnf4_route_permute_static")
    assert st["calls"] == 1 and st["engaged"] == 1 and st["rows"] == T * k
    assert g.call_stats_get("gnf4_route_permute")["calls"] == 0  # run on the static call's behalf
    gm = g.call_stats_get("gnf4_grouped_gemm_nf4")
    assert gm["engaged"] == 1 and gm["decode_path"] == 1 and gm["native_path"] == 0 and gm["gemv_path"] == 0
    gv = g.call_stats_get("gnf4_grouped_gemv_nf4")
    assert gv["engaged"] == 1 and gv["gemv_path"] == 1 and gv["decode_path"] == 0
    assert g.device_errors() == 0


def test_fused_combine_without_rows_engages_no_gemm(g):
    """No routed row: the call only zeroes out (engaged, but no GEMM family)."""
    g.call_stats_get(None, reset=True)
    E, T, k, K, N = 4, 5, 2, 256, 128
    w = inputs.device_random_bytes(6, (E, N, K // 2))
    sc = inputs.device_random_bytes(7, (E, N, K // 32), lo=120, hi=130)
    a = torch.empty(0, K, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(0, N, dtype=torch.bfloat16, device="cuda")
    off = torch.zeros(E + 1, dtype=torch.int32, device="cuda")
    f2s = torch.full((T * k,), -1, dtype=torch.int32, device="cuda")
    wts = torch.ones(T, k, dtype=torch.float32, device="cuda")
    out = torch.full((T, N), 7.0, dtype=torch.bfloat16, device="cuda")
    cnt = torch.zeros(max(g.combine_counters_bytes(T, N) // 4, 1), dtype=torch.int32, device="cuda")
    s2f = torch.empty(0, dtype=torch.int32, device="cuda")
    g.grouped_gemm_mxfp4_combine(a, w, sc, y, s2f, f2s, wts, out, cnt, offsets=off)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out.float()).item() == 0
    s = g.call_stats_get("gnf4_grouped_gemm_mxfp4_combine")
    assert s["calls"] == 1 and s["engaged"] == 1 and s["rows"] == 0
    assert s["decode_path"] == 0 and s["native_path"] == 0 and s["gemv_path"] == 0
    assert g.device_errors() == 0
