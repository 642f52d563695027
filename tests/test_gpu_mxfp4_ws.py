"""The MXFP4 grouped GEMM with a workspace (gnf4_grouped_gemm_mxfp4_ws): groups
of at most 96 rows on the native two-term block-scaled path, larger groups on
the decode path.

- Parity: the standard tolerance of the path against the bf16-activation
  oracle, on a group mix that straddles the 96-row split (grouped-nf4-gemm
  releases, v0.2.0 "the MXFP4 native-byte lane").
- Structure: the rows of the small groups are bit-identical to the two-term
  native GEMM (split quantiser + gnf4_grouped_gemm_w4a8x2), the rows of the
  large groups to gnf4_grouped_gemm_mxfp4; without a workspace every row is
  the decode path's.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_grouped_moe_b200 import inputs
from tests._util import assert_within_tolerance, bf16_to_f64, offsets_from_counts, set_oracle_threads, to_dev, \
    to_dev_bf16

pytestmark = pytest.mark.gpu

# around the split (96), the 128-row weight tile and the 256-row decode unit
GROUPS = [0, 1, 2, 31, 95, 96, 97, 0, 128, 200, 7, 300, 64, 33]


@pytest.fixture(scope="module")
def g():
    assert torch.cuda.is_available()
    from bit_grouped_moe_b200 import gnf4
    set_oracle_threads()
    gnf4.device_errors(clear=True)
    return gnf4


def _case(K, N, seed, groups=GROUPS):
    E = len(groups)
    offsets = offsets_from_counts(groups)
    M = int(offsets[-1]) + 3  # rows past offsets[E] stay untouched
    w, sc = inputs.mxfp4_random(inputs.rng(seed), E, N, K)
    a = inputs.bf16_normal(inputs.rng(seed + 1), (M, K))
    return offsets, M, w, sc, a


def _ws(g, M, K):
    n = g.mxfp4_workspace_bytes(M, K)
    assert n > 0
    return torch.empty(n, dtype=torch.uint8, device="cuda")


def test_native_max_rows_is_the_two_term_unit(g):
    assert g.mxfp4_native_max_rows() == 96


@pytest.mark.parametrize("K,N", [(320, 392), (512, 256), (2880, 264)])
def test_ws_parity_against_the_oracle(g, K, N):
    offsets, M, w, sc, a = _case(K, N, seed=900 + K)
    y = torch.full((M, N), -3.0, dtype=torch.bfloat16, device="cuda")
    g.grouped_gemm_mxfp4_ws(to_dev_bf16(a), to_dev(w), to_dev(sc), y, _ws(g, M, K), offsets=to_dev(offsets))
    torch.cuda.synchronize()
    assert g.device_errors() == 0
    nv = int(offsets[-1])
    got = bf16_to_f64(y)
    assert_within_tolerance(got[:nv], oracle.grouped_gemm_mxfp4(a, w, sc, offsets), f"mxfp4 ws K={K}")
    assert np.all(got[nv:] == -3.0), "rows past offsets[E] were written"


@pytest.mark.parametrize("use_counts", [False, True])
def test_ws_rows_come_from_the_two_paths_bit_for_bit(g, use_counts):
    K, N = 384, 264
    offsets, M, w, sc, a = _case(K, N, seed=950)
    a_d, w_d, sc_d = to_dev_bf16(a), to_dev(w), to_dev(sc)
    grp = dict(counts=to_dev(np.array(GROUPS, np.int32))) if use_counts else dict(offsets=to_dev(offsets))
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    g.grouped_gemm_mxfp4_ws(a_d, w_d, sc_d, y, _ws(g, M, K), **grp)
    y_dec = torch.empty_like(y)
    g.grouped_gemm_mxfp4(a_d, w_d, sc_d, y_dec, **grp)
    hq = torch.empty(M, K, dtype=torch.uint8, device="cuda")
    hs = torch.empty(M, K // 32, dtype=torch.uint8, device="cuda")
    lq, ls = torch.empty_like(hq), torch.empty_like(hs)
    g.quantize_mxfp8_split(a_d, hq, hs, lq, ls)
    y_nat = torch.empty_like(y)
    g.grouped_gemm_w4a8x2(hq, hs, lq, ls, w_d, sc_d, y_nat, **grp)
    y_none = torch.empty_like(y)
    g.grouped_gemm_mxfp4_ws(a_d, w_d, sc_d, y_none, None, **grp)
    torch.cuda.synchronize()
    assert g.device_errors() == 0
    bits = lambda t: t.view(torch.int16).cpu().numpy()
    got, dec, nat = bits(y), bits(y_dec), bits(y_nat)
    for e, r in enumerate(GROUPS):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        ref = nat if r <= 96 else dec
        assert np.array_equal(got[lo:hi], ref[lo:hi]), f"group {e} ({r} rows) is not from the expected path"
    nv = int(offsets[-1])
    assert np.array_equal(bits(y_none)[:nv], dec[:nv]), "without a workspace every row is the decode path's"


def test_ws_all_small_groups_and_tiny_M(g):
    """M <= 96: only the native launches run."""
    groups = [5, 0, 40, 1]
    K, N = 256, 128
    offsets, M, w, sc, a = _case(K, N, seed=970, groups=groups)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    g.grouped_gemm_mxfp4_ws(to_dev_bf16(a), to_dev(w), to_dev(sc), y, _ws(g, M, K), offsets=to_dev(offsets))
    torch.cuda.synchronize()
    assert g.device_errors() == 0
    nv = int(offsets[-1])
    assert_within_tolerance(bf16_to_f64(y)[:nv], oracle.grouped_gemm_mxfp4(a, w, sc, offsets), "mxfp4 ws small")


def test_ws_refuses_a_short_workspace(g):
    K, N = 256, 128
    offsets, M, w, sc, a = _case(K, N, seed=980, groups=[3, 4])
    need = g.mxfp4_workspace_bytes(M, K)
    short = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(g.Gnf4Error, match="workspace"):
        g.grouped_gemm_mxfp4_ws(to_dev_bf16(a), to_dev(w), to_dev(sc), y, short, offsets=to_dev(offsets))


def test_ws_shapes_outside_the_native_rules_take_the_decode_path(g):
    """K % 64 != 0: no workspace size, and a workspace passed anyway is unused."""
    K, N = 96, 128
    assert g.mxfp4_workspace_bytes(10, K) == 0
    offsets, M, w, sc, a = _case(K, N, seed=990, groups=[3, 0, 9])
    a_d, w_d, sc_d, off_d = to_dev_bf16(a), to_dev(w), to_dev(sc), to_dev(offsets)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    y_dec = torch.empty_like(y)
    g.grouped_gemm_mxfp4_ws(a_d, w_d, sc_d, y, torch.empty(4096, dtype=torch.uint8, device="cuda"), offsets=off_d)
    g.grouped_gemm_mxfp4(a_d, w_d, sc_d, y_dec, offsets=off_d)
    torch.cuda.synchronize()
    nv = int(offsets[-1])
    assert torch.equal(y[:nv].view(torch.int16), y_dec[:nv].view(torch.int16))
