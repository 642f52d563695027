"""Full-size parity of the dgrad, the native block-scaled MXFP4 modes and the
MXFP4 GEMM with a workspace (small groups native, large groups decoded) at the
Kimi-class shapes (384 experts, 4096 tokens top-8 with Zipf(1.2) skew; gate_up
K=7168 N=4096, down K=2048 N=7168), on sampled rows.

The stacks (up to 5.6 GB) are drawn on the device; the oracle decodes only the
experts of the sampled rows, compacted into a small stack.  Each mode is held
to the bound it is held to at small sizes: the two-term form and the dgrad to
the path's tolerance against the bf16-activation oracle, W4A8 and W4A4 to
2^-8 |ref| + 2^-12 max|ref| against their own oracle modes (quantised
activations).
"""
import numpy as np
import pytest
import torch

import oracle
from bit_grouped_moe_b200 import inputs
from tests._util import assert_within_tolerance, bf16_to_f64, offsets_from_counts, set_oracle_threads, to_dev, \
    to_dev_bf16

pytestmark = pytest.mark.gpu

OWN_REL = 2.0 ** -8
OWN_ABS_OF_MAX = 2.0 ** -12


@pytest.fixture(scope="module")
def g():
    assert torch.cuda.is_available()
    from bit_grouped_moe_b200 import gnf4
    set_oracle_threads()
    gnf4.device_errors(clear=True)
    return gnf4


@pytest.fixture(scope="module")
def routing():
    wl = inputs.WORKLOADS["kimi-prefill"]
    ids, _ = inputs.routing_for(wl, inputs.rng(41))
    off, _, _, _ = oracle.route(ids, wl.E)
    assert (np.diff(off) == 0).any(), "the skewed routing should leave empty experts"
    return wl, off


def _sampled(off, seed):
    """Rows of a dozen experts (the largest, the smallest non-empty, the first
    and last non-empty, random others): first, last and random rows of each."""
    rng = np.random.default_rng(seed)
    sizes = np.diff(off)
    ne = np.nonzero(sizes)[0]
    pick = {int(ne[0]), int(ne[-1]), int(ne[np.argmax(sizes[ne])]), int(ne[np.argmin(sizes[ne])])}
    rest = [e for e in ne if e not in pick]
    pick.update(int(e) for e in rng.choice(rest, size=min(len(rest), 8), replace=False))
    experts = sorted(pick)
    rows = set()
    for e in experts:
        lo, hi = int(off[e]), int(off[e + 1])
        rows.update([lo, hi - 1])
        rows.update(int(r) for r in rng.integers(lo, hi, size=min(2, hi - lo)))
    rows = np.array(sorted(rows), np.int64)
    sub_off = offsets_from_counts(sizes[experts])
    row_map = {}
    for i, e in enumerate(experts):
        for r in range(int(off[e]), int(off[e + 1])):
            row_map[r] = int(sub_off[i]) + (r - int(off[e]))
    sub_rows = np.array([row_map[int(r)] for r in rows], np.int64)
    return experts, rows, sub_off, sub_rows


def _own_bound(got, ref, what):
    amax = float(np.abs(ref).max())
    bad = np.argwhere(~(np.abs(got - ref) <= OWN_REL * np.abs(ref) + OWN_ABS_OF_MAX * amax))
    assert bad.size == 0, (f"{what}: {len(bad)} outputs out of tolerance (max|ref| {amax:.4g}), first "
                           + ", ".join(f"{tuple(i)} gpu={got[tuple(i)]:.6g} ref={ref[tuple(i)]:.6g}" for i in bad[:5]))


@pytest.mark.parametrize("mode", ["w4a8", "w4a8x2", "w4a4", "dgrad", "ws"])
@pytest.mark.parametrize("proj", [0, 1])
def test_kimi_native_modes_and_dgrad_sampled(g, routing, mode, proj):
    wl, off = routing
    E, M = wl.E, int(off[-1])
    p = wl.projections[proj]
    N, K = p.N, p.K
    w_d = inputs.device_random_bytes(60 + proj, (E, N, K // 2))
    sc_d = inputs.device_random_bytes(61 + proj, (E, N, K // 32), lo=118, hi=131)
    off_d = to_dev(off)
    experts, rows, sub_off, sub_rows = _sampled(off, seed=7 * proj + len(mode))
    w_small, s_small = w_d[experts].cpu().numpy(), sc_d[experts].cpu().numpy()
    if mode == "dgrad":
        dy = inputs.bf16_normal(inputs.rng(70 + proj), (M, N))
        dx = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
        g.grouped_dgrad_mxfp4(to_dev_bf16(dy), w_d, sc_d, dx, offsets=off_d)
        torch.cuda.synchronize()
        assert g.device_errors() == 0
        sub_dy = np.concatenate([dy[int(off[e]):int(off[e + 1])] for e in experts])
        ref = oracle.grouped_dgrad("mxfp4", sub_dy, w_small, s_small, sub_off, rows=sub_rows)
        assert_within_tolerance(bf16_to_f64(dx)[rows], ref, f"kimi dgrad {p.name}")
        return
    a = inputs.bf16_normal(inputs.rng(80 + proj), (M, K))
    a_d = to_dev_bf16(a)
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    sub_a = np.concatenate([a[int(off[e]):int(off[e + 1])] for e in experts])
    if mode == "ws":  # small groups native two-term, large groups decode path: the path's own tolerance
        ws = torch.empty(g.mxfp4_workspace_bytes(M, K), dtype=torch.uint8, device="cuda")
        g.grouped_gemm_mxfp4_ws(a_d, w_d, sc_d, y, ws, offsets=off_d)
        torch.cuda.synchronize()
        assert g.device_errors() == 0
        sizes = np.diff(off)[experts]
        assert (sizes <= 96).any() and (sizes > 96).any(), "the sample should hold groups of both paths"
        ref16 = oracle.grouped_gemm_mxfp4(sub_a, w_small, s_small, sub_off, rows=sub_rows)
        assert_within_tolerance(bf16_to_f64(y)[rows], ref16, f"kimi mxfp4 ws {p.name}")
        return
    if mode == "w4a4":
        qa = torch.empty(M, K // 2, dtype=torch.uint8, device="cuda")
        sa = torch.empty(M, K // 32, dtype=torch.uint8, device="cuda")
        g.quantize_mxfp4_act(a_d, qa, sa)
        g.grouped_gemm_w4a4(qa, sa, w_d, sc_d, y, offsets=off_d)
        ref = oracle.grouped_gemm_w4a4(*oracle.quant_mxfp4_act(sub_a), w_small, s_small, sub_off, rows=sub_rows)
    elif mode == "w4a8":
        qa = torch.empty(M, K, dtype=torch.uint8, device="cuda")
        sa = torch.empty(M, K // 32, dtype=torch.uint8, device="cuda")
        g.quantize_mxfp8(a_d, qa, sa)
        g.grouped_gemm_w4a8(qa, sa, w_d, sc_d, y, offsets=off_d)
        ref = oracle.grouped_gemm_w4a8(*oracle.quant_mxfp8(sub_a), w_small, s_small, sub_off, rows=sub_rows)
    else:
        hq = torch.empty(M, K, dtype=torch.uint8, device="cuda")
        hs = torch.empty(M, K // 32, dtype=torch.uint8, device="cuda")
        lq, ls = torch.empty_like(hq), torch.empty_like(hs)
        g.quantize_mxfp8_split(a_d, hq, hs, lq, ls)
        g.grouped_gemm_w4a8x2(hq, hs, lq, ls, w_d, sc_d, y, offsets=off_d)
        ref = oracle.grouped_gemm_w4a8x2(*oracle.quant_mxfp8_split(sub_a), w_small, s_small, sub_off, rows=sub_rows)
    torch.cuda.synchronize()
    assert g.device_errors() == 0
    got = bf16_to_f64(y)[rows]
    _own_bound(got, ref, f"kimi {mode} {p.name}")
    if mode == "w4a8x2":  # the two-term form also meets the path's bf16-activation tolerance
        ref16 = oracle.grouped_gemm_mxfp4(sub_a, w_small, s_small, sub_off, rows=sub_rows)
        assert_within_tolerance(got, ref16, f"kimi two-term vs bf16 activations {p.name}")
