"""GPU parity at the pages' workload shapes, in the launch configuration the
bench times: route -> projection 1 -> projection 2 -> combine.

Routing and gathers are compared bit-exactly in full.  GEMM / GEMV outputs
are compared with the oracle on sampled rows (first and last row of sampled
groups, the largest and smallest groups, the first and last non-empty group,
plus random rows); decode shapes, where every row is cheap, are compared in
full.  The combine is compared in full against the oracle's combine of the
GPU's own projection-2 output.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_grouped_moe_b200 import inputs
from tests._util import (assert_within_tolerance, bf16_bits, bf16_to_f64, offsets_from_counts,
                         set_oracle_threads, to_dev, to_dev_bf16)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    assert torch.cuda.is_available()
    from bit_grouped_moe_b200 import gnf4
    set_oracle_threads()
    gnf4.device_errors(clear=True)
    return gnf4


def _pick_rows(offsets, n_groups=16, per_group=3, seed=0):
    rng = np.random.default_rng(seed)
    E = offsets.shape[0] - 1
    sizes = np.diff(offsets)
    ne = np.nonzero(sizes)[0]
    pick = {int(ne[0]), int(ne[-1]), int(ne[np.argmax(sizes[ne])]), int(ne[np.argmin(sizes[ne])])}
    rest = [e for e in ne if e not in pick]
    if rest:
        pick.update(int(e) for e in rng.choice(rest, size=min(len(rest), n_groups - len(pick)), replace=False))
    rows = set()
    for e in sorted(pick):
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        rows.update([lo, hi - 1])
        rows.update(int(r) for r in rng.integers(lo, hi, size=min(per_group, hi - lo)))
    return np.array(sorted(rows), np.int64)


def _stack(fmt, E, N, K, seed):
    """(host w, host scales, device w, device scales).  NF4 stacks are N(0,0.02)
    weights quantised by the oracle; MXFP4 stacks are drawn directly."""
    rng = inputs.rng(seed)
    if fmt == "nf4":
        w, sc = oracle.quant_nf4(inputs.normal_weights(rng, (E, N, K)))
    else:
        w, sc = inputs.mxfp4_random(rng, E, N, K)
    return w, sc, to_dev(w), to_dev(sc)


def _proj(g, fmt, decode, a_d, w_d, sc_d, off_d, M, N):
    y = torch.full((M, N), -5.0, dtype=torch.bfloat16, device="cuda")
    fn = {("nf4", True): g.grouped_gemv_nf4, ("nf4", False): g.grouped_gemm_nf4,
          ("mxfp4", True): g.grouped_gemv_mxfp4, ("mxfp4", False): g.grouped_gemm_mxfp4}[(fmt, decode)]
    fn(a_d, w_d, sc_d, y, offsets=off_d)
    return y


def _check_proj(fmt, y, a_bits, w, sc, offsets, rows, what):
    fn = oracle.grouped_gemm_nf4 if fmt == "nf4" else oracle.grouped_gemm_mxfp4
    ref = fn(a_bits, w, sc, offsets, rows=rows)
    got = bf16_to_f64(y)[rows]
    return assert_within_tolerance(got, ref, what)


WL = ["tiny-nf4", "olmoe-decode-t1", "olmoe-decode-t8", "qwen3-30b-prefill", "gptoss-t1", "gptoss-t64",
      "gptoss-t512"]


@pytest.mark.parametrize("name", WL)
def test_workload_path(g, name):
    wl = inputs.WORKLOADS[name]
    rng = inputs.rng(7)
    T, k, E = wl.T, wl.k, wl.E
    M = T * k
    ids, wts = inputs.routing_for(wl, rng)
    K1 = wl.projections[0].K
    x = inputs.bf16_normal(rng, (T, K1))
    # route
    off = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    s2f = torch.empty(M, dtype=torch.int32, device="cuda")
    f2s = torch.empty(M, dtype=torch.int32, device="cuda")
    xs = torch.empty(M, K1, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(g.route_workspace_bytes(T, k, E), 16), dtype=torch.uint8, device="cuda")
    g.route_permute(to_dev(ids), to_dev_bf16(x), E, off, s2f, f2s, xs, ws)
    o_off, o_s2f, o_f2s, _ = oracle.route(ids, E)
    torch.cuda.synchronize()
    assert np.array_equal(off.cpu().numpy(), o_off)
    assert np.array_equal(s2f.cpu().numpy(), o_s2f) and np.array_equal(f2s.cpu().numpy(), o_f2s)
    xs_bits = bf16_bits(xs)
    assert np.array_equal(xs_bits, oracle.gather(x, k, o_s2f, int(o_off[E])))
    decode = T <= 8
    full = decode or M <= 64
    rows = np.arange(M, dtype=np.int64) if full else _pick_rows(o_off, seed=T)
    # projection 1 on the gathered rows
    p1 = wl.projections[0]
    w1, s1, w1d, s1d = _stack(wl.fmt, E, p1.N, p1.K, seed=11)
    y1 = _proj(g, wl.fmt, decode, xs, w1d, s1d, off, M, p1.N)
    torch.cuda.synchronize()
    _check_proj(wl.fmt, y1, xs_bits, w1, s1, o_off, rows, f"{name} {p1.name}")
    if decode:  # the tiled GEMM must agree on decode shapes too
        y1t = _proj(g, wl.fmt, False, xs, w1d, s1d, off, M, p1.N)
        torch.cuda.synchronize()
        _check_proj(wl.fmt, y1t, xs_bits, w1, s1, o_off, rows, f"{name} {p1.name} tiled")
    del w1d, s1d
    out_proj = y1
    if len(wl.projections) > 1:
        # projection 2 on a synthetic [M, K2] input (the activation between
        # the two projections is not part of the path)
        p2 = wl.projections[1]
        h = inputs.bf16_normal(inputs.rng(13), (M, p2.K))
        w2, s2, w2d, s2d = _stack(wl.fmt, E, p2.N, p2.K, seed=12)
        out_proj = _proj(g, wl.fmt, decode, to_dev_bf16(h), w2d, s2d, off, M, p2.N)
        torch.cuda.synchronize()
        _check_proj(wl.fmt, out_proj, h, w2, s2, o_off, rows, f"{name} {p2.name}")
        del w2d, s2d
    # combine of the last projection
    Nc = out_proj.shape[1]
    out = torch.empty(T, Nc, dtype=torch.bfloat16, device="cuda")
    g.combine(out_proj, f2s, to_dev(wts), out)
    torch.cuda.synchronize()
    assert_within_tolerance(bf16_to_f64(out), oracle.combine(bf16_bits(out_proj), o_f2s, wts), f"{name} combine")
    assert g.device_errors() == 0


def _device_stack(fmt, E, N, K, seed):
    w = inputs.device_random_bytes(seed, (E, N, K // 2))
    if fmt == "nf4":
        sc = inputs.device_absmax(seed + 1, (E, N, K // 64))
    else:
        sc = inputs.device_random_bytes(seed + 1, (E, N, K // 32), lo=118, hi=131)
    return w, sc


@pytest.mark.parametrize("proj", [0, 1])
def test_kimi_prefill_sampled(g, proj):
    """Kimi-class MXFP4 prefill (E=384, T=4096, top-8): expert stacks drawn on
    the device (up to 5.6 GB); the oracle decodes only the sampled experts."""
    wl = inputs.WORKLOADS["kimi-prefill"]
    rng = inputs.rng(17)
    T, k, E = wl.T, wl.k, wl.E
    M = T * k
    ids, _ = inputs.routing_for(wl, rng)
    o_off, _, _, _ = oracle.route(ids, E)
    assert (np.diff(o_off) == 0).any(), "the skewed routing should leave empty experts"
    p = wl.projections[proj]
    a = inputs.bf16_normal(rng, (M, p.K))
    w_d, sc_d = _device_stack("mxfp4", E, p.N, p.K, seed=20 + proj)
    y = _proj(g, "mxfp4", False, to_dev_bf16(a), w_d, sc_d, to_dev(o_off), M, p.N)
    torch.cuda.synchronize()
    rows = _pick_rows(o_off, n_groups=12, per_group=2, seed=proj)
    experts = sorted({int(np.searchsorted(o_off, r, side="right") - 1) for r in rows})
    # compact the sampled experts into a small stack for the oracle
    w_small = w_d[experts].cpu().numpy()
    s_small = sc_d[experts].cpu().numpy()
    counts = np.diff(o_off)[experts]
    sub_off = offsets_from_counts(counts)
    # rows of the sampled experts, in compact numbering
    row_map = {}
    for i, e in enumerate(experts):
        for r in range(int(o_off[e]), int(o_off[e + 1])):
            row_map[r] = int(sub_off[i]) + (r - int(o_off[e]))
    sub_a = np.concatenate([a[int(o_off[e]):int(o_off[e + 1])] for e in experts])
    sub_rows = np.array([row_map[int(r)] for r in rows], np.int64)
    ref = oracle.grouped_gemm_mxfp4(sub_a, w_small, s_small, sub_off, rows=sub_rows)
    assert_within_tolerance(bf16_to_f64(y)[rows], ref, f"kimi {p.name}")
    assert g.device_errors() == 0


@pytest.mark.parametrize("fmt,E,N,K", [("mxfp4", 384, 4096, 7168), ("nf4", 160, 4096, 7168)])
def test_expert_offset_boundary(g, fmt, E, N, K):
    """Rows only in the first and the LAST expert of a stack larger than
    2 GiB: the last expert's bytes start beyond 2^31 (grouped-nf4-gemm status
    page: the int32 offset overflow issue and its boundary test)."""
    assert E * N * (K // 2) > 2 ** 31
    counts = np.zeros(E, np.int32)
    counts[0], counts[E - 1] = 3, 5
    offsets = offsets_from_counts(counts)
    M = int(offsets[-1])
    w_d, sc_d = _device_stack(fmt, E, N, K, seed=30)
    a = inputs.bf16_normal(inputs.rng(31), (M, K))
    sel = [0, E - 1]
    w_small, s_small = w_d[sel].cpu().numpy(), sc_d[sel].cpu().numpy()
    sub_off = offsets_from_counts(counts[sel])
    fn = oracle.grouped_gemm_nf4 if fmt == "nf4" else oracle.grouped_gemm_mxfp4
    ref = fn(a, w_small, s_small, sub_off)
    for decode in (False, True):
        y = _proj(g, fmt, decode, to_dev_bf16(a), w_d, sc_d, to_dev(offsets), M, N)
        torch.cuda.synchronize()
        assert_within_tolerance(bf16_to_f64(y), ref, f"{fmt} boundary decode={decode}")
    assert g.device_errors() == 0
