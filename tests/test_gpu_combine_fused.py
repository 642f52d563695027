"""GPU checks of the decode GEMV with the top-k combine in its epilogue.

The fused call must give exactly (bit for bit) what the separate GEMV and
combine give -- the combine runs the same fp32 fmaf sequence -- and both are
checked against the oracle (tolerance 1e-2 * max|ref| + 2^-7 * |ref|).  The
counters must be left zero, so repeated calls (and graph replays) agree.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_grouped_moe_b200 import inputs
from tests._util import assert_within_tolerance, bf16_bits, bf16_to_f64, set_oracle_threads, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_grouped_moe_b200 import gnf4
    set_oracle_threads()
    gnf4.device_errors(clear=True)
    return gnf4


def _setup(g, fmt, T, k, E, N, K, seed, drop=()):
    rng = inputs.rng(seed)
    ids, wts = inputs.route_topk(rng, T, k, E)
    for (t, j) in drop:
        ids[t, j] = E + 5  # dropped by the routing
    x = inputs.bf16_normal(rng, (T, K))
    if fmt == "nf4":
        w, sc = oracle.quant_nf4(inputs.normal_weights(rng, (E, N, K)))
    else:
        w, sc = inputs.mxfp4_random(rng, E, N, K)
    M = T * k
    d = {"off": torch.empty(E + 1, dtype=torch.int32, device="cuda"),
         "s2f": torch.empty(M, dtype=torch.int32, device="cuda"),
         "f2s": torch.empty(M, dtype=torch.int32, device="cuda"),
         "xs": torch.empty(M, K, dtype=torch.bfloat16, device="cuda")}
    ws = torch.empty(max(g.route_workspace_bytes(T, k, E), 16), dtype=torch.uint8, device="cuda")
    g.route_permute(to_dev(ids), to_dev_bf16(x), E, d["off"], d["s2f"], d["f2s"], d["xs"], ws)
    d.update(w=to_dev(w), sc=to_dev(sc), wts=to_dev(wts), ids=ids, wts_h=wts, w_h=w, sc_h=sc, x=x, M=M, N=N)
    return d


def _fused(g, fmt, d, counters, use_counts=False):
    fn = g.grouped_gemv_nf4_combine if fmt == "nf4" else g.grouped_gemv_mxfp4_combine
    T = d["wts"].shape[0]
    y = torch.full((d["M"], d["N"]), 3.0, dtype=torch.bfloat16, device="cuda")
    out = torch.full((T, d["N"]), 5.0, dtype=torch.bfloat16, device="cuda")
    kw = {"offsets": d["off"]}
    if use_counts:
        kw = {"counts": (d["off"][1:] - d["off"][:-1]).contiguous()}
    fn(d["xs"], d["w"], d["sc"], y, d["s2f"], d["f2s"], d["wts"], out, counters, **kw)
    torch.cuda.synchronize()
    assert g.device_errors() == 0
    return y, out


def _unfused(g, fmt, d):
    fn = g.grouped_gemv_nf4 if fmt == "nf4" else g.grouped_gemv_mxfp4
    T = d["wts"].shape[0]
    y = torch.full((d["M"], d["N"]), 3.0, dtype=torch.bfloat16, device="cuda")
    out = torch.empty((T, d["N"]), dtype=torch.bfloat16, device="cuda")
    fn(d["xs"], d["w"], d["sc"], y, offsets=d["off"])
    g.combine(y, d["f2s"], d["wts"], out)
    torch.cuda.synchronize()
    return y, out


def _counters(g, T, N):
    return torch.zeros(g.combine_counters_bytes(T, N) // 4, dtype=torch.int32, device="cuda")


@pytest.mark.parametrize("fmt,N,K", [("nf4", 2048, 1024), ("mxfp4", 2880, 2880), ("nf4", 136, 256)])
def test_fused_combine_equals_gemv_then_combine(g, fmt, N, K):
    T, k, E = 8, 8, 64 if fmt == "nf4" else 128
    d = _setup(g, fmt, T, k, E, N, K, seed=1300 + N)
    cnt = _counters(g, T, N)
    yf, of = _fused(g, fmt, d, cnt)
    yu, ou = _unfused(g, fmt, d)
    nv = int(d["off"][-1].item())
    assert torch.equal(yf[:nv].view(torch.int16), yu[:nv].view(torch.int16))
    assert torch.equal(of.view(torch.int16), ou.view(torch.int16)), "fused combine differs from the separate one"
    assert int(cnt.abs().sum().item()) == 0, "counters not left at zero"
    off, s2f, f2s, _ = oracle.route(d["ids"], E)
    xs = oracle.gather(d["x"], k, s2f, int(off[E]))
    gem = oracle.grouped_gemm_nf4 if fmt == "nf4" else oracle.grouped_gemm_mxfp4
    y_ref = gem(xs, d["w_h"], d["sc_h"], off)
    assert_within_tolerance(bf16_to_f64(yf)[:nv], y_ref, "fused GEMV rows")
    out_ref = oracle.combine(bf16_bits(yf), f2s, d["wts_h"])
    assert_within_tolerance(bf16_to_f64(of), out_ref, "fused combine")


def test_fused_combine_dropped_pairs_and_empty_tokens(g):
    T, k, E, N, K = 6, 4, 16, 128, 256
    drop = [(1, 2)] + [(4, j) for j in range(k)]  # token 4 loses every pair
    d = _setup(g, "nf4", T, k, E, N, K, seed=1400, drop=drop)
    cnt = _counters(g, T, N)
    yf, of = _fused(g, "nf4", d, cnt)
    yu, ou = _unfused(g, "nf4", d)
    assert torch.equal(of.view(torch.int16), ou.view(torch.int16))
    assert torch.all(of[4] == 0)
    assert int(cnt.abs().sum().item()) == 0


def test_fused_combine_repeats_and_counts_form(g):
    T, k, E, N, K = 8, 8, 64, 1024, 512
    d = _setup(g, "mxfp4", T, k, E, N, K, seed=1500)
    cnt = _counters(g, T, N)
    _, o1 = _fused(g, "mxfp4", d, cnt)
    _, o2 = _fused(g, "mxfp4", d, cnt)
    _, o3 = _fused(g, "mxfp4", d, cnt, use_counts=True)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(o1.view(torch.int16), o3.view(torch.int16))
    assert int(cnt.abs().sum().item()) == 0
