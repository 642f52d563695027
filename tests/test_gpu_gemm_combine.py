"""GPU checks of the grouped GEMM with the top-k combine after each work unit
(gnf4_grouped_gemm_{nf4,mxfp4}_combine; grouped-nf4-gemm releases, v0.2.5
"arena -> kernel": gate -> GLU -> down, then the weighted unsort).

The fused call must give, bit for bit, what gnf4_grouped_gemm_* followed by
gnf4_combine gives (the same fp32 fmaf sequence, pairs in slot order), and
its output is checked against oracle.combine of the GEMM rows (tolerance
1e-2 * max|ref| + 2^-7 * |ref|).  Counters must be left zero.  Sizes: a
ragged case with dropped pairs and a token without any pair, and the second
projection of the Qwen3-shaped and Kimi-class prefill workloads.
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


def _route(g, ids, E):
    T, k = ids.shape
    M = T * k
    d = {"off": torch.empty(E + 1, dtype=torch.int32, device="cuda"),
         "s2f": torch.empty(M, dtype=torch.int32, device="cuda"),
         "f2s": torch.empty(M, dtype=torch.int32, device="cuda")}
    x = torch.zeros(T, 8, dtype=torch.bfloat16, device="cuda")  # only the permutation is used here
    xs = torch.empty(M, 8, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(g.route_workspace_bytes(T, k, E), 16), dtype=torch.uint8, device="cuda")
    g.route_permute(to_dev(ids), x, E, d["off"], d["s2f"], d["f2s"], xs, ws)
    return d


def _stack(fmt, E, N, K, seed, host):
    if host:
        rng = inputs.rng(seed)
        if fmt == "nf4":
            w, sc = oracle.quant_nf4(inputs.normal_weights(rng, (E, N, K)))
        else:
            w, sc = inputs.mxfp4_random(rng, E, N, K)
        return to_dev(w), to_dev(sc)
    w = inputs.device_random_bytes(seed, (E, N, K // 2))
    if fmt == "nf4":
        return w, inputs.device_absmax(seed + 1, (E, N, K // 64))
    return w, inputs.device_random_bytes(seed + 1, (E, N, K // 32), lo=118, hi=131)


def _run(g, fmt, ids, wts, E, N, K, seed, host_stack=True):
    T, k = ids.shape
    M = T * k
    d = _route(g, ids, E)
    w, sc = _stack(fmt, E, N, K, seed, host_stack)
    gen = torch.Generator(device="cuda").manual_seed(seed + 7)
    a = torch.randn(M, K, device="cuda", generator=gen).to(torch.bfloat16)
    wts_d = to_dev(wts)
    cnt = torch.zeros(g.combine_counters_bytes(T, N) // 4, dtype=torch.int32, device="cuda")
    fused = g.grouped_gemm_nf4_combine if fmt == "nf4" else g.grouped_gemm_mxfp4_combine
    plain = g.grouped_gemm_nf4 if fmt == "nf4" else g.grouped_gemm_mxfp4
    yf = torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda")
    of = torch.full((T, N), 5.0, dtype=torch.bfloat16, device="cuda")
    fused(a, w, sc, yf, d["s2f"], d["f2s"], wts_d, of, cnt, offsets=d["off"])
    yu = torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda")
    ou = torch.empty((T, N), dtype=torch.bfloat16, device="cuda")
    plain(a, w, sc, yu, offsets=d["off"])
    g.combine(yu, d["f2s"], wts_d, ou)
    torch.cuda.synchronize()
    assert g.device_errors() == 0
    nv = int(d["off"][-1].item())
    assert torch.equal(yf[:nv].view(torch.int16), yu[:nv].view(torch.int16)), "the GEMM rows changed"
    assert torch.equal(of.view(torch.int16), ou.view(torch.int16)), "fused combine differs from GEMM + combine"
    assert int(cnt.abs().sum().item()) == 0, "counters not left at zero"
    out_ref = oracle.combine(bf16_bits(yf), d["f2s"].cpu().numpy(), wts)
    assert_within_tolerance(bf16_to_f64(of), out_ref, f"{fmt} fused combine")
    return of, d, cnt, (a, w, sc, wts_d, fused)


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_gemm_combine_ragged_with_dropped_pairs(g, fmt):
    """~170 rows per expert (chunks of 256 and ragged 32-row tails), N = 392
    (a last column tile of 8), a dropped pair and a token with none left."""
    T, k, E, N, K = 512, 4, 12, 392, 256
    ids, wts = inputs.route_topk(inputs.rng(1700), T, k, E)
    ids[3, 1] = E + 2
    ids[10, :] = E + 9
    of, d, cnt, (a, w, sc, wts_d, fused) = _run(g, fmt, ids, wts, E, N, K, seed=1710)
    assert torch.all(of[10] == 0), "a token without a valid pair must get a zero row"
    # a second call on the same counters and the counts form agree
    of2 = torch.empty_like(of)
    y2 = torch.empty(T * k, N, dtype=torch.bfloat16, device="cuda")
    fused(a, w, sc, y2, d["s2f"], d["f2s"], wts_d, of2, cnt, counts=(d["off"][1:] - d["off"][:-1]).contiguous())
    torch.cuda.synchronize()
    assert torch.equal(of.view(torch.int16), of2.view(torch.int16))
    assert int(cnt.abs().sum().item()) == 0


@pytest.mark.parametrize("name,fmt", [("qwen3-30b-prefill", "nf4"), ("kimi-prefill", "mxfp4")])
def test_gemm_combine_second_projection_full_size(g, name, fmt):
    """The down projection of the Qwen3-shaped NF4 (T=2048, top-8, K=768,
    N=2048) and the Kimi-class MXFP4 (T=4096, top-8, K=2048, N=7168)
    workloads with their Zipf-skewed routing; stacks drawn on the device."""
    wl = inputs.WORKLOADS[name]
    assert wl.fmt == fmt
    ids, wts = inputs.routing_for(wl, inputs.rng(1800))
    p = wl.projections[-1]
    _run(g, fmt, ids, wts, wl.E, p.N, p.K, seed=1810, host_stack=False)


def test_gemm_combine_with_no_routed_rows(g):
    """Every pair dropped (M rows exist but offsets[E] = 0): out is zero."""
    T, k, E, N, K = 4, 2, 8, 128, 128
    ids = np.full((T, k), E + 1, np.int32)
    wts = np.full((T, k), 0.5, np.float32)
    d = _route(g, ids, E)
    w, sc = _stack("nf4", E, N, K, 1900, True)
    a = torch.zeros(T * k, K, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(T * k, N, dtype=torch.bfloat16, device="cuda")
    out = torch.full((T, N), 5.0, dtype=torch.bfloat16, device="cuda")
    cnt = torch.zeros(g.combine_counters_bytes(T, N) // 4, dtype=torch.int32, device="cuda")
    g.grouped_gemm_nf4_combine(a, w, sc, y, d["s2f"], d["f2s"], to_dev(wts), out, cnt, offsets=d["off"])
    torch.cuda.synchronize()
    assert g.device_errors() == 0
    assert torch.all(out == 0)
