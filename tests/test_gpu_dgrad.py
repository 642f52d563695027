"""GPU parity of the grouped dgrad (dX = dY . W on the packed stacks) against the oracle.

Tolerance: |gpu - oracle| <= 1e-2 * max|oracle| + 2^-7 * |oracle|.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_grouped_moe_b200 import inputs
from tests._util import assert_within_tolerance, bf16_to_f64, offsets_from_counts, set_oracle_threads, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_grouped_moe_b200 import gnf4
    set_oracle_threads()
    gnf4.device_errors(clear=True)
    return gnf4


def _stack(fmt, E, N, K, seed):
    rng = inputs.rng(seed)
    if fmt == "nf4":
        return oracle.quant_nf4(inputs.normal_weights(rng, (E, N, K)))
    return inputs.mxfp4_random(rng, E, N, K)


def _run(g, fmt, counts, N, K, seed, use_counts=False):
    E = len(counts)
    offsets = offsets_from_counts(counts)
    M = int(offsets[-1]) + 3  # rows past offsets[E] must stay untouched
    w, sc = _stack(fmt, E, N, K, seed)
    dy = inputs.bf16_normal(inputs.rng(seed + 1), (M, N))
    dx = torch.full((M, K), 9.0, dtype=torch.bfloat16, device="cuda")
    fn = g.grouped_dgrad_nf4 if fmt == "nf4" else g.grouped_dgrad_mxfp4
    kw = {"counts": to_dev(np.array(counts, np.int32))} if use_counts else {"offsets": to_dev(offsets)}
    fn(to_dev_bf16(dy), to_dev(w), to_dev(sc), dx, **kw)
    torch.cuda.synchronize()
    assert g.device_errors() == 0
    nv = int(offsets[-1])
    ref = oracle.grouped_dgrad(fmt, dy, w, sc, offsets)
    got = bf16_to_f64(dx)
    assert_within_tolerance(got[:nv], ref, f"dgrad {fmt} N={N} K={K}")
    assert np.all(got[nv:] == 9.0), "rows past offsets[E] were written"
    return dx


GROUPS = [0, 1, 15, 16, 33, 127, 128, 129, 0, 200, 2]


@pytest.mark.parametrize("fmt,N,K", [("nf4", 256, 256), ("mxfp4", 200, 416), ("nf4", 72, 448), ("mxfp4", 136, 96),
                                     ("nf4", 1536, 2048)])
def test_dgrad_ragged_parity(g, fmt, N, K):
    _run(g, fmt, GROUPS, N, K, seed=1000 + N + K)


def test_dgrad_counts_equal_offsets(g):
    counts = [40, 0, 129, 1, 7]
    a = _run(g, "nf4", counts, 128, 256, seed=1100)
    b = _run(g, "nf4", counts, 128, 256, seed=1100, use_counts=True)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_dgrad_is_adjoint_to_the_gpu_forward(g):
    """<dY, GEMM(X)> = <dgrad(dY), X> within the bf16 rounding of both outputs."""
    counts = [3, 17, 0, 40]
    E, N, K = len(counts), 256, 384
    offsets = offsets_from_counts(counts)
    M = int(offsets[-1])
    w, sc = _stack("mxfp4", E, N, K, 1200)
    x = to_dev_bf16(inputs.bf16_normal(inputs.rng(1201), (M, K)))
    dy = to_dev_bf16(inputs.bf16_normal(inputs.rng(1202), (M, N)))
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    dx = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    off = to_dev(offsets)
    g.grouped_gemm_mxfp4(x, to_dev(w), to_dev(sc), y, offsets=off)
    g.grouped_dgrad_mxfp4(dy, to_dev(w), to_dev(sc), dx, offsets=off)
    torch.cuda.synchronize()
    lhs = float((dy.double() * y.double()).sum())
    rhs = float((dx.double() * x.double()).sum())
    scale = float(dy.double().abs().mul(y.double().abs()).sum())
    assert abs(lhs - rhs) <= 2.0 ** -6 * scale
