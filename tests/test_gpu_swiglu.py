"""GPU parity of the fused gate_up projection + SwiGLU calls against the oracle
(plain grouped GEMM over the [E, 2I, K] stack, then silu(gate) * up, fp64).

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


def _fn(g, fmt, kind):
    return {("nf4", "gemm"): g.grouped_gemm_nf4_swiglu, ("mxfp4", "gemm"): g.grouped_gemm_mxfp4_swiglu,
            ("nf4", "gemv"): g.grouped_gemv_nf4_swiglu, ("mxfp4", "gemv"): g.grouped_gemv_mxfp4_swiglu}[(fmt, kind)]


def _run(g, fmt, kind, counts, I, K, seed, use_counts=False):
    E = len(counts)
    offsets = offsets_from_counts(counts)
    M = int(offsets[-1]) + 3  # rows past offsets[E] must stay untouched
    w, sc = _stack(fmt, E, 2 * I, K, seed)
    a = inputs.bf16_normal(inputs.rng(seed + 1), (M, K))
    h = torch.full((M, I), 7.0, dtype=torch.bfloat16, device="cuda")
    kw = {"counts": to_dev(np.array(counts, np.int32))} if use_counts else {"offsets": to_dev(offsets)}
    _fn(g, fmt, kind)(to_dev_bf16(a), to_dev(w), to_dev(sc), h, **kw)
    torch.cuda.synchronize()
    assert g.device_errors() == 0
    nv = int(offsets[-1])
    ref = oracle.grouped_gemm_swiglu(fmt, a, w, sc, offsets)
    got = bf16_to_f64(h)
    assert_within_tolerance(got[:nv], ref, f"{kind} swiglu {fmt} I={I} K={K}")
    assert np.all(got[nv:] == 7.0), "rows past offsets[E] were written"
    return h


GEMM_GROUPS = [0, 1, 15, 16, 17, 31, 33, 64, 65, 0, 127, 128, 129, 300, 2]


@pytest.mark.parametrize("fmt,I,K", [("nf4", 192, 448), ("mxfp4", 192, 416), ("mxfp4", 128, 2880), ("nf4", 64, 2048)])
def test_gemm_swiglu_ragged_parity(g, fmt, I, K):
    _run(g, fmt, "gemm", GEMM_GROUPS, I, K, seed=500 + K)


@pytest.mark.parametrize("fmt,I,K", [("nf4", 128, 512), ("mxfp4", 192, 480), ("nf4", 256, 2048), ("mxfp4", 64, 2880)])
def test_gemv_swiglu_parity(g, fmt, I, K):
    _run(g, fmt, "gemv", [1, 0, 2, 3, 4, 5, 6, 7, 8, 0, 1, 8], I, K, seed=600 + K)


@pytest.mark.parametrize("kind", ["gemm", "gemv"])
def test_swiglu_counts_equal_offsets(g, kind):
    counts = [3, 0, 8, 1, 5] if kind == "gemv" else [40, 0, 129, 1, 7]
    h1 = _run(g, "nf4", kind, counts, 128, 256, seed=700)
    h2 = _run(g, "nf4", kind, counts, 128, 256, seed=700, use_counts=True)
    assert torch.equal(h1.view(torch.int16), h2.view(torch.int16))


def test_gemv_and_gemm_swiglu_agree_on_decode_groups(g):
    """Both fused forms compute the same values (within the rounding of bf16 h)."""
    counts = [2, 0, 1, 8, 3]
    ha = _run(g, "mxfp4", "gemm", counts, 128, 512, seed=710)
    hb = _run(g, "mxfp4", "gemv", counts, 128, 512, seed=710)
    nv = sum(counts)
    a, b = bf16_to_f64(ha)[:nv], bf16_to_f64(hb)[:nv]
    assert np.max(np.abs(a - b)) <= 2.0 ** -6 * max(1.0, float(np.abs(a).max()))


def test_swiglu_width_must_be_a_multiple_of_64(g):
    w = torch.zeros((1, 2 * 96, 64), dtype=torch.uint8, device="cuda")
    sc = torch.ones((1, 2 * 96, 2), dtype=torch.float32, device="cuda")
    a = torch.zeros((1, 128), dtype=torch.bfloat16, device="cuda")
    h = torch.zeros((1, 96), dtype=torch.bfloat16, device="cuda")
    off = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    with pytest.raises(g.Gnf4Error) as ei:
        g.grouped_gemm_nf4_swiglu(a, w, sc, h, offsets=off)
    assert ei.value.status == g.ERR_UNSUPPORTED_SHAPE
