"""GPU parity of the fused router epilogue + routing against the oracle.

Bit-exact: selected ids (the selection is taken in fp32 on both sides),
offsets, permutations, gathered rows.  Weights: |gpu - oracle| <= 2e-6.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_grouped_moe_b200 import inputs
from tests._util import bf16_bits, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_grouped_moe_b200 import gnf4
    gnf4.device_errors(clear=True)
    return gnf4


def _run(g, logits, k, K, bias=None, seed=0):
    T, E = logits.shape
    x = inputs.bf16_normal(inputs.rng(seed), (T, K))
    M = T * k
    dev = "cuda"
    ids = torch.full((T, k), -7, dtype=torch.int32, device=dev)
    wts = torch.full((T, k), -1.0, dtype=torch.float32, device=dev)
    off = torch.empty(E + 1, dtype=torch.int32, device=dev)
    s2f = torch.empty(M, dtype=torch.int32, device=dev)
    f2s = torch.empty(M, dtype=torch.int32, device=dev)
    xs = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(g.route_workspace_bytes(T, k, E), 16), dtype=torch.uint8, device=dev)
    g.route_topk_permute(to_dev(logits), to_dev_bf16(x), k, ids, wts, off, s2f, f2s, xs, ws,
                         bias=None if bias is None else to_dev(bias))
    torch.cuda.synchronize()
    o_ids, o_w = oracle.router_topk(logits, k, bias)
    assert np.array_equal(ids.cpu().numpy(), o_ids)
    np.testing.assert_allclose(wts.cpu().numpy(), o_w, rtol=0, atol=2e-6)
    o_off, o_s2f, o_f2s, _ = oracle.route(o_ids, E)
    assert np.array_equal(off.cpu().numpy(), o_off)
    assert np.array_equal(s2f.cpu().numpy(), o_s2f)
    assert np.array_equal(f2s.cpu().numpy(), o_f2s)
    assert np.array_equal(bf16_bits(xs), oracle.gather(x, k, o_s2f, int(o_off[E])))


@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (8, 64, 8), (32, 384, 8), (3, 4096, 4), (64, 128, 4)])
def test_router_single_launch(g, T, E, k):
    logits = inputs.rng(800 + T).standard_normal((T, E)).astype(np.float32)
    _run(g, logits, k, 256, seed=T)


@pytest.mark.parametrize("T,E,k", [(65, 64, 4), (512, 128, 4), (300, 384, 8), (40, 1000, 32)])
def test_router_multi_launch(g, T, E, k):
    logits = inputs.rng(900 + T).standard_normal((T, E)).astype(np.float32)
    _run(g, logits, k, 128, seed=T)


def test_router_ties_bias_and_nan(g):
    rng = inputs.rng(950)
    T, E, k = 24, 40, 6
    logits = (np.round(rng.standard_normal((T, E)) * 2) / 2).astype(np.float32)  # many ties
    logits[3, [0, 7, 9]] = np.nan
    logits[5, :] = 1.0
    bias = (np.round(rng.standard_normal(E)) / 4).astype(np.float32)
    _run(g, logits, k, 64, bias=bias, seed=5)
    _run(g, np.where(np.isnan(logits), 0.0, logits).astype(np.float32), k, 64, seed=6)


def test_router_zipf_workload_matches_the_input_recipe(g):
    """The Zipf-skewed workloads select by logits + bias: the GPU router picks
    the same experts as the input generator's argsort."""
    rng = inputs.rng(960)
    T, E, k = 200, 128, 8
    logits = rng.standard_normal((T, E), dtype=np.float32)
    rank = rng.permutation(E).astype(np.float32) + 1.0
    bias = (-np.float32(1.1) * np.log(rank)).astype(np.float32)
    _run(g, logits, k, 64, bias=bias, seed=7)
