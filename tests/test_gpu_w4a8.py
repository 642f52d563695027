"""GPU parity of the native W4A8 mode (MXFP8 activations x MXFP4 weights on
block-scaled tcgen05 MMAs) against the oracle.

* gnf4_quantize_mxfp8 is byte work: codes and scales must equal the oracle's
  bit for bit.
* gnf4_grouped_gemm_w4a8 sees exactly the oracle's operands (every product of
  an e4m3 and an e2m1 value with power-of-two scales is exact), so it differs
  from the fp64 oracle only by fp32 accumulation and the final bf16 rounding:
      |gpu - oracle| <= 2^-8 |oracle| + 2^-12 max|oracle|
  (bf16 output: 2^-9 relative; fp32 sums over K <= 2880: far below 2^-12 of
  the largest output).
* Against the bf16-activation oracle the mode carries the e4m3 quantisation
  error of the activations; the stated looser bound is an rms relative error
  below 4% of the output.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_grouped_moe_b200 import inputs
from tests._util import bf16_to_f64, offsets_from_counts, set_oracle_threads, to_dev, to_dev_bf16

pytestmark = pytest.mark.gpu

W4A8_REL = 2.0 ** -8
W4A8_ABS_OF_MAX = 2.0 ** -12


@pytest.fixture(scope="module")
def g():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_grouped_moe_b200 import gnf4
    set_oracle_threads()
    gnf4.device_errors(clear=True)
    return gnf4


def _bits(x: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(x, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _activations(seed, M, K):
    """bf16 rows with a different power-of-two level per 32-block, plus the
    special cases: an all-zero block, bf16 subnormals, negative zeros, exact
    e4m3 ties and values that saturate."""
    rng = inputs.rng(seed)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x *= np.exp2(rng.integers(-24, 24, size=(M, K // 32, 1))).repeat(32, axis=2).reshape(M, K).astype(np.float32)
    if M > 3 and K >= 64:
        x[1, 32:64] = 0.0
        x[2, :32] = np.float32(2.0 ** -130) * rng.integers(-3, 4, size=32)  # bf16 subnormals only
        x[3, :32] = -0.0
        x[3, 0] = 1.0
        x[3, 1] = 1.9375 * 2.0 ** -8  # tie between two e4m3 values after scaling
        x[3, 2] = -3.814697265625e-06  # rounds to negative zero
        x[0, :32] = 1.9375  # the block's amax scales to 496: saturates at 448
    return _bits(x)


def _check_quant(g, bits):
    M, K = bits.shape
    codes = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    scales = torch.empty((M, K // 32), dtype=torch.uint8, device="cuda")
    g.quantize_mxfp8(to_dev_bf16(bits), codes, scales)
    torch.cuda.synchronize()
    rc, rs = oracle.quant_mxfp8(bits)
    gs = scales.cpu().numpy()
    gc = codes.cpu().numpy()
    assert np.array_equal(gs, rs), f"scales differ at {np.argwhere(gs != rs)[:5].tolist()}"
    bad = np.argwhere(gc != rc)
    assert bad.size == 0, f"{len(bad)} codes differ, first {[(tuple(i), int(gc[tuple(i)]), int(rc[tuple(i)])) for i in bad[:5]]}"
    return codes, scales


@pytest.mark.parametrize("M,K", [(37, 2880), (128, 2048), (1, 32), (300, 416), (5, 64)])
def test_quantize_mxfp8_is_bit_exact(g, M, K):
    _check_quant(g, _activations(900 + K + M, M, K))


def _run(g, counts, N, K, seed, use_counts=False):
    E = len(counts)
    offsets = offsets_from_counts(counts)
    nv = int(offsets[-1])
    M = nv + 3  # rows past offsets[E] must stay untouched
    w, sw = inputs.mxfp4_random(inputs.rng(seed), E, N, K)
    bits = _activations(seed + 1, M, K)
    codes, scales = _check_quant(g, bits)
    y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    kw = {"counts": to_dev(np.array(counts, np.int32))} if use_counts else {"offsets": to_dev(offsets)}
    g.grouped_gemm_w4a8(codes, scales, to_dev(w), to_dev(sw), y, **kw)
    torch.cuda.synchronize()
    assert g.device_errors() == 0
    rc, rs = oracle.quant_mxfp8(bits)
    ref = oracle.grouped_gemm_w4a8(rc, rs, w, sw, offsets)
    got = bf16_to_f64(y)
    if nv:
        amax = float(np.abs(ref).max())
        bound = W4A8_REL * np.abs(ref) + W4A8_ABS_OF_MAX * amax
        err = np.abs(got[:nv] - ref)
        bad = np.argwhere(~(err <= bound))
        assert bad.size == 0, (f"{len(bad)} outputs out of tolerance (max|ref| {amax:.4g}), first "
                               + ", ".join(f"{tuple(i)} gpu={got[tuple(i)]:.6g} ref={ref[tuple(i)]:.6g}"
                                           for i in bad[:5]))
    assert np.all(got[nv:] == 7.0), "rows past offsets[E] were written"
    return y, (w, sw, bits, offsets)


GROUPS = [0, 1, 15, 16, 17, 31, 33, 64, 65, 0, 127, 128, 129, 300, 2]


@pytest.mark.parametrize("N,K", [(128, 128), (136, 192), (256, 2880), (128, 2048), (384, 448)])
def test_w4a8_gemm_ragged_parity(g, N, K):
    _run(g, GROUPS, N, K, seed=1000 + K + N)


def test_w4a8_counts_equal_offsets(g):
    counts = [40, 0, 129, 1, 7]
    y1, _ = _run(g, counts, 128, 256, seed=1100)
    y2, _ = _run(g, counts, 128, 256, seed=1100, use_counts=True)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_w4a8_tracks_the_bf16_activation_result(g):
    """The stated looser bound against the bf16-activation MXFP4 oracle."""
    counts = [3, 60, 0, 130, 9]
    y, (w, sw, bits, offsets) = _run(g, counts, 256, 2880, seed=1200)
    nv = int(offsets[-1])
    ref16 = oracle.grouped_gemm_mxfp4(bits, w, sw, offsets)
    got = bf16_to_f64(y)[:nv]
    rel = np.linalg.norm(got - ref16) / np.linalg.norm(ref16)
    assert rel < 0.04, rel


@pytest.mark.parametrize("K", [96, 2848, 64])
def test_w4a8_refuses_k_that_is_not_a_multiple_of_64(g, K):
    w = torch.zeros((1, 128, K // 2), dtype=torch.uint8, device="cuda")
    sw = torch.full((1, 128, K // 32), 127, dtype=torch.uint8, device="cuda")
    codes = torch.zeros((4, K), dtype=torch.uint8, device="cuda")
    sa = torch.full((4, K // 32), 127, dtype=torch.uint8, device="cuda")
    y = torch.zeros((4, 128), dtype=torch.bfloat16, device="cuda")
    off = torch.tensor([0, 4], dtype=torch.int32, device="cuda")
    with pytest.raises(g.Gnf4Error) as ei:
        g.grouped_gemm_w4a8(codes, sa, w, sw, y, offsets=off)
    assert ei.value.status == g.ERR_UNSUPPORTED_SHAPE


# ---------------------------------------------------------------- two-term split (hi + lo)


def _check_split(g, bits):
    M, K = bits.shape
    t = [torch.empty((M, K), dtype=torch.uint8, device="cuda"), torch.empty((M, K // 32), dtype=torch.uint8, device="cuda"),
         torch.empty((M, K), dtype=torch.uint8, device="cuda"), torch.empty((M, K // 32), dtype=torch.uint8, device="cuda")]
    g.quantize_mxfp8_split(to_dev_bf16(bits), *t)
    torch.cuda.synchronize()
    ref = oracle.quant_mxfp8_split(bits)
    for name, got, r in zip(("hi codes", "hi scales", "lo codes", "lo scales"), t, ref):
        got = got.cpu().numpy()
        bad = np.argwhere(got != r)
        assert bad.size == 0, f"{name}: {len(bad)} differ, first {[(tuple(i), int(got[tuple(i)]), int(r[tuple(i)])) for i in bad[:5]]}"
    return t


@pytest.mark.parametrize("M,K", [(37, 2880), (128, 2048), (1, 32), (300, 416)])
def test_quantize_mxfp8_split_is_bit_exact(g, M, K):
    _check_split(g, _activations(950 + K + M, M, K))


def _run_split(g, counts, N, K, seed, use_counts=False):
    E = len(counts)
    offsets = offsets_from_counts(counts)
    nv = int(offsets[-1])
    M = nv + 3
    w, sw = inputs.mxfp4_random(inputs.rng(seed), E, N, K)
    bits = _activations(seed + 1, M, K)
    hc, hs, lc, ls = _check_split(g, bits)
    y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    kw = {"counts": to_dev(np.array(counts, np.int32))} if use_counts else {"offsets": to_dev(offsets)}
    g.grouped_gemm_w4a8x2(hc, hs, lc, ls, to_dev(w), to_dev(sw), y, **kw)
    torch.cuda.synchronize()
    assert g.device_errors() == 0
    got = bf16_to_f64(y)
    assert np.all(got[nv:] == 7.0), "rows past offsets[E] were written"
    return got[:nv], (w, sw, bits, offsets)


@pytest.mark.parametrize("N,K", [(128, 128), (136, 192), (256, 2880), (384, 448)])
def test_w4a8x2_gemm_ragged_parity(g, N, K):
    got, (w, sw, bits, offsets) = _run_split(g, GROUPS, N, K, seed=1600 + K + N)
    ref = oracle.grouped_gemm_w4a8x2(*oracle.quant_mxfp8_split(bits), w, sw, offsets)
    amax = float(np.abs(ref).max())
    err = np.abs(got - ref)
    bad = np.argwhere(~(err <= W4A8_REL * np.abs(ref) + W4A8_ABS_OF_MAX * amax))
    assert bad.size == 0, f"{len(bad)} outputs out of tolerance, first {[tuple(i) for i in bad[:5]]}"


@pytest.mark.parametrize("N,K", [(256, 2880), (128, 2048)])
def test_w4a8x2_meets_the_bf16_activation_tolerance(g, N, K):
    """The two-term native path holds the standard tolerance of the grouped
    GEMM against the bf16-activation oracle (1e-2 max|ref| + 2^-7 |ref|)."""
    counts = [3, 60, 0, 130, 9, 1, 33]
    got, (w, sw, bits, offsets) = _run_split(g, counts, N, K, seed=1700 + K)
    from tests._util import assert_within_tolerance
    assert_within_tolerance(got, oracle.grouped_gemm_mxfp4(bits, w, sw, offsets), "w4a8x2 vs bf16 activations")


def test_w4a8x2_counts_equal_offsets(g):
    counts = [40, 0, 129, 1, 7, 96, 97]
    a, _ = _run_split(g, counts, 128, 256, seed=1800)
    b, _ = _run_split(g, counts, 128, 256, seed=1800, use_counts=True)
    assert np.array_equal(a, b)


# ---------------------------------------------------------------- W4A4 (MXFP4 activations, kind::mxf4)


def _check_quant4(g, bits):
    M, K = bits.shape
    blocks = torch.empty((M, K // 2), dtype=torch.uint8, device="cuda")
    scales = torch.empty((M, K // 32), dtype=torch.uint8, device="cuda")
    g.quantize_mxfp4_act(to_dev_bf16(bits), blocks, scales)
    torch.cuda.synchronize()
    rb, rs = oracle.quant_mxfp4_act(bits)
    gb, gs = blocks.cpu().numpy(), scales.cpu().numpy()
    assert np.array_equal(gs, rs), f"scales differ at {np.argwhere(gs != rs)[:5].tolist()}"
    bad = np.argwhere(gb != rb)
    assert bad.size == 0, f"{len(bad)} bytes differ, first {[(tuple(i), int(gb[tuple(i)]), int(rb[tuple(i)])) for i in bad[:5]]}"
    return blocks, scales


@pytest.mark.parametrize("M,K", [(37, 2880), (128, 2048), (1, 32), (300, 416)])
def test_quantize_mxfp4_act_is_bit_exact(g, M, K):
    _check_quant4(g, _activations(2000 + K + M, M, K))


def _run4(g, counts, N, K, seed, use_counts=False):
    E = len(counts)
    offsets = offsets_from_counts(counts)
    nv = int(offsets[-1])
    M = nv + 3
    w, sw = inputs.mxfp4_random(inputs.rng(seed), E, N, K)
    bits = _activations(seed + 1, M, K)
    ab, as_ = _check_quant4(g, bits)
    y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
    kw = {"counts": to_dev(np.array(counts, np.int32))} if use_counts else {"offsets": to_dev(offsets)}
    g.grouped_gemm_w4a4(ab, as_, to_dev(w), to_dev(sw), y, **kw)
    torch.cuda.synchronize()
    assert g.device_errors() == 0
    got = bf16_to_f64(y)
    assert np.all(got[nv:] == 7.0), "rows past offsets[E] were written"
    return got[:nv], (w, sw, bits, offsets)


@pytest.mark.parametrize("N,K", [(128, 256), (136, 320), (256, 2880), (384, 512)])
def test_w4a4_gemm_ragged_parity(g, N, K):
    got, (w, sw, bits, offsets) = _run4(g, GROUPS, N, K, seed=2100 + K + N)
    ref = oracle.grouped_gemm_w4a4(*oracle.quant_mxfp4_act(bits), w, sw, offsets)
    amax = float(np.abs(ref).max())
    err = np.abs(got - ref)
    bad = np.argwhere(~(err <= W4A8_REL * np.abs(ref) + W4A8_ABS_OF_MAX * amax))
    assert bad.size == 0, (f"{len(bad)} outputs out of tolerance (max|ref| {amax:.4g}), first "
                           + ", ".join(f"{tuple(i)} gpu={got[tuple(i)]:.6g} ref={ref[tuple(i)]:.6g}" for i in bad[:5]))


def test_w4a4_counts_equal_offsets(g):
    counts = [40, 0, 129, 1, 7]
    a, _ = _run4(g, counts, 128, 512, seed=2200)
    b, _ = _run4(g, counts, 128, 512, seed=2200, use_counts=True)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("K", [128, 192, 288])
def test_w4a4_refuses_short_or_unaligned_k(g, K):
    w = torch.zeros((1, 128, K // 2), dtype=torch.uint8, device="cuda")
    sw = torch.full((1, 128, K // 32), 127, dtype=torch.uint8, device="cuda")
    ab = torch.zeros((4, K // 2), dtype=torch.uint8, device="cuda")
    sa = torch.full((4, K // 32), 127, dtype=torch.uint8, device="cuda")
    y = torch.zeros((4, 128), dtype=torch.bfloat16, device="cuda")
    off = torch.tensor([0, 4], dtype=torch.int32, device="cuda")
    with pytest.raises(g.Gnf4Error) as ei:
        g.grouped_gemm_w4a4(ab, sa, w, sw, y, offsets=off)
    assert ei.value.status == g.ERR_UNSUPPORTED_SHAPE
