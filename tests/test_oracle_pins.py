"""Pins for the CPU oracle: checks against what the pages and the mathematics
fix, never against the oracle's own formulas retyped.

Each check is chosen so that a plausible slip in the oracle fails it: a wrong
codebook entry or nibble order (byte examples, quantile construction, pack
identity), a wrong scale (e8m0 closed form), a dropped or misplaced term in
the GEMM (closed forms, one-hot weights, numpy's matmul on E=1, brute force),
a wrong expert index (per-expert power-of-two weights), an unstable or lossy
routing sort (brute force by Python's sorted), and a wrong combine weight or
index (one-hot weights, brute force with math.fsum).
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from bit_grouped_moe_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- formats


def test_nf4_codebook_structure():
    v = oracle.nf4_values().astype(np.float64)
    assert v.shape == (16,)
    assert np.all(np.diff(v) > 0), "codebook must be strictly increasing"
    assert v[0] == -1.0 and v[15] == 1.0
    assert v[7] == 0.0 and np.count_nonzero(v == 0.0) == 1
    assert np.count_nonzero(v < 0) == 7 and np.count_nonzero(v > 0) == 8


def test_nf4_codebook_matches_quantile_construction():
    """Rebuild the NormalFloat table from N(0,1) quantiles (QLoRA's
    construction) with scipy and compare to the stored constants."""
    from scipy.stats import norm

    g = _golden("formats.json")
    off = g["nf4_quantile_offset"]
    pos = norm.ppf(np.linspace(off, 0.5, 9)[:-1])
    neg = -norm.ppf(np.linspace(off, 0.5, 8)[:-1])
    v = np.sort(np.concatenate([pos, [0.0], neg]))
    v = v / np.abs(v).max()
    got = oracle.nf4_values().astype(np.float64)
    assert np.max(np.abs(got - v)) <= g["nf4_quantile_tolerance"]


def test_e2m1_table():
    g = _golden("formats.json")
    t = oracle.e2m1_values()
    mags = np.array(g["e2m1_magnitudes"], np.float32)
    assert np.array_equal(np.abs(t[:8]), mags) and np.all(np.signbit(t[:8]) == False)  # noqa: E712
    assert np.array_equal(np.abs(t[8:]), mags) and np.all(np.signbit(t[8:]))
    assert t[8] == 0.0 and np.signbit(t[8]), "code 8 is negative zero"


def test_e8m0_closed_form():
    for e in range(1, 255):
        assert oracle.e8m0_value(e) == math.ldexp(1.0, e - 127)
    assert oracle.e8m0_value(0) == math.ldexp(1.0, -127) > 0.0  # fp32 subnormal, not flushed
    assert math.isnan(oracle.e8m0_value(255))


def test_byte_examples_pin_nibble_order():
    g = _golden("formats.json")
    for ex in g["nf4_byte_examples"]:
        packed = np.array([[ex["byte"]] * 32], np.uint8)
        absmax = np.array([[ex["absmax"]]], np.float32)
        out = oracle.dequant_nf4(packed, absmax)
        assert out[0, 0] == ex["values"][0] and out[0, 1] == ex["values"][1]
    for ex in g["mxfp4_byte_examples"]:
        blocks = np.array([[ex["byte"]] * 16], np.uint8)
        scales = np.array([[ex["scale"]]], np.uint8)
        out = oracle.dequant_mxfp4(blocks, scales)
        assert out[0, 0] == ex["values"][0] and out[0, 1] == ex["values"][1]


def test_mxfp4_decode_matches_compressed_tensors():
    """Reading C5 (element 2i in the low nibble), C6 (e2m1 code map) and C7
    (e8m0 rule) against an independent library: compressed-tensors' FP4
    unpacking and MX scale decompression, the decode the pages report their
    MXFP4 reference as bit-identical to (grouped-nf4-gemm index.json,
    problems_solved: MXFP4 reference decode vs compressed-tensors).  Every
    byte value, scales over the bf16-exact range of the configs and beyond."""
    helpers = pytest.importorskip("compressed_tensors.compressors.nvfp4.helpers")
    mx = pytest.importorskip("compressed_tensors.compressors.mx_utils")
    import torch

    g = inputs.rng(5)
    rows, K = 24, 512
    blocks = g.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
    blocks[0, :] = np.arange(256, dtype=np.uint8)  # every byte value once
    scales = g.integers(100, 160, size=(rows, K // 32), dtype=np.uint8)
    ours = oracle.dequant_mxfp4(blocks, scales)
    vals = helpers.unpack_fp4_from_uint8(torch.from_numpy(blocks), rows, K, dtype=torch.float32)
    sc = mx.decompress_mx_scale(torch.from_numpy(scales)).to(torch.float32).repeat_interleave(32, dim=1)
    theirs = (vals * sc).numpy()
    # bit patterns, except that the library multiplies a zero by a signed scale
    # to +0 while the oracle keeps the code's sign (code 8 is -0, reading C6)
    assert np.array_equal(ours, theirs)
    nz = theirs != 0
    assert np.array_equal(ours.view(np.uint32)[nz], theirs.view(np.uint32)[nz])


def _codes_from_values(vals, table):
    """Map decoded values back to code indices by exact match (bit pattern)."""
    tb = table.view(np.uint32)
    vb = vals.astype(np.float32).view(np.uint32)
    idx = np.full(vals.shape, -1, np.int64)
    for i, b in enumerate(tb):
        idx[vb == b] = i
    return idx


def test_pack_unpack_identity_nf4():
    g = inputs.rng(1)
    packed = g.integers(0, 256, size=(7, 64), dtype=np.uint8)  # K = 128
    absmax = np.ones((7, 2), np.float32)
    vals = oracle.dequant_nf4(packed, absmax)
    codes = _codes_from_values(vals, oracle.nf4_values())
    assert np.all(codes >= 0)
    hi = (packed >> 4).astype(np.int64)
    lo = (packed & 15).astype(np.int64)
    assert np.array_equal(codes[:, 0::2], hi) and np.array_equal(codes[:, 1::2], lo)
    # and quantising the decoded values gives the same bytes back
    p2, a2 = oracle.quant_nf4(vals)
    # blocks that lack a +-1 code renormalise; compare only blocks holding one
    full = np.array([[np.any((c == 0) | (c == 15)) for c in np.split(row, 2)] for row in codes])
    for r in range(7):
        for b in range(2):
            if full[r, b] and a2[r, b] == 1.0:
                assert np.array_equal(p2[r, 32 * b:32 * b + 32], packed[r, 32 * b:32 * b + 32])


def test_pack_unpack_identity_mxfp4():
    g = inputs.rng(2)
    blocks = g.integers(0, 256, size=(5, 48), dtype=np.uint8)  # K = 96
    scales = np.full((5, 3), 127, np.uint8)
    vals = oracle.dequant_mxfp4(blocks, scales)
    codes = _codes_from_values(vals, oracle.e2m1_values())
    assert np.all(codes >= 0)
    assert np.array_equal(codes[:, 0::2], blocks & 15) and np.array_equal(codes[:, 1::2], blocks >> 4)


def test_pages_roundtrip_nf4():
    g = _golden("pages_roundtrip.json")["nf4"]
    w = inputs.rng(0).standard_normal(g["weight_shape"], dtype=np.float32)
    packed, absmax = oracle.quant_nf4(w)
    assert list(packed.shape) == g["packed_shape"] and packed.dtype == np.uint8
    assert list(absmax.shape) == g["absmax_shape"] and absmax.dtype == np.float32
    wq = oracle.dequant_nf4(packed, absmax)
    rel = np.linalg.norm(wq - w) / np.linalg.norm(w)
    lo, hi = g["rel_err_band"]
    assert lo <= rel <= hi, rel
    p2, a2 = oracle.quant_nf4(wq)
    assert np.array_equal(p2, packed) == g["repack_idempotent"]
    assert np.array_equal(a2, absmax)


def test_pages_roundtrip_mxfp4():
    g = _golden("pages_roundtrip.json")["mxfp4"]
    w = inputs.rng(0).standard_normal(g["weight_shape"], dtype=np.float32)
    blocks, scales = oracle.quant_mxfp4(w)
    assert blocks.size == int(np.prod(g["blocks_shape_pages"]))
    assert blocks.reshape(g["blocks_shape_pages"]).shape == tuple(g["blocks_shape_pages"])
    assert list(scales.shape) == g["scales_shape"]
    wq = oracle.dequant_mxfp4(blocks, scales)
    rel = np.linalg.norm(wq - w) / np.linalg.norm(w)
    lo, hi = g["rel_err_band"]
    assert lo <= rel <= hi, rel


def test_mxfp4_quantiser_is_ocp_rounding():
    """Values exactly on the e2m1 grid survive; midpoints round to even codes;
    values beyond 6*scale saturate."""
    row = np.zeros(32, np.float32)
    row[:8] = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    row[8:14] = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5]
    row[14] = 5.0
    row[15] = -7.0  # amax 7 -> shared exponent floor(log2 7) - 2 = 0 -> saturates to -6
    b, s = oracle.quant_mxfp4(row[None, :])
    assert s[0, 0] == 127
    out = oracle.dequant_mxfp4(b, s)[0]
    assert np.array_equal(out[:8], row[:8])
    assert np.array_equal(out[8:14], np.array([0.0, 1.0, 1.0, 2.0, 2.0, 4.0], np.float32))
    assert out[14] == 4.0 and out[15] == -6.0


# ---------------------------------------------------------------- routing


def _brute_route(ids, E):
    pairs = [(int(e), f) for f, e in enumerate(ids.reshape(-1)) if 0 <= e < E]
    pairs.sort()
    offsets = [0] * (E + 1)
    for e, _ in pairs:
        offsets[e + 1] += 1
    for e in range(E):
        offsets[e + 1] += offsets[e]
    return np.array(offsets, np.int32), np.array([f for _, f in pairs], np.int32)


@pytest.mark.parametrize("T,k,E", [(16, 2, 8), (37, 4, 128), (5, 8, 64), (1, 1, 1), (0, 2, 4)])
def test_route_matches_brute_force(T, k, E):
    g = inputs.rng(T * 31 + k)
    ids = g.integers(0, E, size=(T, k)).astype(np.int32)
    offsets, s2f, f2s, bad = oracle.route(ids, E)
    bo, bs = _brute_route(ids, E)
    assert bad == 0
    assert np.array_equal(offsets, bo)
    assert np.array_equal(s2f, bs)
    M = T * k
    assert np.array_equal(np.sort(s2f), np.arange(M))  # bijection
    assert np.array_equal(s2f[f2s], np.arange(M))
    assert np.array_equal(np.diff(offsets), np.bincount(ids.reshape(-1), minlength=E))


def test_route_drops_bad_ids_near_boundary():
    E = 16
    ids = np.array([[15, 16], [-1, 14], [15, 0], [2**30, 15]], np.int32)
    offsets, s2f, f2s, bad = oracle.route(ids, E)
    assert bad == 3
    assert offsets[E] == 5
    assert list(f2s[[1, 2, 6]]) == [-1, -1, -1]
    # expert 15 rows keep ascending flat order 0, 4, 7
    assert list(s2f[offsets[15]:offsets[16]]) == [0, 4, 7]
    assert list(s2f[offsets[E]:]) == [-1, -1, -1]


def test_gather_rows():
    g = inputs.rng(3)
    T, k, E, K = 9, 3, 5, 24
    ids = inputs.route_uniform(g, T, k, E)[0]
    x = inputs.bf16_normal(g, (T, K))
    offsets, s2f, f2s, bad = oracle.route(ids, E)
    xs = oracle.gather(x, k, s2f, int(offsets[E]))
    for p in range(T * k):
        assert np.array_equal(xs[p], x[s2f[p] // k])


# ---------------------------------------------------------------- GEMM


def _af(bits):
    return inputs.bf16_bits_to_float(bits).astype(np.float64)


def test_gemm_closed_form_row_sums_mxfp4():
    """All codes 0b0010 (= 1.0) and scale 127: Y[r, n] = sum_k A[r, k]."""
    g = inputs.rng(4)
    E, N, K, M = 3, 8, 96, 10
    a = inputs.bf16_normal(g, (M, K))
    w = np.full((E, N, K // 2), 0x22, np.uint8)
    s = np.full((E, N, K // 32), 127, np.uint8)
    offsets = np.array([0, 4, 4, M], np.int32)
    y = oracle.grouped_gemm_mxfp4(a, w, s, offsets)
    for r in range(M):
        assert np.all(y[r] == math.fsum(_af(a[r])))


def test_gemm_selects_expert_by_offsets():
    """Expert e's weights are 2^e: a wrong group index changes the power."""
    g = inputs.rng(5)
    E, N, K = 4, 16, 64
    counts = [3, 0, 5, 2]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(offsets[-1])
    a = inputs.bf16_normal(g, (M, K))
    w = np.full((E, N, K // 2), 0x22, np.uint8)
    s = np.stack([np.full((N, K // 32), 127 + e, np.uint8) for e in range(E)])
    y = oracle.grouped_gemm_mxfp4(a, w, s, offsets)
    for e in range(E):
        for r in range(offsets[e], offsets[e + 1]):
            assert np.all(y[r] == (2.0 ** e) * math.fsum(_af(a[r])))


def test_gemm_one_hot_weights_nf4():
    """Codes all 7 (zero) except one +1 per row at column pi(n): Y = A[:, pi]."""
    g = inputs.rng(6)
    E, N, K, M = 2, 32, 128, 7
    pi = g.integers(0, K, size=(E, N))
    codes = np.full((E, N, K), 7, np.uint8)
    for e in range(E):
        codes[e, np.arange(N), pi[e]] = 15
    packed = ((codes[..., 0::2] << 4) | codes[..., 1::2]).astype(np.uint8)
    absmax = np.ones((E, N, K // 64), np.float32)
    a = inputs.bf16_normal(g, (M, K))
    offsets = np.array([0, 3, M], np.int32)
    y = oracle.grouped_gemm_nf4(a, packed, absmax, offsets)
    af = _af(a)
    for r in range(M):
        e = 0 if r < 3 else 1
        assert np.array_equal(y[r], af[r, pi[e]])


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_gemm_single_expert_is_numpy_matmul(fmt):
    """E = 1 reduces to a plain GEMM Y = A W^T (N != K catches a transpose)."""
    g = inputs.rng(7)
    N, K, M = 48, 192, 13
    a = inputs.bf16_normal(g, (M, K))
    offsets = np.array([0, M], np.int32)
    if fmt == "nf4":
        w, sc = oracle.quant_nf4(inputs.normal_weights(g, (1, N, K)))
        wd = oracle.dequant_nf4(w, sc)[0].astype(np.float64)
        y = oracle.grouped_gemm_nf4(a, w, sc, offsets)
    else:
        w, sc = inputs.mxfp4_random(g, 1, N, K)
        wd = oracle.dequant_mxfp4(w, sc)[0].astype(np.float64)
        y = oracle.grouped_gemm_mxfp4(a, w, sc, offsets)
    ref = _af(a) @ wd.T
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_gemm_brute_force_tiny():
    g = inputs.rng(8)
    E, N, K, T, k = 3, 8, 64, 5, 2
    ids, _ = inputs.route_uniform(g, T, k, E)
    offsets, s2f, _, _ = oracle.route(ids, E)
    w, sc = oracle.quant_nf4(inputs.normal_weights(g, (E, N, K)))
    wd = oracle.dequant_nf4(w, sc).astype(np.float64)
    a = inputs.bf16_normal(g, (T * k, K))
    af = _af(a)
    y = oracle.grouped_gemm_nf4(a, w, sc, offsets)
    for e in range(E):
        for r in range(offsets[e], offsets[e + 1]):
            for n in range(N):
                ref = math.fsum(af[r, kk] * wd[e, n, kk] for kk in range(K))
                assert abs(y[r, n] - ref) <= 1e-14 * max(1.0, abs(ref))


def test_gemm_requested_rows_subset():
    g = inputs.rng(9)
    E, N, K, M = 4, 16, 64, 20
    offsets = np.array([0, 5, 5, 12, M], np.int32)
    w, sc = inputs.mxfp4_random(g, E, N, K)
    a = inputs.bf16_normal(g, (M, K))
    full = oracle.grouped_gemm_mxfp4(a, w, sc, offsets)
    rows = np.array([19, 0, 7, 11], np.int64)
    part = oracle.grouped_gemm_mxfp4(a, w, sc, offsets, rows=rows)
    assert np.array_equal(part, full[rows])


# ---------------------------------------------------------------- combine


def test_combine_one_hot_is_gather():
    g = inputs.rng(10)
    T, k, E, N = 6, 3, 4, 40
    ids, _ = inputs.route_uniform(g, T, k, E)
    offsets, s2f, f2s, _ = oracle.route(ids, E)
    y = inputs.bf16_normal(g, (T * k, N))
    w = np.zeros((T, k), np.float32)
    pick = g.integers(0, k, size=T)
    w[np.arange(T), pick] = 1.0
    out = oracle.combine(y, f2s, w)
    for t in range(T):
        assert np.array_equal(out[t], _af(y[f2s[t * k + pick[t]]]))


def test_combine_brute_force_and_dropped_pairs():
    g = inputs.rng(11)
    T, k, E, N = 7, 4, 6, 16
    ids, wts = inputs.route_uniform(g, T, k, E)
    ids[2, 1] = E  # dropped pair
    offsets, s2f, f2s, bad = oracle.route(ids, E)
    assert bad == 1
    y = inputs.bf16_normal(g, (T * k, N))
    out = oracle.combine(y, f2s, wts)
    yf = _af(y)
    for t in range(T):
        for n in range(N):
            terms = [float(wts[t, j]) * yf[f2s[t * k + j], n] for j in range(k) if f2s[t * k + j] >= 0]
            assert abs(out[t, n] - math.fsum(terms)) <= 1e-14 * max(1.0, sum(abs(x) for x in terms))


def test_combine_weights_summing_to_one_reproduce_a_shared_row():
    g = inputs.rng(12)
    T, k, E, N = 4, 4, 8, 32
    ids, wts = inputs.route_uniform(g, T, k, E)
    offsets, s2f, f2s, _ = oracle.route(ids, E)
    row = inputs.bf16_normal(g, (1, N))
    y = np.repeat(row, T * k, axis=0)
    out = oracle.combine(y, f2s, wts)
    wsum = wts.astype(np.float64).sum(axis=1)
    assert np.allclose(out, wsum[:, None] * _af(row), rtol=1e-15, atol=0)
    assert np.allclose(wsum, 1.0, atol=1e-6)


# ------------------------------------------------------------------ SwiGLU (reading C17)


def test_silu_closed_forms():
    """sigmoid(ln 3) = 3/4, so silu(ln 3) = 0.75 ln 3 and silu(-ln 3) = -0.25 ln 3;
    silu(0) = 0; an up value of 0 zeroes the product."""
    L = math.log(3.0)
    gu = np.array([[L, -L, 0.0, 5.0, 1.0, 1.0, 1.0, 0.0]], np.float64)  # gate | up, I = 4
    h = oracle.swiglu(gu)[0]
    assert abs(h[0] - 0.75 * L) <= 1e-15
    assert abs(h[1] + 0.25 * L) <= 1e-15
    assert h[2] == 0.0
    assert h[3] == 0.0


def test_silu_odd_part_is_identity():
    """x*sigmoid(x) - (-x)*sigmoid(-x) = x (since sigmoid(x) + sigmoid(-x) = 1)."""
    g = inputs.rng(50).standard_normal(64) * 4
    gu = np.stack([np.concatenate([g, np.ones(64)]), np.concatenate([-g, np.ones(64)])])
    h = oracle.swiglu(gu)
    np.testing.assert_allclose(h[0] - h[1], g, rtol=0, atol=1e-13)


def test_swiglu_takes_the_gate_half_first():
    """MXFP4 codes all 1.0: the gate half with scale 127 gives the row sum s,
    the up half with scale 126 gives s/2, so h = silu(s) * s/2; swapping the
    halves would give silu(s/2) * s."""
    g = inputs.rng(51)
    E, I, K, M = 2, 8, 64, 5
    a = inputs.bf16_normal(g, (M, K))
    w = np.full((E, 2 * I, K // 2), 0x22, np.uint8)
    s = np.full((E, 2 * I, K // 32), 127, np.uint8)
    s[:, I:, :] = 126
    offsets = np.array([0, 2, M], np.int32)
    h = oracle.grouped_gemm_swiglu("mxfp4", a, w, s, offsets)
    for r in range(M):
        rs = math.fsum(_af(a[r]))
        ref = oracle.swiglu(np.array([[rs, rs / 2.0]]))[0, 0]
        swapped = oracle.swiglu(np.array([[rs / 2.0, rs]]))[0, 0]
        assert np.all(h[r] == ref)
        assert rs == 0.0 or ref != swapped


# ------------------------------------------------------------------ router epilogue (reading C18)


def test_router_selection_is_a_stable_descending_sort():
    """numpy's stable argsort of the negated fp32 scores (ties to the lower index)."""
    g = inputs.rng(60)
    T, E, k = 40, 24, 6
    logits = (np.round(g.standard_normal((T, E)) * 2) / 2).astype(np.float32)  # coarse grid: many ties
    bias = (np.round(g.standard_normal(E)) / 4).astype(np.float32)
    ids, _ = oracle.router_topk(logits, k, bias)
    score = (logits + bias[None, :]).astype(np.float32)
    ref = np.argsort(-score, axis=1, kind="stable")[:, :k]
    assert np.array_equal(ids, ref)
    ids0, _ = oracle.router_topk(logits, k)
    assert np.array_equal(ids0, np.argsort(-logits, axis=1, kind="stable")[:, :k])


def test_router_weights_closed_forms():
    """softmax(0, ln 3) = (1/4, 3/4); one expert gets weight 1; equal logits share 1/k."""
    L = math.log(3.0)
    logits = np.array([[0.0, -5.0, np.float32(L), -7.0],
                       [1.0, 1.0, 1.0, 1.0]], np.float32)
    ids, w = oracle.router_topk(logits, 2)
    assert list(ids[0]) == [2, 0]
    assert abs(w[0, 0] - 0.75) < 1e-7 and abs(w[0, 1] - 0.25) < 1e-7  # L rounded to fp32
    assert list(ids[1]) == [0, 1] and np.all(w[1] == 0.5)
    _, w1 = oracle.router_topk(logits, 1)
    assert np.all(w1 == 1.0)
    _, w4 = oracle.router_topk(logits[1:], 4)
    assert np.all(w4 == 0.25)


def test_router_bias_moves_selection_not_weights():
    """A bias picks experts 3 and 1, whose raw logits ln 3 and 0 set the weights."""
    L = np.float32(math.log(3.0))
    logits = np.array([[5.0, 0.0, 4.0, L]], np.float32)
    bias = np.array([-100.0, 50.0, -100.0, 60.0], np.float32)
    ids, w = oracle.router_topk(logits, 2, bias)
    assert list(ids[0]) == [3, 1]
    assert abs(w[0, 0] - 0.75) < 1e-7 and abs(w[0, 1] - 0.25) < 1e-7


def test_router_ranks_nan_scores_last():
    logits = np.array([[np.nan, -1e30, 2.0, np.nan]], np.float32)
    ids, _ = oracle.router_topk(logits, 4)
    assert list(ids[0]) == [2, 1, 0, 3]


# ------------------------------------------------------------------ dgrad


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
def test_dgrad_single_expert_is_numpy_matmul(fmt):
    """E = 1: dX = dY @ dequant(W) (numpy matmul in fp64 on the dequantised stack)."""
    g = inputs.rng(70)
    N, K, M = 48, 128, 7
    if fmt == "nf4":
        w, s = oracle.quant_nf4(inputs.normal_weights(g, (1, N, K)))
        wd = oracle.dequant_nf4(w[0], s[0])
    else:
        w, s = inputs.mxfp4_random(g, 1, N, K)
        wd = oracle.dequant_mxfp4(w[0], s[0])
    dy = inputs.bf16_normal(g, (M, N))
    dx = oracle.grouped_dgrad(fmt, dy, w, s, np.array([0, M], np.int32))
    ref = _af(dy) @ wd.astype(np.float64)
    np.testing.assert_allclose(dx, ref, rtol=1e-12, atol=1e-12)


def test_dgrad_closed_form_column_sums_mxfp4():
    """All codes 1.0, scale 127 + e for expert e: dX[r, k] = 2^e * sum_n dY[r, n]."""
    g = inputs.rng(71)
    E, N, K = 3, 40, 64
    counts = [2, 0, 3]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(offsets[-1])
    dy = inputs.bf16_normal(g, (M, N))
    w = np.full((E, N, K // 2), 0x22, np.uint8)
    s = np.stack([np.full((N, K // 32), 127 + e, np.uint8) for e in range(E)])
    dx = oracle.grouped_dgrad("mxfp4", dy, w, s, offsets)
    for e in range(E):
        for r in range(offsets[e], offsets[e + 1]):
            assert np.all(dx[r] == (2.0 ** e) * math.fsum(_af(dy[r])))


def test_dgrad_is_the_transpose_of_the_forward_gemm():
    """<dY, X W^T> = <dY W, X>: the forward GEMM and dgrad are adjoint on the same stack."""
    g = inputs.rng(72)
    E, N, K = 2, 24, 128
    counts = [3, 4]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(offsets[-1])
    w, s = oracle.quant_nf4(inputs.normal_weights(g, (E, N, K)))
    x = inputs.bf16_normal(g, (M, K))
    dy = inputs.bf16_normal(g, (M, N))
    y = oracle.grouped_gemm_nf4(x, w, s, offsets)
    dx = oracle.grouped_dgrad("nf4", dy, w, s, offsets)
    lhs = math.fsum((_af(dy) * y).ravel())
    rhs = math.fsum((dx * _af(x)).ravel())
    assert abs(lhs - rhs) <= 1e-9 * (abs(lhs) + 1.0)


# ---------------------------------------------------------------- native W4A8 (MXFP8 activations)


def _bf16_bits(vals):
    return (np.asarray(vals, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_e4m3_table_matches_torch_float8():
    """Every e4m3 code decodes as torch's float8_e4m3fn does (an independent
    implementation of the OCP E4M3 format), NaN at the same two codes."""
    torch = pytest.importorskip("torch")
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_values()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])
    assert np.flatnonzero(np.isnan(got)).tolist() == [0x7F, 0xFF]


def test_e4m3_codes_from_the_specification():
    g = _golden("mxfp8.json")
    v = oracle.e4m3_values()
    for c in g["e4m3_codes"]:
        assert v[c["code"]] == c["value"], c


def test_mxfp8_worked_block():
    """The hand-worked block: scale byte, every code (ties to even, subnormals,
    negative zero)."""
    g = _golden("mxfp8.json")
    x = np.zeros(32, np.float32)
    for i, e in enumerate(g["block"]):
        x[i] = e["x"]
    codes, scales = oracle.quant_mxfp8(_bf16_bits(x)[None, :])
    assert scales[0, 0] == g["block_scale_byte"]
    for i, e in enumerate(g["block"]):
        assert codes[0, i] == e["code"], (e, codes[0, i])
    assert np.all(codes[0, len(g["block"]):] == 0)


def test_mxfp8_saturates_above_448():
    g = _golden("mxfp8.json")["saturation"]
    x = np.zeros(32, np.float32)
    x[3] = g["amax"]
    x[4] = -g["amax"]
    codes, scales = oracle.quant_mxfp8(_bf16_bits(x)[None, :])
    assert scales[0, 0] == g["scale_byte"]
    assert codes[0, 3] == g["code"] and codes[0, 4] == (g["code"] | 0x80)


def test_mxfp8_rounding_matches_torch_float8_conversion():
    """Inside each block the codes are torch's round-to-nearest-even fp32 ->
    float8_e4m3fn conversion of x / 2^X, wherever that conversion is finite
    (|x / 2^X| < 464); beyond it the oracle saturates to 448."""
    torch = pytest.importorskip("torch")
    rng = inputs.rng(71)
    rows, K = 64, 256
    x = rng.standard_normal((rows, K)).astype(np.float32)
    x *= np.exp2(rng.integers(-20, 20, size=(rows, K // 32, 1))).repeat(32, axis=2).reshape(rows, K)
    x[5, 32:64] = 0.0  # an all-zero block
    bits = _bf16_bits(x)
    xf = (bits.astype(np.uint32) << 16).view(np.float32)
    codes, scales = oracle.quant_mxfp8(bits)
    inv = np.exp2(127.0 - scales.astype(np.float64)).repeat(32, axis=1)
    scaled = (xf.astype(np.float64) * inv).astype(np.float32)  # exact: power-of-two scaling of a bf16
    ref = torch.from_numpy(scaled).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    fin = np.abs(scaled) < 464
    assert np.array_equal(codes[fin], ref[fin])
    assert np.all((codes[~fin] & 0x7F) == 0x7E)
    assert scales[5, 1] == 0 and np.all(codes[5, 32:64] == 0)


def test_mxfp8_shared_exponent_is_the_smallest_without_overflow():
    """X is the OCP choice: the block's largest element lands in [256, 512)
    after division by 2^X (so one exponent lower would leave e4m3's range and
    one higher would waste the top binade)."""
    rng = inputs.rng(72)
    x = rng.standard_normal((200, 64)).astype(np.float32) * np.exp2(rng.integers(-30, 30, (200, 1))).astype(np.float32)
    bits = _bf16_bits(x)
    xf = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    _, scales = oracle.quant_mxfp8(bits)
    amax = np.abs(xf.reshape(200, 2, 32)).max(axis=2)
    lead = amax / np.exp2(scales.astype(np.float64) - 127.0)
    assert np.all((lead >= 256) & (lead < 512))


def test_mxfp8_dequant_error_bounds():
    """|x - dequant| <= 2^-4 |x| for normal e4m3 results (half an ulp of a
    3-bit mantissa), <= 2^-10 * 2^X for subnormal ones, < 64 * 2^X when
    saturated."""
    rng = inputs.rng(73)
    x = rng.standard_normal((128, 128)).astype(np.float32)
    x[:, ::7] *= 1e-3
    bits = _bf16_bits(x)
    xf = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    codes, scales = oracle.quant_mxfp8(bits)
    deq = oracle.dequant_mxfp8(codes, scales)
    s = np.exp2(scales.astype(np.float64) - 127.0).repeat(32, axis=1)
    v = np.abs(xf) / s
    err = np.abs(deq - xf)
    normal = (v >= 2.0 ** -6) & (v < 448)
    sub = v < 2.0 ** -6
    sat = v >= 448
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(xf[normal]))
    assert np.all(err[sub] <= 2.0 ** -10 * s[sub])
    assert np.all(err[sat] < 64 * s[sat])


def test_w4a8_gemm_is_numpy_matmul_of_the_dequantised_operands():
    rng = inputs.rng(74)
    E, N, K = 3, 24, 192
    counts = [5, 0, 7]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    M = int(offsets[-1])
    w, sw = inputs.mxfp4_random(rng, E, N, K)
    codes, sa = oracle.quant_mxfp8(inputs.bf16_normal(rng, (M, K)))
    y = oracle.grouped_gemm_w4a8(codes, sa, w, sw, offsets)
    ad = oracle.dequant_mxfp8(codes, sa)
    for e in range(E):
        r0, r1 = offsets[e], offsets[e + 1]
        if r1 == r0:
            continue
        wd = oracle.dequant_mxfp4(w[e], sw[e]).astype(np.float64)
        assert np.allclose(y[r0:r1], ad[r0:r1] @ wd.T, rtol=1e-13, atol=1e-13)


def test_w4a8_gemm_closed_form():
    """Codes 0x38 (= 1.0) with activation scale byte 127 + s and weights all
    e2m1 1.0 with scale byte 127 + t: every output is K * 2^(s + t)."""
    E, N, K = 2, 8, 128
    offsets = np.array([0, 3, 4], np.int32)
    codes = np.full((4, K), 0x38, np.uint8)
    sa = np.full((4, K // 32), 127, np.uint8)
    sa[3] = 129
    w = np.full((E, N, K // 2), 0x22, np.uint8)
    sw = np.full((E, N, K // 32), 127, np.uint8)
    sw[1] = 124
    y = oracle.grouped_gemm_w4a8(codes, sa, w, sw, offsets)
    assert np.all(y[:3] == K) and np.all(y[3] == K * 2.0 ** (2 - 3))


def test_w4a8_stays_within_the_e4m3_bound_of_the_bf16_activation_result():
    """Quantising the activations moves each product by at most 1/8 of its
    size (2^-4 when not saturated), so |Y_w4a8 - Y_bf16| <= sum |a w| / 8."""
    rng = inputs.rng(75)
    E, N, K = 2, 16, 256
    offsets = np.array([0, 6, 9], np.int32)
    w, sw = inputs.mxfp4_random(rng, E, N, K)
    a = inputs.bf16_normal(rng, (9, K))
    codes, sa = oracle.quant_mxfp8(a)
    y8 = oracle.grouped_gemm_w4a8(codes, sa, w, sw, offsets)
    y16 = oracle.grouped_gemm_mxfp4(a, w, sw, offsets)
    af = np.abs(_af(a))
    for e in range(E):
        r0, r1 = offsets[e], offsets[e + 1]
        wd = np.abs(oracle.dequant_mxfp4(w[e], sw[e]).astype(np.float64))
        bound = af[r0:r1] @ wd.T / 8
        assert np.all(np.abs(y8[r0:r1] - y16[r0:r1]) <= bound)
    rel = np.linalg.norm(y8 - y16) / np.linalg.norm(y16)
    assert rel < 0.04, rel


# ---------------------------------------------------------------- two-term MXFP8 split


def test_mxfp8_split_worked_example():
    """x = 1 + 2^-7 alone in its block, headroom rule (exponent
    floor(log2 amax) - 7): hi = 129 at scale 2^-7 rounds to 128 (code 0x70,
    scale byte 120); the residual 2^-7 is exact in lo (128 at scale 2^-14,
    code 0x70, scale byte 113): hi + lo == x.  A block of 1.9375 (which the
    single-term rule saturates at 448): 248 at scale 2^-7 is a tie between
    240 (odd code 0x77) and 256 (even code 0x78) and goes to 256; the
    residual -1/16 is exact in lo (-128 at scale 2^-11: code 0xF0, scale byte
    116)."""
    x = np.zeros(32, np.float32)
    x[5] = 1.0 + 2.0 ** -7
    hc, hs, lc, ls = oracle.quant_mxfp8_split(_bf16_bits(x)[None, :])
    assert hs[0, 0] == 120 and hc[0, 5] == 0x70
    assert ls[0, 0] == 113 and lc[0, 5] == 0x70
    assert np.all(np.delete(hc[0], 5) == 0) and np.all(np.delete(lc[0], 5) == 0)
    x[:] = 1.9375
    hc, hs, lc, ls = oracle.quant_mxfp8_split(_bf16_bits(x)[None, :])
    assert hs[0, 0] == 120 and np.all(hc[0] == 0x78)
    assert ls[0, 0] == 116 and np.all(lc[0] == 0xF0)


def test_mxfp8_split_never_saturates():
    rng = inputs.rng(81)
    x = rng.standard_normal((32, 256)).astype(np.float32) * np.float32(1.99)
    hc, hs, lc, ls = oracle.quant_mxfp8_split(_bf16_bits(x))
    v = oracle.e4m3_values()
    assert np.abs(v[hc]).max() <= 256 and np.abs(v[lc]).max() <= 256  # far below 448: nothing saturates


def test_mxfp8_split_error_bound_and_exact_residuals():
    """The residual x - hi is computed here with numpy in float64; lo must
    reproduce it within one e4m3 rounding (half an ulp: 2^-4 relative for
    normal codes, 2^-10 * 2^X_lo absolute for subnormal ones), so the split
    error never exceeds 2^-8 of the block's largest |x|; and most residuals
    (few significant bits) come back exactly."""
    rng = inputs.rng(82)
    x = rng.standard_normal((64, 512)).astype(np.float32)
    x *= np.exp2(rng.integers(-12, 12, size=(64, 16, 1))).repeat(32, axis=2).reshape(64, 512).astype(np.float32)
    bits = _bf16_bits(x)
    xf = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    hc, hs, lc, ls = oracle.quant_mxfp8_split(bits)
    hi = oracle.dequant_mxfp8(hc, hs)
    lo = oracle.dequant_mxfp8(lc, ls)
    res = xf - hi
    sl = np.exp2(ls.astype(np.float64) - 127.0).repeat(32, axis=1)
    v = np.abs(res) / sl
    err = np.abs(lo - res)
    normal = (v >= 2.0 ** -6) & (v < 448)
    assert np.all(err[normal] <= 2.0 ** -4 * np.abs(res[normal]))
    assert np.all(err[v < 2.0 ** -6] <= 2.0 ** -10 * sl[v < 2.0 ** -6])
    amax = np.abs(xf.reshape(64, 16, 32)).max(axis=2).repeat(32, axis=1)
    assert np.all(np.abs(xf - hi - lo) <= 2.0 ** -8 * amax)
    assert np.mean(hi + lo == xf) > 0.9


def test_w4a8x2_gemm_meets_the_bf16_activation_tolerance():
    """With both terms the native mode lands within the path's standard
    tolerance of the bf16-activation result (1e-2 max|ref| + 2^-7 |ref|)."""
    rng = inputs.rng(83)
    E, N, K = 3, 32, 2880
    offsets = np.array([0, 7, 7, 20], np.int32)
    w, sw = inputs.mxfp4_random(rng, E, N, K)
    a = inputs.bf16_normal(rng, (20, K))
    hc, hs, lc, ls = oracle.quant_mxfp8_split(a)
    y2 = oracle.grouped_gemm_w4a8x2(hc, hs, lc, ls, w, sw, offsets)
    y16 = oracle.grouped_gemm_mxfp4(a, w, sw, offsets)
    bound = 1e-2 * np.abs(y16).max() + 2.0 ** -7 * np.abs(y16)
    assert np.all(np.abs(y2 - y16) <= bound)
    # and it is the sum of the two single-term products
    y_hi = oracle.grouped_gemm_w4a8(hc, hs, w, sw, offsets)
    y_lo = oracle.grouped_gemm_w4a8(lc, ls, w, sw, offsets)
    assert np.allclose(y2, y_hi + y_lo, rtol=1e-14, atol=1e-12)


# ---------------------------------------------------------------- native W4A4 (MXFP4 activations)


def test_mxfp4_act_quantiser_is_the_weight_quantiser_on_bf16():
    """The activation quantiser is the pinned MXFP4 weight quantiser applied to
    the (exact) fp32 value of each bf16."""
    rng = inputs.rng(91)
    bits = inputs.bf16_normal(rng, (24, 256))
    b1, s1 = oracle.quant_mxfp4_act(bits)
    b2, s2 = oracle.quant_mxfp4(_af(bits).astype(np.float32))
    assert np.array_equal(b1, b2) and np.array_equal(s1, s2)


def test_w4a4_gemm_is_numpy_matmul_of_the_dequantised_operands():
    rng = inputs.rng(92)
    E, N, K = 3, 16, 256
    offsets = np.array([0, 5, 5, 11], np.int32)
    w, sw = inputs.mxfp4_random(rng, E, N, K)
    ab, as_ = oracle.quant_mxfp4_act(inputs.bf16_normal(rng, (11, K)))
    y = oracle.grouped_gemm_w4a4(ab, as_, w, sw, offsets)
    ad = oracle.dequant_mxfp4(ab, as_).astype(np.float64)
    for e in range(E):
        r0, r1 = offsets[e], offsets[e + 1]
        if r1 == r0:
            continue
        wd = oracle.dequant_mxfp4(w[e], sw[e]).astype(np.float64)
        assert np.allclose(y[r0:r1], ad[r0:r1] @ wd.T, rtol=1e-13, atol=1e-13)


def test_w4a4_gemm_closed_form():
    """Activation codes 0x22 (1.0, 1.0) with scale 2^s and weights 1.0 with
    scale 2^t: every output is K * 2^(s + t)."""
    E, N, K = 2, 8, 256
    offsets = np.array([0, 2, 3], np.int32)
    ab = np.full((3, K // 2), 0x22, np.uint8)
    as_ = np.full((3, K // 32), 127, np.uint8)
    as_[2] = 125
    w = np.full((E, N, K // 2), 0x22, np.uint8)
    sw = np.full((E, N, K // 32), 128, np.uint8)
    y = oracle.grouped_gemm_w4a4(ab, as_, w, sw, offsets)
    assert np.all(y[:2] == 2 * K) and np.all(y[2] == K * 2.0 ** (1 - 2))


def test_w4a4_stays_within_the_e2m1_bound_of_the_bf16_activation_result():
    """e2m1 rounds to nearest with one mantissa bit.  After division by the
    block scale 2^X, a value of at least 0.5 moves by at most 1/5 of itself
    (1/4 when saturated at 6 from below 8), and a smaller one by at most 0.25
    (it lands on 0 or 0.5).  So |a - q(a)| <= |a|/3 + 2^(X-2) for every
    activation, which bounds |Y_w4a4 - Y_bf16|.  The rms error is far larger
    than the e4m3 mode's."""
    rng = inputs.rng(93)
    E, N, K = 2, 16, 512
    offsets = np.array([0, 6, 9], np.int32)
    w, sw = inputs.mxfp4_random(rng, E, N, K)
    a = inputs.bf16_normal(rng, (9, K))
    ab, as_ = oracle.quant_mxfp4_act(a)
    y4 = oracle.grouped_gemm_w4a4(ab, as_, w, sw, offsets)
    y16 = oracle.grouped_gemm_mxfp4(a, w, sw, offsets)
    af = np.abs(_af(a))
    err_a = af / 3 + np.exp2(as_.astype(np.float64) - 127.0 - 2.0).repeat(32, axis=1)
    assert np.all(np.abs(oracle.dequant_mxfp4(ab, as_).astype(np.float64) - _af(a)) <= err_a)
    for e in range(E):
        r0, r1 = offsets[e], offsets[e + 1]
        wd = np.abs(oracle.dequant_mxfp4(w[e], sw[e]).astype(np.float64))
        assert np.all(np.abs(y4[r0:r1] - y16[r0:r1]) <= err_a[r0:r1] @ wd.T)
    rel = np.linalg.norm(y4 - y16) / np.linalg.norm(y16)
    assert 0.04 < rel < 0.2, rel
