"""GPU parity: libgnf4 through its C ABI against the CPU oracle.

Bit-exact: dequantised weights, offsets, permutations, gathered rows.
Tolerance (floating point): |gpu - oracle| <= 1e-2 * max|oracle| + 2^-7 * |oracle|.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_grouped_moe_b200 import inputs
from tests._util import (assert_within_tolerance, bf16_bits, bf16_to_f64, offsets_from_counts, sample_rows,
                         set_oracle_threads, to_dev, to_dev_bf16)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def g():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from bit_grouped_moe_b200 import gnf4
    set_oracle_threads()
    gnf4.device_errors(clear=True)
    return gnf4


def _same_float_bits(a: np.ndarray, b: np.ndarray) -> bool:
    na, nb = np.isnan(a), np.isnan(b)
    if not np.array_equal(na, nb):
        return False
    return np.array_equal(a[~na].view(np.uint32), b[~nb].view(np.uint32))


# ------------------------------------------------------------------ decode


def test_dequant_nf4_bit_exact(g):
    rng = inputs.rng(100)
    E, N, K = 3, 40, 256
    w, am = oracle.quant_nf4(inputs.normal_weights(rng, (E, N, K)))
    w = rng.integers(0, 256, size=w.shape, dtype=np.uint8)  # every code in every position
    am = am.copy()
    am[0, 0, 0] = 0.0
    am[0, 1, 1] = 1e-40  # subnormal absmax: products stay unflushed
    am[1, 2, 2] = 3.0e38
    am[2, 3, 3] = -0.5
    out = torch.empty(E, N, K, dtype=torch.float32, device="cuda")
    g.dequant_nf4_f32(to_dev(w), to_dev(am), out)
    ref = oracle.dequant_nf4(w, am)
    assert _same_float_bits(out.cpu().numpy(), ref)


def test_dequant_mxfp4_bit_exact(g):
    rng = inputs.rng(101)
    E, N, K = 2, 128, 256
    w = rng.integers(0, 256, size=(E, N, K // 2), dtype=np.uint8)
    sc = np.arange(E * N * K // 32, dtype=np.int64).reshape(E, N, K // 32) % 256  # every e8m0 value
    sc = sc.astype(np.uint8)
    out = torch.empty(E, N, K, dtype=torch.float32, device="cuda")
    g.dequant_mxfp4_f32(to_dev(w), to_dev(sc), out)
    ref = oracle.dequant_mxfp4(w, sc)
    assert _same_float_bits(out.cpu().numpy(), ref)


# ------------------------------------------------------------------ routing


def _run_route(g, ids: np.ndarray, E: int, K: int, seed: int):
    T, k = ids.shape
    M = T * k
    x = inputs.bf16_normal(inputs.rng(seed), (max(T, 1), K))[:T]
    d_ids, d_x = to_dev(ids), to_dev_bf16(x)
    off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    s2f = torch.full((max(M, 1),), -7, dtype=torch.int32, device="cuda")
    f2s = torch.full((max(M, 1),), -7, dtype=torch.int32, device="cuda")
    xs = torch.full((max(M, 1), K), 7.0, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(max(g.route_workspace_bytes(T, k, E), 16), dtype=torch.uint8, device="cuda")
    bad = torch.full((1,), -7, dtype=torch.int32, device="cuda")
    g.route_permute(d_ids, d_x, E, off, s2f, f2s, xs, ws, bad_id_count=bad)
    torch.cuda.synchronize()
    assert np.array_equal(d_ids.cpu().numpy(), ids), "topk_ids must not be modified"
    return x, off.cpu().numpy(), s2f.cpu().numpy()[:M], f2s.cpu().numpy()[:M], bf16_bits(xs)[:M], int(bad.item())


ROUTE_CASES = [
    ("tiny", 16, 2, 8, 256, "uniform"),
    ("ragged", 37, 4, 128, 64, "uniform"),
    ("decode", 1, 8, 64, 2048, "topk"),
    ("single-expert", 9, 1, 1, 32, "uniform"),
    ("empty", 0, 2, 8, 64, "uniform"),
    ("multi-chunk", 1000, 3, 5, 16, "uniform"),
    ("kimi-full", 4096, 8, 384, 7168, "zipf"),
]


@pytest.mark.parametrize("name,T,k,E,K,kind", ROUTE_CASES, ids=[c[0] for c in ROUTE_CASES])
def test_route_permute_bit_exact(g, name, T, k, E, K, kind):
    rng = inputs.rng(200 + T)
    if kind == "uniform":
        ids = inputs.route_uniform(rng, T, k, E)[0] if T else np.zeros((0, k), np.int32)
    else:
        ids = inputs.route_topk(rng, T, k, E, zipf_s=1.2 if kind == "zipf" else None)[0]
    x, off, s2f, f2s, xs, bad = _run_route(g, ids, E, K, seed=T)
    o_off, o_s2f, o_f2s, o_bad = oracle.route(ids, E)
    assert np.array_equal(off, o_off)
    assert np.array_equal(s2f, o_s2f)
    assert np.array_equal(f2s, o_f2s)
    assert bad == o_bad == 0
    if T:
        assert np.array_equal(xs, oracle.gather(x, k, o_s2f, int(o_off[E])))


def test_route_drops_and_counts_bad_ids(g):
    E = 16
    ids = np.array([[15, 16], [-1, 14], [15, 0], [2 ** 30, 15], [3, 15]], np.int32)
    x, off, s2f, f2s, xs, bad = _run_route(g, ids, E, 64, seed=5)
    o_off, o_s2f, o_f2s, o_bad = oracle.route(ids, E)
    assert bad == o_bad == 3
    assert np.array_equal(off, o_off) and np.array_equal(s2f, o_s2f) and np.array_equal(f2s, o_f2s)
    assert np.array_equal(xs, oracle.gather(x, 2, o_s2f, int(o_off[E])))


# ------------------------------------------------------------------ GEMM / GEMV


def _make_stack(fmt, E, N, K, seed):
    rng = inputs.rng(seed)
    if fmt == "nf4":
        return oracle.quant_nf4(inputs.normal_weights(rng, (E, N, K)))
    return inputs.mxfp4_random(rng, E, N, K)


def _oracle_gemm(fmt, a, w, sc, offsets, rows=None):
    fn = oracle.grouped_gemm_nf4 if fmt == "nf4" else oracle.grouped_gemm_mxfp4
    return fn(a, w, sc, offsets, rows=rows)


def _gpu_call(g, fmt, kind, a_d, w_d, sc_d, y_d, off_d=None, cnt_d=None):
    fn = {("nf4", "gemm"): g.grouped_gemm_nf4, ("mxfp4", "gemm"): g.grouped_gemm_mxfp4,
          ("nf4", "gemv"): g.grouped_gemv_nf4, ("mxfp4", "gemv"): g.grouped_gemv_mxfp4}[(fmt, kind)]
    fn(a_d, w_d, sc_d, y_d, offsets=off_d, counts=cnt_d)


GEMM_GROUPS = [0, 1, 15, 16, 17, 31, 33, 0, 127, 128, 129, 255, 300, 2]


@pytest.mark.parametrize("fmt,K", [("nf4", 448), ("mxfp4", 416), ("mxfp4", 2880), ("nf4", 2048)])
def test_grouped_gemm_ragged_parity(g, fmt, K):
    E, N = len(GEMM_GROUPS), 392  # N: three full 128-row weight tiles and an 8-row tail
    offsets = offsets_from_counts(GEMM_GROUPS)
    M = int(offsets[-1]) + 5  # trailing rows past offsets[E] must stay untouched
    w, sc = _make_stack(fmt, E, N, K, seed=300 + K)
    a = inputs.bf16_normal(inputs.rng(301), (M, K))
    y = torch.full((M, N), -3.0, dtype=torch.bfloat16, device="cuda")
    off_d = to_dev(offsets)
    _gpu_call(g, fmt, "gemm", to_dev_bf16(a), to_dev(w), to_dev(sc), y, off_d=off_d)
    torch.cuda.synchronize()
    assert g.device_errors() == 0
    assert np.array_equal(off_d.cpu().numpy(), offsets), "offsets must not be modified"
    ref = _oracle_gemm(fmt, a, w, sc, offsets)
    got = bf16_to_f64(y)
    nv = int(offsets[-1])
    assert_within_tolerance(got[:nv], ref, f"{fmt} K={K}")
    assert np.all(got[nv:] == -3.0), "rows past offsets[E] were written"


@pytest.mark.parametrize("fmt", ["nf4", "mxfp4"])
@pytest.mark.parametrize("kind", ["gemm", "gemv"])
def test_counts_and_offsets_agree(g, fmt, kind):
    counts = [3, 0, 8, 1, 5, 0, 2] if kind == "gemv" else [40, 0, 129, 1, 7]
    E, N, K = len(counts), 256, 256
    offsets = offsets_from_counts(counts)
    M = int(offsets[-1])
    w, sc = _make_stack(fmt, E, N, K, seed=310)
    a_d = to_dev_bf16(inputs.bf16_normal(inputs.rng(311), (M, K)))
    w_d, sc_d = to_dev(w), to_dev(sc)
    y1 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    cnt_d = to_dev(np.array(counts, np.int32))
    _gpu_call(g, fmt, kind, a_d, w_d, sc_d, y1, off_d=to_dev(offsets))
    _gpu_call(g, fmt, kind, a_d, w_d, sc_d, y2, cnt_d=cnt_d)
    # the same counts tensor feeds a second call unchanged (the pages' build_group_tiles bug)
    _gpu_call(g, fmt, kind, a_d, w_d, sc_d, y2, cnt_d=cnt_d)
    torch.cuda.synchronize()
    assert np.array_equal(cnt_d.cpu().numpy(), np.array(counts, np.int32))
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("fmt,K", [("nf4", 512), ("mxfp4", 480), ("nf4", 2048), ("mxfp4", 2880)])
def test_grouped_gemv_parity(g, fmt, K):
    counts = [1, 0, 2, 3, 4, 5, 6, 7, 8, 0, 1, 8]
    E, N = len(counts), 264
    offsets = offsets_from_counts(counts)
    M = int(offsets[-1]) + 3
    w, sc = _make_stack(fmt, E, N, K, seed=400 + K)
    a = inputs.bf16_normal(inputs.rng(401), (M, K))
    y = torch.full((M, N), 5.0, dtype=torch.bfloat16, device="cuda")
    _gpu_call(g, fmt, "gemv", to_dev_bf16(a), to_dev(w), to_dev(sc), y, off_d=to_dev(offsets))
    torch.cuda.synchronize()
    assert g.device_errors() == 0
    ref = _oracle_gemm(fmt, a, w, sc, offsets)
    got = bf16_to_f64(y)
    nv = int(offsets[-1])
    assert_within_tolerance(got[:nv], ref, f"gemv {fmt} K={K}")
    assert np.all(got[nv:] == 5.0)


def test_gemv_group_over_8_rows_is_refused_on_device(g):
    counts = [2, 9, 1]
    E, N, K = 3, 64, 128
    offsets = offsets_from_counts(counts)
    M = int(offsets[-1])
    w, sc = _make_stack("nf4", E, N, K, seed=410)
    a = inputs.bf16_normal(inputs.rng(411), (M, K))
    y = torch.full((M, N), 9.0, dtype=torch.bfloat16, device="cuda")
    g.grouped_gemv_nf4(to_dev_bf16(a), to_dev(w), to_dev(sc), y, offsets=to_dev(offsets))
    torch.cuda.synchronize()
    assert g.device_errors() & g.DEVERR_GEMV_ROWS
    got = bf16_to_f64(y)
    assert np.all(got[2:11] == 9.0), "the oversized group must be skipped"
    ref = _oracle_gemm("nf4", a, w, sc, offsets, rows=np.array([0, 1, 11]))
    assert_within_tolerance(got[[0, 1, 11]], ref, "other groups")


@pytest.mark.parametrize("kind", ["gemm", "gemv"])
def test_bad_offsets_flagged_not_computed(g, kind):
    E, N, K = 3, 64, 128
    offsets = np.array([0, 5, 3, 6], np.int32)  # not monotone
    w, sc = _make_stack("nf4", E, N, K, seed=420)
    a = inputs.bf16_normal(inputs.rng(421), (6, K))
    y = torch.full((6, N), 2.0, dtype=torch.bfloat16, device="cuda")
    _gpu_call(g, "nf4", kind, to_dev_bf16(a), to_dev(w), to_dev(sc), y, off_d=to_dev(offsets))
    torch.cuda.synchronize()
    assert g.device_errors() & g.DEVERR_BAD_OFFSETS
    assert torch.all(y == 2.0)


def test_bounded_wait_times_out_and_the_context_stays_usable(g):
    """The pipelines' bounded wait, run on a barrier nothing arrives on with a
    ~0.5 ms limit, raises GNF4_DEVERR_TIMEOUT and returns; the next grouped
    GEMM on the same context is still correct."""
    g.device_errors(clear=True)
    g.selftest_bounded_wait(1 << 20)
    torch.cuda.synchronize()
    assert g.device_errors(clear=True) == g.DEVERR_TIMEOUT
    E, N, K = 2, 64, 128
    offsets = np.array([0, 3, 5], np.int32)
    w, sc = _make_stack("mxfp4", E, N, K, seed=430)
    a = inputs.bf16_normal(inputs.rng(431), (5, K))
    y = torch.empty((5, N), dtype=torch.bfloat16, device="cuda")
    _gpu_call(g, "mxfp4", "gemm", to_dev_bf16(a), to_dev(w), to_dev(sc), y, off_d=to_dev(offsets))
    torch.cuda.synchronize()
    assert g.device_errors() == 0
    assert_within_tolerance(bf16_to_f64(y), _oracle_gemm("mxfp4", a, w, sc, offsets), "after the timeout")


def test_bounded_wait_rejects_a_zero_limit(g):
    with pytest.raises(g.Gnf4Error) as ei:
        g.selftest_bounded_wait(0)
    assert ei.value.status == g.ERR_INVALID_ARG


# ------------------------------------------------------------------ combine


def test_combine_parity(g):
    rng = inputs.rng(500)
    T, k, E, N = 33, 4, 16, 264
    ids, wts = inputs.route_uniform(rng, T, k, E)
    ids[3, 2] = E  # dropped pair
    off, s2f, f2s, bad = oracle.route(ids, E)
    y = inputs.bf16_normal(rng, (T * k, N))
    out = torch.empty(T, N, dtype=torch.bfloat16, device="cuda")
    g.combine(to_dev_bf16(y), to_dev(f2s), to_dev(wts), out)
    torch.cuda.synchronize()
    assert_within_tolerance(bf16_to_f64(out), oracle.combine(y, f2s, wts), "combine")
