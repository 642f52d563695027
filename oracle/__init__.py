"""CPU oracle for the grouped 4-bit MoE expert GEMM -- TEST INFRASTRUCTURE.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU legs of
``bench.py`` (its CPU baseline and its ``--impl reference`` arm) may import
this package.  The product path (the CUDA library and
its Python binding) never imports it and shares no code with it.

The arithmetic lives in ``gnf4_oracle.c`` (plain C, fp64 sums, fp32 decode).
This module compiles it with gcc on first use and wraps it with ctypes over
numpy arrays.  Every function cites the page section it follows in the C file.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gnf4_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle_gnf4.so")
_lib = None

_CFLAGS = ["-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-fno-fast-math", "-ffp-contract=off"]


def build(force: bool = False) -> str:
    """Compile the oracle shared library with gcc (no CUDA involved)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    lib.orc_set_threads.argtypes = [ctypes.c_int]
    lib.orc_get_threads.restype = ctypes.c_int
    lib.orc_nf4_values.argtypes = [P]
    lib.orc_e2m1_values.argtypes = [P]
    lib.orc_e8m0_value.argtypes = [ctypes.c_int]
    lib.orc_e8m0_value.restype = ctypes.c_float
    lib.orc_quant_nf4.argtypes = [P, I64, I64, P, P]
    lib.orc_dequant_nf4.argtypes = [P, P, I64, I64, P]
    lib.orc_quant_mxfp4.argtypes = [P, I64, I64, P, P]
    lib.orc_dequant_mxfp4.argtypes = [P, P, I64, I64, P]
    lib.orc_route.argtypes = [P, I64, I64, I64, P, P, P, P]
    lib.orc_route.restype = ctypes.c_int
    lib.orc_gather.argtypes = [P, I64, I64, P, I64, I64, P]
    lib.orc_grouped_gemm_nf4.argtypes = [P, P, P, P, I64, I64, I64, P, I64, P]
    lib.orc_grouped_gemm_mxfp4.argtypes = [P, P, P, P, I64, I64, I64, P, I64, P]
    lib.orc_combine.argtypes = [P, P, P, I64, I64, I64, P]
    lib.orc_swiglu.argtypes = [P, I64, I64, P]
    lib.orc_router_topk.argtypes = [P, P, I64, I64, I64, P, P]
    lib.orc_grouped_dgrad_nf4.argtypes = [P, P, P, P, I64, I64, I64, P, I64, P]
    lib.orc_grouped_dgrad_mxfp4.argtypes = [P, P, P, P, I64, I64, I64, P, I64, P]
    lib.orc_e4m3_values.argtypes = [P]
    lib.orc_quant_mxfp8.argtypes = [P, I64, I64, P, P]
    lib.orc_dequant_mxfp8.argtypes = [P, P, I64, I64, P]
    lib.orc_grouped_gemm_w4a8.argtypes = [P, P, P, P, P, I64, I64, I64, P, I64, P]
    lib.orc_quant_mxfp8_split.argtypes = [P, I64, I64, P, P, P, P]
    lib.orc_quant_mxfp4_act.argtypes = [P, I64, I64, P, P]
    lib.orc_grouped_gemm_w4a4.argtypes = [P, P, P, P, P, I64, I64, I64, P, I64, P]
    lib.orc_grouped_gemm_w4a8x2.argtypes = [P, P, P, P, P, P, P, I64, I64, I64, P, I64, P]
    _lib = lib
    return lib


def _c(a: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=dtype)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def set_threads(n: int) -> None:
    _load().orc_set_threads(int(n))


def get_threads() -> int:
    return int(_load().orc_get_threads())


def nf4_values() -> np.ndarray:
    out = np.empty(16, np.float32)
    _load().orc_nf4_values(_p(out))
    return out


def e2m1_values() -> np.ndarray:
    out = np.empty(16, np.float32)
    _load().orc_e2m1_values(_p(out))
    return out


def e8m0_value(e: int) -> float:
    return float(np.float32(_load().orc_e8m0_value(int(e))))


def quant_nf4(w: np.ndarray):
    """[..., K] fp32 -> (packed [..., K/2] u8, absmax [..., K/64] fp32)."""
    w = _c(w, np.float32)
    K = w.shape[-1]
    if K % 64:
        raise ValueError("NF4 needs K % 64 == 0")
    rows = w.size // K
    packed = np.empty(w.shape[:-1] + (K // 2,), np.uint8)
    absmax = np.empty(w.shape[:-1] + (K // 64,), np.float32)
    _load().orc_quant_nf4(_p(w), rows, K, _p(packed), _p(absmax))
    return packed, absmax


def dequant_nf4(packed: np.ndarray, absmax: np.ndarray) -> np.ndarray:
    packed = _c(packed, np.uint8)
    absmax = _c(absmax, np.float32)
    K = packed.shape[-1] * 2
    rows = packed.size // (K // 2)
    out = np.empty(packed.shape[:-1] + (K,), np.float32)
    _load().orc_dequant_nf4(_p(packed), _p(absmax), rows, K, _p(out))
    return out


def quant_mxfp4(w: np.ndarray):
    """[..., K] fp32 -> (blocks [..., K/2] u8, scales [..., K/32] u8)."""
    w = _c(w, np.float32)
    K = w.shape[-1]
    if K % 32:
        raise ValueError("MXFP4 needs K % 32 == 0")
    rows = w.size // K
    blocks = np.empty(w.shape[:-1] + (K // 2,), np.uint8)
    scales = np.empty(w.shape[:-1] + (K // 32,), np.uint8)
    _load().orc_quant_mxfp4(_p(w), rows, K, _p(blocks), _p(scales))
    return blocks, scales


def dequant_mxfp4(blocks: np.ndarray, scales: np.ndarray) -> np.ndarray:
    blocks = _c(blocks, np.uint8)
    scales = _c(scales, np.uint8)
    K = blocks.shape[-1] * 2
    rows = blocks.size // (K // 2)
    out = np.empty(blocks.shape[:-1] + (K,), np.float32)
    _load().orc_dequant_mxfp4(_p(blocks), _p(scales), rows, K, _p(out))
    return out


def route(topk_ids: np.ndarray, E: int):
    """Stable counting sort of (token, slot) pairs by expert.

    Returns (offsets [E+1] i32, sorted_to_flat [M] i32, flat_to_sorted [M] i32, bad).
    """
    ids = _c(topk_ids, np.int32)
    T, k = ids.shape
    M = T * k
    offsets = np.empty(E + 1, np.int32)
    s2f = np.empty(max(M, 1), np.int32)
    f2s = np.empty(max(M, 1), np.int32)
    bad = ctypes.c_int64(0)
    _load().orc_route(_p(ids), T, k, E, _p(offsets), _p(s2f), _p(f2s), ctypes.cast(ctypes.pointer(bad), ctypes.c_void_p))
    return offsets, s2f[:M], f2s[:M], int(bad.value)


def gather(x_bits: np.ndarray, k: int, sorted_to_flat: np.ndarray, n_valid: int) -> np.ndarray:
    """x_bits: [T, K] uint16 (bf16 patterns) -> x_sorted [T*k, K] uint16."""
    x_bits = _c(x_bits, np.uint16)
    T, K = x_bits.shape
    M = T * k
    s2f = _c(sorted_to_flat, np.int32)
    out = np.empty((M, K), np.uint16)
    _load().orc_gather(_p(x_bits), K, k, _p(s2f), M, int(n_valid), _p(out))
    return out


def _gemm(fn, a_bits, w, scales, offsets, N, K, rows):
    a_bits = _c(a_bits, np.uint16)
    offsets = _c(offsets, np.int32)
    E = offsets.shape[0] - 1
    if rows is None:
        rows = np.arange(int(offsets[-1]), dtype=np.int64)
    rows = _c(rows, np.int64)
    y = np.empty((rows.shape[0], N), np.float64)
    fn(_p(a_bits), _p(w), _p(scales), _p(offsets), E, N, K, _p(rows), rows.shape[0], _p(y))
    return y


def grouped_gemm_nf4(a_bits, w, absmax, offsets, rows=None):
    """fp64 Y[rows, N] for the requested sorted rows (all valid rows by default)."""
    w = _c(w, np.uint8)
    absmax = _c(absmax, np.float32)
    E, N, K2 = w.shape
    return _gemm(_load().orc_grouped_gemm_nf4, a_bits, w, absmax, offsets, N, 2 * K2, rows)


def grouped_gemm_mxfp4(a_bits, w, scales, offsets, rows=None):
    w = _c(w, np.uint8)
    scales = _c(scales, np.uint8)
    E, N, K2 = w.shape
    return _gemm(_load().orc_grouped_gemm_mxfp4, a_bits, w, scales, offsets, N, 2 * K2, rows)


def combine(y_bits: np.ndarray, flat_to_sorted: np.ndarray, weights: np.ndarray) -> np.ndarray:
    """fp64 out [T, N] = sum_j weights[t, j] * Y[flat_to_sorted[t*k+j]]."""
    y_bits = _c(y_bits, np.uint16)
    f2s = _c(flat_to_sorted, np.int32)
    w = _c(weights, np.float32)
    T, k = w.shape
    N = y_bits.shape[1]
    out = np.empty((T, N), np.float64)
    _load().orc_combine(_p(y_bits), _p(f2s), _p(w), T, k, N, _p(out))
    return out


def swiglu(gate_up: np.ndarray) -> np.ndarray:
    """fp64 h [R, I] = silu(gate_up[:, :I]) * gate_up[:, I:] (gate half first)."""
    gu = _c(gate_up, np.float64)
    R, I2 = gu.shape
    I = I2 // 2
    h = np.empty((R, I), np.float64)
    _load().orc_swiglu(_p(gu), R, I, _p(h))
    return h


def grouped_gemm_swiglu(fmt: str, a_bits, w, scales, offsets, rows=None):
    """fp64 fused gate_up projection + SwiGLU: the plain GEMM over the [E, 2I, K]
    stack followed by swiglu()."""
    fn = grouped_gemm_nf4 if fmt == "nf4" else grouped_gemm_mxfp4
    return swiglu(fn(a_bits, w, scales, offsets, rows=rows))


def router_topk(logits: np.ndarray, k: int, bias: np.ndarray | None = None):
    """(ids int32 [T, k], weights fp64 [T, k]): top-k of logits + bias (fp32),
    softmax over the selected raw logits."""
    lg = _c(logits, np.float32)
    T, E = lg.shape
    b = None if bias is None else _c(bias, np.float32)
    ids = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float64)
    _load().orc_router_topk(_p(lg), None if b is None else _p(b), T, E, k, _p(ids), _p(w))
    return ids, w


def grouped_dgrad(fmt: str, dy_bits, w, scales, offsets, rows=None):
    """fp64 dX[rows, K] = dY[rows, :] . W_e for each row's expert (dY [M, N] bf16 patterns)."""
    dy_bits = _c(dy_bits, np.uint16)
    w = _c(w, np.uint8)
    scales = _c(scales, np.float32 if fmt == "nf4" else np.uint8)
    offsets = _c(offsets, np.int32)
    E, N, K2 = w.shape
    K = 2 * K2
    if rows is None:
        rows = np.arange(int(offsets[-1]), dtype=np.int64)
    rows = _c(rows, np.int64)
    dx = np.empty((rows.shape[0], K), np.float64)
    fn = _load().orc_grouped_dgrad_nf4 if fmt == "nf4" else _load().orc_grouped_dgrad_mxfp4
    fn(_p(dy_bits), _p(w), _p(scales), _p(offsets), E, N, K, _p(rows), rows.shape[0], _p(dx))
    return dx


def e4m3_values() -> np.ndarray:
    """fp64 value of every e4m3 code 0..255 (NaN for 0x7F and 0xFF)."""
    out = np.empty(256, np.float64)
    _load().orc_e4m3_values(_p(out))
    return out


def quant_mxfp8(x_bits: np.ndarray):
    """[..., K] bf16 patterns (uint16) -> (codes [..., K] u8 e4m3, scales [..., K/32] u8 e8m0)."""
    x_bits = _c(x_bits, np.uint16)
    K = x_bits.shape[-1]
    if K % 32:
        raise ValueError("MXFP8 needs K % 32 == 0")
    rows = x_bits.size // K if K else 0
    codes = np.empty(x_bits.shape, np.uint8)
    scales = np.empty(x_bits.shape[:-1] + (K // 32,), np.uint8)
    _load().orc_quant_mxfp8(_p(x_bits), rows, K, _p(codes), _p(scales))
    return codes, scales


def dequant_mxfp8(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    K = codes.shape[-1]
    rows = codes.size // K if K else 0
    out = np.empty(codes.shape, np.float64)
    _load().orc_dequant_mxfp8(_p(codes), _p(scales), rows, K, _p(out))
    return out


def grouped_gemm_w4a8(codes, a_scales, w, w_scales, offsets, rows=None):
    """fp64 Y[rows, N] of the native W4A8 mode: MXFP8 activations x MXFP4 weights."""
    codes = _c(codes, np.uint8)
    a_scales = _c(a_scales, np.uint8)
    w = _c(w, np.uint8)
    w_scales = _c(w_scales, np.uint8)
    offsets = _c(offsets, np.int32)
    E, N, K2 = w.shape
    K = 2 * K2
    if rows is None:
        rows = np.arange(int(offsets[-1]), dtype=np.int64)
    rows = _c(rows, np.int64)
    y = np.empty((rows.shape[0], N), np.float64)
    _load().orc_grouped_gemm_w4a8(_p(codes), _p(a_scales), _p(w), _p(w_scales), _p(offsets), E, N, K, _p(rows),
                                  rows.shape[0], _p(y))
    return y


def quant_mxfp8_split(x_bits: np.ndarray):
    """Two-term MXFP8 split of bf16 activations: (hi_codes, hi_scales, lo_codes, lo_scales)."""
    x_bits = _c(x_bits, np.uint16)
    K = x_bits.shape[-1]
    if K % 32:
        raise ValueError("MXFP8 needs K % 32 == 0")
    rows = x_bits.size // K if K else 0
    hc = np.empty(x_bits.shape, np.uint8)
    lc = np.empty(x_bits.shape, np.uint8)
    hs = np.empty(x_bits.shape[:-1] + (K // 32,), np.uint8)
    ls = np.empty(x_bits.shape[:-1] + (K // 32,), np.uint8)
    _load().orc_quant_mxfp8_split(_p(x_bits), rows, K, _p(hc), _p(hs), _p(lc), _p(ls))
    return hc, hs, lc, ls


def grouped_gemm_w4a8x2(hi_codes, hi_scales, lo_codes, lo_scales, w, w_scales, offsets, rows=None):
    """fp64 Y[rows, N] of the two-term native mode: (hi + lo) MXFP8 activations x MXFP4 weights."""
    hc, hs = _c(hi_codes, np.uint8), _c(hi_scales, np.uint8)
    lc, ls = _c(lo_codes, np.uint8), _c(lo_scales, np.uint8)
    w = _c(w, np.uint8)
    w_scales = _c(w_scales, np.uint8)
    offsets = _c(offsets, np.int32)
    E, N, K2 = w.shape
    K = 2 * K2
    if rows is None:
        rows = np.arange(int(offsets[-1]), dtype=np.int64)
    rows = _c(rows, np.int64)
    y = np.empty((rows.shape[0], N), np.float64)
    _load().orc_grouped_gemm_w4a8x2(_p(hc), _p(hs), _p(lc), _p(ls), _p(w), _p(w_scales), _p(offsets), E, N, K,
                                    _p(rows), rows.shape[0], _p(y))
    return y


def quant_mxfp4_act(x_bits: np.ndarray):
    """bf16 activations [..., K] -> MXFP4 (blocks [..., K/2] u8, scales [..., K/32] u8), OCP rule."""
    x_bits = _c(x_bits, np.uint16)
    K = x_bits.shape[-1]
    if K % 32:
        raise ValueError("MXFP4 needs K % 32 == 0")
    rows = x_bits.size // K if K else 0
    blocks = np.empty(x_bits.shape[:-1] + (K // 2,), np.uint8)
    scales = np.empty(x_bits.shape[:-1] + (K // 32,), np.uint8)
    _load().orc_quant_mxfp4_act(_p(x_bits), rows, K, _p(blocks), _p(scales))
    return blocks, scales


def grouped_gemm_w4a4(a_blocks, a_scales, w, w_scales, offsets, rows=None):
    """fp64 Y[rows, N] of the native W4A4 mode: MXFP4 activations x MXFP4 weights."""
    a_blocks, a_scales = _c(a_blocks, np.uint8), _c(a_scales, np.uint8)
    w, w_scales = _c(w, np.uint8), _c(w_scales, np.uint8)
    offsets = _c(offsets, np.int32)
    E, N, K2 = w.shape
    K = 2 * K2
    if rows is None:
        rows = np.arange(int(offsets[-1]), dtype=np.int64)
    rows = _c(rows, np.int64)
    y = np.empty((rows.shape[0], N), np.float64)
    _load().orc_grouped_gemm_w4a4(_p(a_blocks), _p(a_scales), _p(w), _p(w_scales), _p(offsets), E, N, K, _p(rows),
                                  rows.shape[0], _p(y))
    return y
