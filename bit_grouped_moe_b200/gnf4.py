"""Thin ctypes binding of libgnf4 (the C ABI in include/gnf4.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (device memory and streams are the
only things torch provides); the library refuses host memory, so there is no
CPU fallback anywhere.  Importing this module loads ``libgnf4.so`` and fails
loudly if it has not been built (``python -m bit_grouped_moe_b200.build``).
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgnf4.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "gnf4.h")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m bit_grouped_moe_b200.build` "
        "(libgnf4 has no CPU implementation to fall back to)")

_lib = ctypes.CDLL(LIB_PATH)

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_SHAPE, ERR_CUDA, ERR_TIMEOUT = 0, 1, 2, 3, 4
DEVERR_TIMEOUT, DEVERR_BAD_OFFSETS, DEVERR_GEMV_ROWS, DEVERR_INTERNAL = 0x1, 0x2, 0x4, 0x8
MAX_GEMV_ROWS = 8

_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t

_lib.gnf4_last_error.restype = ctypes.c_char_p
_lib.gnf4_version.restype = ctypes.c_char_p
_lib.gnf4_device_errors.argtypes = [_P, _I]
_lib.gnf4_route_workspace_bytes.argtypes = [_I, _I, _I]
_lib.gnf4_route_workspace_bytes.restype = _SZ
_lib.gnf4_route_permute.argtypes = [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _SZ, _P, _P]
_lib.gnf4_route_permute_static.argtypes = [_P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P]
_lib.gnf4_route_topk_permute.argtypes = [_P, _P, _I, _I, _I, _P, _I, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]
_GROUPED = ("gnf4_grouped_gemm_nf4", "gnf4_grouped_gemm_mxfp4", "gnf4_grouped_gemv_nf4", "gnf4_grouped_gemv_mxfp4",
            "gnf4_grouped_gemm_nf4_swiglu", "gnf4_grouped_gemm_mxfp4_swiglu", "gnf4_grouped_gemv_nf4_swiglu",
            "gnf4_grouped_gemv_mxfp4_swiglu", "gnf4_grouped_dgrad_nf4", "gnf4_grouped_dgrad_mxfp4")
for _name in _GROUPED:
    getattr(_lib, _name).argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P]
_lib.gnf4_combine_counters_bytes.argtypes = [_I, _I]
_lib.gnf4_combine_counters_bytes.restype = _SZ
for _name in ("gnf4_grouped_gemv_nf4_combine", "gnf4_grouped_gemv_mxfp4_combine", "gnf4_grouped_gemm_nf4_combine",
              "gnf4_grouped_gemm_mxfp4_combine"):
    getattr(_lib, _name).argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _I, _I, _P, _P, _P]
_lib.gnf4_selftest_bounded_wait.argtypes = [ctypes.c_ulonglong, _P]
_lib.gnf4_quantize_mxfp8.argtypes = [_P, _I, _I, _P, _P, _P]
_lib.gnf4_grouped_gemm_w4a8.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P]
_lib.gnf4_quantize_mxfp8_split.argtypes = [_P, _I, _I, _P, _P, _P, _P, _P]
_lib.gnf4_quantize_mxfp4_act.argtypes = [_P, _I, _I, _P, _P, _P]
_lib.gnf4_grouped_gemm_w4a4.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P]
_lib.gnf4_grouped_gemm_w4a8x2.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P]
_lib.gnf4_combine.argtypes = [_P, _P, _P, _I, _I, _I, _P, _P]
_lib.gnf4_grouped_gemm_mxfp4_workspace_bytes.argtypes = [_I, _I]
_lib.gnf4_grouped_gemm_mxfp4_workspace_bytes.restype = _SZ
_lib.gnf4_grouped_gemm_mxfp4_native_max_rows.argtypes = []
_lib.gnf4_grouped_gemm_mxfp4_native_max_rows.restype = _I
_lib.gnf4_grouped_gemm_mxfp4_ws.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _P, _SZ, _P]
_lib.gnf4_dequant_nf4_f32.argtypes = [_P, _P, _I64, _I, _P, _P]
_lib.gnf4_dequant_mxfp4_f32.argtypes = [_P, _P, _I64, _I, _P, _P]
_lib.gnf4_call_stats_get.argtypes = [ctypes.c_char_p, _P, _I]
_lib.gnf4_call_stats_get.restype = _I
_lib.gnf4_call_stats_name.argtypes = [_I]
_lib.gnf4_call_stats_name.restype = ctypes.c_char_p
for _name in ("gnf4_device_errors", "gnf4_route_permute", "gnf4_route_permute_static", "gnf4_route_topk_permute",
              *_GROUPED, "gnf4_combine", "gnf4_quantize_mxfp8", "gnf4_grouped_gemm_w4a8",
              "gnf4_quantize_mxfp8_split", "gnf4_grouped_gemm_w4a8x2",
              "gnf4_quantize_mxfp4_act", "gnf4_grouped_gemm_w4a4", "gnf4_selftest_bounded_wait",
              "gnf4_grouped_gemv_nf4_combine", "gnf4_grouped_gemv_mxfp4_combine", "gnf4_grouped_gemm_nf4_combine",
              "gnf4_grouped_gemm_mxfp4_combine",
              "gnf4_dequant_nf4_f32", "gnf4_dequant_mxfp4_f32", "gnf4_grouped_gemm_mxfp4_ws"):
    getattr(_lib, _name).restype = _I


class Gnf4Error(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"libgnf4 status {status}: {message}")
        self.status = status


def declared_symbols() -> list[str]:
    """Names of the entry points declared in include/gnf4.h."""
    with open(HEADER_PATH) as f:
        text = f.read()
    return sorted(set(re.findall(r"^[A-Za-z_][\w \*]*?\b(gnf4_\w+)\s*\(", text, flags=re.M)))


def version() -> str:
    return _lib.gnf4_version().decode()


def last_error() -> str:
    return _lib.gnf4_last_error().decode()


def _check(status: int) -> None:
    if status != OK:
        raise Gnf4Error(status, last_error())


# Pointers and streams go to ctypes as plain ints (every entry point has its
# argtypes set, so each is passed as a full-width pointer).  Building
# c_void_p objects and torch.cuda.current_stream() per call cost ~10 us of
# host time per launch, more than a single-token decode kernel takes.
def _ptr(t):
    return None if t is None else t.data_ptr()


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)
_cur_device = getattr(torch._C, "_cuda_getDevice", None)


def _stream(stream):
    if stream is not None:
        return stream.cuda_stream
    if _raw_stream is not None and _cur_device is not None:
        return _raw_stream(_cur_device())
    return torch.cuda.current_stream().cuda_stream


def device_errors(clear: bool = True) -> int:
    """Device error word (synchronising; diagnostics only)."""
    v = ctypes.c_uint32(0)
    _check(_lib.gnf4_device_errors(ctypes.cast(ctypes.pointer(v), ctypes.c_void_p), int(clear)))
    return int(v.value)


class CallStats(ctypes.Structure):
    """gnf4_call_stats: one entry point's engagement counters."""
    _fields_ = [(n, ctypes.c_uint64) for n in
                ("calls", "refused", "engaged", "rows", "decode_path", "native_path", "gemv_path")]


def call_stats_get(entry: str | None = None, reset: bool = False) -> dict:
    """Engagement counters of the entry point `entry` (its C name, e.g.
    "gnf4_grouped_gemm_mxfp4_ws"), or their sums over every counted entry
    point when `entry` is None; `reset` zeroes what was read.  Host-side,
    no device access."""
    s = CallStats()
    _check(_lib.gnf4_call_stats_get(None if entry is None else entry.encode(), ctypes.addressof(s), int(reset)))
    return {n: int(getattr(s, n)) for n, _ in CallStats._fields_}


def call_stats_name(i: int) -> str | None:
    """C name of the i-th counted entry point, None past the last."""
    n = _lib.gnf4_call_stats_name(i)
    return None if n is None else n.decode()


def call_stats_names() -> list[str]:
    names, i = [], 0
    while (n := call_stats_name(i)) is not None:
        names.append(n)
        i += 1
    return names


def route_workspace_bytes(T: int, k: int, E: int) -> int:
    return int(_lib.gnf4_route_workspace_bytes(T, k, E))


def route_permute(topk_ids, x, E, offsets, sorted_to_flat, flat_to_sorted, x_sorted, workspace,
                  bad_id_count=None, stream=None) -> None:
    """Stable sort of (token, slot) pairs by expert + activation gather (all outputs preallocated)."""
    T, k = topk_ids.shape
    K = x.shape[1]
    _check(_lib.gnf4_route_permute(_ptr(topk_ids), _ptr(x), T, k, E, K, _ptr(offsets), _ptr(sorted_to_flat),
                                   _ptr(flat_to_sorted), _ptr(x_sorted), _ptr(workspace),
                                   0 if workspace is None else workspace.numel() * workspace.element_size(),
                                   _ptr(bad_id_count), _stream(stream)))


def route_topk_permute(logits, x, k, topk_ids, topk_weights, offsets, sorted_to_flat, flat_to_sorted, x_sorted,
                       workspace, bias=None, stream=None) -> None:
    """Router epilogue (top-k of logits + bias, softmax over the selected logits)
    followed by route_permute on the selected ids; all outputs preallocated."""
    T, E = logits.shape
    K = x.shape[1]
    _check(_lib.gnf4_route_topk_permute(_ptr(logits), _ptr(bias), T, E, k, _ptr(x), K, _ptr(topk_ids),
                                        _ptr(topk_weights), _ptr(offsets), _ptr(sorted_to_flat),
                                        _ptr(flat_to_sorted), _ptr(x_sorted), _ptr(workspace),
                                        0 if workspace is None else workspace.numel() * workspace.element_size(),
                                        _stream(stream)))


ROUTE_STATIC_SCRATCH_BYTES = 1 << 20  # GNF4_ROUTE_STATIC_SCRATCH_BYTES in include/gnf4.h


def route_permute_static(topk_ids, x, E, offsets, sorted_to_flat, flat_to_sorted, x_sorted, bad_id_count=None,
                         stream=None) -> None:
    """route_permute without a workspace argument, for callers that cannot
    allocate device memory: the scratch is a fixed array inside libgnf4 (one
    per device, ROUTE_STATIC_SCRATCH_BYTES).  Calls that overlap on the GPU
    share that array and must be ordered; the first call on a device does a
    one-time address lookup and should come before any stream capture."""
    T, k = topk_ids.shape
    K = x.shape[1]
    _check(_lib.gnf4_route_permute_static(_ptr(topk_ids), _ptr(x), T, k, E, K, _ptr(offsets),
                                          _ptr(sorted_to_flat), _ptr(flat_to_sorted), _ptr(x_sorted),
                                          _ptr(bad_id_count), _stream(stream)))


def _grouped(fn, a, w, scales, y, offsets=None, counts=None, stream=None):
    E, N, K2 = w.shape
    M = a.shape[0]
    _check(fn(_ptr(a), _ptr(w), _ptr(scales), _ptr(offsets), _ptr(counts), E, N, 2 * K2, M, _ptr(y),
              _stream(stream)))


def grouped_gemm_nf4(a, w, absmax, y, offsets=None, counts=None, stream=None):
    _grouped(_lib.gnf4_grouped_gemm_nf4, a, w, absmax, y, offsets, counts, stream)


def grouped_gemm_mxfp4(a, w, scales, y, offsets=None, counts=None, stream=None):
    _grouped(_lib.gnf4_grouped_gemm_mxfp4, a, w, scales, y, offsets, counts, stream)


def grouped_gemm_mxfp4_workspace_bytes(M: int, K: int) -> int:
    """Workspace that lets grouped_gemm_mxfp4_ws run small groups natively (0: the native path does not apply)."""
    return int(_lib.gnf4_grouped_gemm_mxfp4_workspace_bytes(M, K))


def grouped_gemm_mxfp4_native_max_rows() -> int:
    """Largest group grouped_gemm_mxfp4_ws runs on the native block-scaled path."""
    return int(_lib.gnf4_grouped_gemm_mxfp4_native_max_rows())


mxfp4_workspace_bytes = grouped_gemm_mxfp4_workspace_bytes
mxfp4_native_max_rows = grouped_gemm_mxfp4_native_max_rows


def grouped_gemm_mxfp4_ws(a, w, scales, y, workspace, offsets=None, counts=None, stream=None):
    """MXFP4 grouped GEMM, small groups on the native two-term path (workspace: a uint8 device tensor of at least
    mxfp4_workspace_bytes(M, K) bytes, or None for the decode path throughout)."""
    E, N, K2 = w.shape
    M = a.shape[0]
    nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.gnf4_grouped_gemm_mxfp4_ws(_ptr(a), _ptr(w), _ptr(scales), _ptr(offsets), _ptr(counts), E, N, 2 * K2,
                                           M, _ptr(y), _ptr(workspace), nbytes, _stream(stream)))


def grouped_gemv_nf4(a, w, absmax, y, offsets=None, counts=None, stream=None):
    _grouped(_lib.gnf4_grouped_gemv_nf4, a, w, absmax, y, offsets, counts, stream)


def grouped_gemv_mxfp4(a, w, scales, y, offsets=None, counts=None, stream=None):
    _grouped(_lib.gnf4_grouped_gemv_mxfp4, a, w, scales, y, offsets, counts, stream)


def grouped_dgrad_nf4(dy, w, absmax, dx, offsets=None, counts=None, stream=None):
    """dX [M, K] = dY [M, N] . W_e for each row's expert (the forward stack [E, N, K/2])."""
    _grouped(_lib.gnf4_grouped_dgrad_nf4, dy, w, absmax, dx, offsets, counts, stream)


def grouped_dgrad_mxfp4(dy, w, scales, dx, offsets=None, counts=None, stream=None):
    _grouped(_lib.gnf4_grouped_dgrad_mxfp4, dy, w, scales, dx, offsets, counts, stream)


def _grouped_swiglu(fn, a, w_gate_up, scales, h, offsets=None, counts=None, stream=None):
    E, N2, K2 = w_gate_up.shape
    M = a.shape[0]
    _check(fn(_ptr(a), _ptr(w_gate_up), _ptr(scales), _ptr(offsets), _ptr(counts), E, N2 // 2, 2 * K2, M, _ptr(h),
              _stream(stream)))


def grouped_gemm_nf4_swiglu(a, w_gate_up, absmax, h, offsets=None, counts=None, stream=None):
    """h [M, I] = silu(gate) * up of the gate_up stack [E, 2I, K/2] (gate rows first)."""
    _grouped_swiglu(_lib.gnf4_grouped_gemm_nf4_swiglu, a, w_gate_up, absmax, h, offsets, counts, stream)


def grouped_gemm_mxfp4_swiglu(a, w_gate_up, scales, h, offsets=None, counts=None, stream=None):
    _grouped_swiglu(_lib.gnf4_grouped_gemm_mxfp4_swiglu, a, w_gate_up, scales, h, offsets, counts, stream)


def grouped_gemv_nf4_swiglu(a, w_gate_up, absmax, h, offsets=None, counts=None, stream=None):
    _grouped_swiglu(_lib.gnf4_grouped_gemv_nf4_swiglu, a, w_gate_up, absmax, h, offsets, counts, stream)


def grouped_gemv_mxfp4_swiglu(a, w_gate_up, scales, h, offsets=None, counts=None, stream=None):
    _grouped_swiglu(_lib.gnf4_grouped_gemv_mxfp4_swiglu, a, w_gate_up, scales, h, offsets, counts, stream)


def combine(y, flat_to_sorted, weights, out, stream=None):
    T, k = weights.shape
    N = y.shape[1]
    _check(_lib.gnf4_combine(_ptr(y), _ptr(flat_to_sorted), _ptr(weights), T, k, N, _ptr(out), _stream(stream)))


def dequant_nf4_f32(w, absmax, out, stream=None):
    K = w.shape[-1] * 2
    rows = w.numel() // (K // 2)
    _check(_lib.gnf4_dequant_nf4_f32(_ptr(w), _ptr(absmax), rows, K, _ptr(out), _stream(stream)))


def dequant_mxfp4_f32(w, scales, out, stream=None):
    K = w.shape[-1] * 2
    rows = w.numel() // (K // 2)
    _check(_lib.gnf4_dequant_mxfp4_f32(_ptr(w), _ptr(scales), rows, K, _ptr(out), _stream(stream)))


# ---------------------------------------------------------------- native MX modes


def quantize_mxfp8(x, codes, scales, stream=None):
    """x bf16 [M, K] -> codes uint8 [M, K] (e4m3) and scales uint8 [M, K/32] (e8m0), preallocated."""
    M, K = x.shape
    _check(_lib.gnf4_quantize_mxfp8(_ptr(x), M, K, _ptr(codes), _ptr(scales), _stream(stream)))


def grouped_gemm_w4a8(a_codes, a_scales, w, w_scales, y, offsets=None, counts=None, stream=None):
    """Native W4A8: y [M, N] = MXFP8 activations (codes, scales) x the MXFP4 stack [E, N, K/2] per group."""
    E, N, K2 = w.shape
    M = a_codes.shape[0]
    _check(_lib.gnf4_grouped_gemm_w4a8(_ptr(a_codes), _ptr(a_scales), _ptr(w), _ptr(w_scales), _ptr(offsets),
                                       _ptr(counts), E, N, 2 * K2, M, _ptr(y), _stream(stream)))


def selftest_bounded_wait(limit_cycles: int, stream=None) -> None:
    """One bounded pipeline wait on a barrier nothing arrives on (gives up after limit_cycles)."""
    _check(_lib.gnf4_selftest_bounded_wait(int(limit_cycles), _stream(stream)))


def combine_counters_bytes(T: int, N: int) -> int:
    return int(_lib.gnf4_combine_counters_bytes(T, N))


def _gemv_combine(fn, a, w, scales, y, sorted_to_flat, flat_to_sorted, weights, out, counters, offsets=None,
                  counts=None, stream=None):
    E, N, K2 = w.shape
    M = a.shape[0]
    T, k = weights.shape
    _check(fn(_ptr(a), _ptr(w), _ptr(scales), _ptr(offsets), _ptr(counts), E, N, 2 * K2, M, _ptr(y),
              _ptr(sorted_to_flat), _ptr(flat_to_sorted), _ptr(weights), T, k, _ptr(out), _ptr(counters),
              _stream(stream)))


def grouped_gemv_nf4_combine(a, w, absmax, y, sorted_to_flat, flat_to_sorted, weights, out, counters,
                             offsets=None, counts=None, stream=None):
    """Decode GEMV (y) with the top-k combine of y into out [T, N] in the same launch.
    counters: zeroed int32 device buffer of combine_counters_bytes(T, N) bytes (left zero)."""
    _gemv_combine(_lib.gnf4_grouped_gemv_nf4_combine, a, w, absmax, y, sorted_to_flat, flat_to_sorted, weights,
                  out, counters, offsets, counts, stream)


def grouped_gemv_mxfp4_combine(a, w, scales, y, sorted_to_flat, flat_to_sorted, weights, out, counters,
                               offsets=None, counts=None, stream=None):
    _gemv_combine(_lib.gnf4_grouped_gemv_mxfp4_combine, a, w, scales, y, sorted_to_flat, flat_to_sorted, weights,
                  out, counters, offsets, counts, stream)


def grouped_gemm_nf4_combine(a, w, absmax, y, sorted_to_flat, flat_to_sorted, weights, out, counters,
                             offsets=None, counts=None, stream=None):
    """Grouped GEMM (y) with the top-k combine of y into out [T, N] after each work unit, in the same launch.
    counters: zeroed int32 device buffer of combine_counters_bytes(T, N) bytes (left zero)."""
    _gemv_combine(_lib.gnf4_grouped_gemm_nf4_combine, a, w, absmax, y, sorted_to_flat, flat_to_sorted, weights,
                  out, counters, offsets, counts, stream)


def grouped_gemm_mxfp4_combine(a, w, scales, y, sorted_to_flat, flat_to_sorted, weights, out, counters,
                               offsets=None, counts=None, stream=None):
    _gemv_combine(_lib.gnf4_grouped_gemm_mxfp4_combine, a, w, scales, y, sorted_to_flat, flat_to_sorted, weights,
                  out, counters, offsets, counts, stream)


def quantize_mxfp8_split(x, hi_codes, hi_scales, lo_codes, lo_scales, stream=None):
    """x bf16 [M, K] -> the two-term MXFP8 split (hi + lo), all outputs preallocated."""
    M, K = x.shape
    _check(_lib.gnf4_quantize_mxfp8_split(_ptr(x), M, K, _ptr(hi_codes), _ptr(hi_scales), _ptr(lo_codes),
                                          _ptr(lo_scales), _stream(stream)))


def grouped_gemm_w4a8x2(hi_codes, hi_scales, lo_codes, lo_scales, w, w_scales, y, offsets=None, counts=None,
                        stream=None):
    """Two-term native MXFP4 GEMM: y = (hi + lo) activations x the MXFP4 stack, per group."""
    E, N, K2 = w.shape
    M = hi_codes.shape[0]
    _check(_lib.gnf4_grouped_gemm_w4a8x2(_ptr(hi_codes), _ptr(hi_scales), _ptr(lo_codes), _ptr(lo_scales), _ptr(w),
                                         _ptr(w_scales), _ptr(offsets), _ptr(counts), E, N, 2 * K2, M, _ptr(y),
                                         _stream(stream)))


def quantize_mxfp4_act(x, blocks, scales, stream=None):
    """x bf16 [M, K] -> MXFP4 blocks uint8 [M, K/2] and scales uint8 [M, K/32], preallocated."""
    M, K = x.shape
    _check(_lib.gnf4_quantize_mxfp4_act(_ptr(x), M, K, _ptr(blocks), _ptr(scales), _stream(stream)))


def grouped_gemm_w4a4(a_blocks, a_scales, w, w_scales, y, offsets=None, counts=None, stream=None):
    """Native W4A4: y [M, N] = MXFP4 activations x the MXFP4 stack [E, N, K/2] per group."""
    E, N, K2 = w.shape
    M = a_blocks.shape[0]
    _check(_lib.gnf4_grouped_gemm_w4a4(_ptr(a_blocks), _ptr(a_scales), _ptr(w), _ptr(w_scales), _ptr(offsets),
                                       _ptr(counts), E, N, 2 * K2, M, _ptr(y), _stream(stream)))
