// api.cu -- the extern "C" boundary of libgnf4 (declared in include/gnf4.h).
//
// Each entry point validates pointers and shapes on the host, encodes the
// TMA descriptors it needs, and enqueues its kernels on the caller's stream.
// Nothing here allocates device memory, synchronises the host, or falls back
// to the CPU.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "gnf4.h"
#include "internal.h"

namespace gnf4 {

// Device error word: one per device (each device holds its own copy of this
// module-scope variable).  Kernels receive its device address as a plain
// pointer; the host reads it only through gnf4_device_errors().
static __device__ unsigned g_device_errors;

namespace {

thread_local char t_last_error[512] = "";

gnf4_status fail(gnf4_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof(t_last_error), fmt, ap);
  va_end(ap);
  return s;
}

gnf4_status cuda_fail(cudaError_t e, const char* what) {
  return fail(GNF4_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

struct DeviceState {
  bool ready = false;
  int num_sms = 0;
  int cc_major = 0, cc_minor = 0;
  unsigned* err = nullptr;  // device address of g_device_errors
};

constexpr int kMaxDevices = 64;
DeviceState g_dev[kMaxDevices];
std::mutex g_dev_mu;

// Per-device set-up on first use: SM count, compute capability and the
// device address of the error word.  Touches no stream.
gnf4_status device_state(DeviceState** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(GNF4_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceState& d = g_dev[dev];
  if (!d.ready) {
    if ((e = cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
    cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_device_errors)) != cudaSuccess)
      return cuda_fail(e, "cudaGetSymbolAddress(device error word)");
    d.err = static_cast<unsigned*>(p);
    d.ready = true;
  }
  if (d.cc_major != 10) return fail(GNF4_ERR_CUDA, "libgnf4 is built for sm_100a; device is sm_%d%d", d.cc_major, d.cc_minor);
  *out = &d;
  return GNF4_OK;
}

// A pointer the GPU can read as device memory: device or managed allocations.
bool is_device_pointer(const void* p) {
  cudaPointerAttributes a;
  cudaError_t e = cudaPointerGetAttributes(&a, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged;
}

gnf4_status check_ptr(const void* p, const char* name, size_t align, bool required = true) {
  if (p == nullptr) {
    if (required) return fail(GNF4_ERR_INVALID_ARG, "%s is NULL", name);
    return GNF4_OK;
  }
  if (reinterpret_cast<uintptr_t>(p) % align != 0)
    return fail(GNF4_ERR_INVALID_ARG, "%s is not %zu-byte aligned", name, align);
  if (!is_device_pointer(p))
    return fail(GNF4_ERR_INVALID_ARG,
                "%s is not device memory: libgnf4 runs on the GPU only and never falls back to the CPU", name);
  return GNF4_OK;
}

#define GNF4_TRY(x)                  \
  do {                               \
    gnf4_status _s = (x);            \
    if (_s != GNF4_OK) return _s;    \
  } while (0)

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// A [M, K] bf16 row-major: 64 x box_rows boxes (128-byte rows), 128B swizzle, zero fill.
gnf4_status encode_act_map(CUtensorMap* m, const void* a, int M, int K, int box_rows = 32) {
  auto fn = encode_fn();
  if (!fn) return fail(GNF4_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
  cuuint64_t strides[1] = {(cuuint64_t)K * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(GNF4_ERR_CUDA, "activation tensor map encode failed (CUresult %d)", (int)r);
  return GNF4_OK;
}

// Y [M, cols] bf16 row-major, written by TMA stores of box_cols x box_rows (no swizzle).
gnf4_status encode_out_map(CUtensorMap* m, void* y, int M, int cols, int box_cols, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(GNF4_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)M};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(GNF4_ERR_CUDA, "output tensor map encode failed (CUresult %d)", (int)r);
  return GNF4_OK;
}

// W [E, N, K/2] u8: box_bytes x box_rows x 1 boxes, no swizzle, zero fill.
gnf4_status encode_weight_map(CUtensorMap* m, const void* w, int E, int N, int K, int box_bytes, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return fail(GNF4_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  cuuint64_t dims[3] = {(cuuint64_t)(K / 2), (cuuint64_t)N, (cuuint64_t)E};
  cuuint64_t strides[2] = {(cuuint64_t)(K / 2), (cuuint64_t)N * (cuuint64_t)(K / 2)};
  cuuint32_t box[3] = {(cuuint32_t)box_bytes, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(w), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(GNF4_ERR_CUDA, "weight tensor map encode failed (CUresult %d)", (int)r);
  return GNF4_OK;
}

// gate_up stack W [E, 2I, K/2] u8 viewed as [E][I/64][2][64][K/2]: one box =
// 32 bytes of 64 gate rows followed by the same 32 bytes of the matching 64 up rows.
gnf4_status encode_swiglu_weight_map(CUtensorMap* m, const void* w, int E, int I, int K) {
  auto fn = encode_fn();
  if (!fn) return fail(GNF4_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const cuuint64_t rb = (cuuint64_t)(K / 2);
  cuuint64_t dims[5] = {rb, 64, 2, (cuuint64_t)(I / 64), (cuuint64_t)E};
  cuuint64_t strides[4] = {rb, (cuuint64_t)I * rb, 64 * rb, 2 * (cuuint64_t)I * rb};
  cuuint32_t box[5] = {32, 64, 2, 1, 1};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 5, const_cast<void*>(w), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(GNF4_ERR_CUDA, "gate_up tensor map encode failed (CUresult %d)", (int)r);
  return GNF4_OK;
}

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// Shared validation of the grouped GEMM / GEMV arguments.
gnf4_status check_grouped(int fmt, const void* a, const uint8_t* w, const void* scales, const int32_t* offsets,
                          const int32_t* counts, int E, int N, int K, int M, const void* y) {
  if (E < 1 || E > kMaxExperts) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "E=%d outside [1, %d]", E, kMaxExperts);
  if (N < 1 || N % 8 != 0) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "N=%d must be a positive multiple of 8", N);
  const int kq = fmt == 0 ? 64 : 32;
  if (K < kq || K % kq != 0 || K > 65536)
    return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "K=%d must be a multiple of %d in [%d, 65536] for %s", K, kq, kq,
                fmt == 0 ? "NF4" : "MXFP4");
  if (M < 0) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "M=%d is negative", M);
  if ((offsets == nullptr) == (counts == nullptr))
    return fail(GNF4_ERR_INVALID_ARG, "pass exactly one of offsets [E+1] and counts [E]");
  if (M == 0) return GNF4_OK;
  GNF4_TRY(check_ptr(a, "a", 16));
  GNF4_TRY(check_ptr(w, "w", 16));
  GNF4_TRY(check_ptr(scales, fmt == 0 ? "absmax" : "scales", fmt == 0 ? 4 : 1));
  GNF4_TRY(check_ptr(offsets, "offsets", 4, false));
  GNF4_TRY(check_ptr(counts, "counts", 4, false));
  GNF4_TRY(check_ptr(y, "y", 16));
  return GNF4_OK;
}

// swiglu: w is a gate_up stack [E, N = 2I, K/2] and y the [M, I] output h.
// min_rows > 0: groups of fewer rows are skipped (their rows of y are left to another kernel).
// combine: the top-k combine after each unit (all groups, not with swiglu).
gnf4_status grouped_gemm(int fmt, bool swiglu, const void* a, const uint8_t* w, const void* scales,
                         const int32_t* offsets, const int32_t* counts, int E, int N, int K, int M, void* y,
                         void* stream, int min_rows = 0, const CombineArgs* combine = nullptr) {
  GNF4_TRY(check_grouped(fmt, a, w, scales, offsets, counts, E, N, K, M, y));
  if (M == 0) return GNF4_OK;
  DeviceState* d = nullptr;
  GNF4_TRY(device_state(&d));
  CUtensorMap tm_a, tm_a_big, tm_w, tm_y;
  GNF4_TRY(encode_act_map(&tm_a, a, M, K, gemm_tc_small_box_rows()));
  GNF4_TRY(encode_out_map(&tm_y, y, M, swiglu ? N / 2 : N, swiglu ? gemm_tc_weight_box_rows() / 2 : gemm_tc_weight_box_rows(),
                          gemm_tc_out_box_rows()));
  GNF4_TRY(encode_act_map(&tm_a_big, a, M, K, gemm_tc_big_box_rows()));
  const int wrows = gemm_tc_weight_rows_per_unit();
  if (swiglu)
    GNF4_TRY(encode_swiglu_weight_map(&tm_w, w, E, N / 2, K));
  else
    GNF4_TRY(encode_weight_map(&tm_w, w, E, N, K, 32, gemm_tc_weight_box_rows()));
  GroupedArgs p{static_cast<const __nv_bfloat16*>(a), w, scales, offsets, counts,
                static_cast<__nv_bfloat16*>(y), d->err, E, N, K, M};
  p.min_rows = min_rows;
  // upper bound on work units: every group adds at most one partial chunk
  const long long nwt = (N + wrows - 1) / wrows;  // SwiGLU: (2I / 128) tiles of 64 gate + 64 up rows
  const long long rpu = gemm_tc_rows_per_unit();
  const long long chunks = (M + rpu - 1) / rpu + (E < M ? E : M);
  const long long units = chunks * nwt;
  if (units >= (1LL << 31)) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "M=%d, N=%d give too many work units", M, N);
  const int grid = gemm_tc_grid(units, d->num_sms);
  cudaError_t e = launch_gemm_tc(fmt, swiglu, tm_a, tm_a_big, tm_w, tm_y, p, grid, as_stream(stream), combine);
  if (e != cudaSuccess) return cuda_fail(e, "grouped GEMM launch");
  note_launch(kPathDecode);
  return GNF4_OK;
}

gnf4_status grouped_gemv(int fmt, bool swiglu, const void* a, const uint8_t* w, const void* scales,
                         const int32_t* offsets, const int32_t* counts, int E, int N, int K, int M, void* y,
                         void* stream) {
  GNF4_TRY(check_grouped(fmt, a, w, scales, offsets, counts, E, N, K, M, y));
  if (M == 0) return GNF4_OK;
  DeviceState* d = nullptr;
  GNF4_TRY(device_state(&d));
  GroupedArgs p{static_cast<const __nv_bfloat16*>(a), w, scales, offsets, counts,
                static_cast<__nv_bfloat16*>(y), d->err, E, N, K, M};
  const long long hit = E < M ? E : M;  // groups with rows
  const long long per = swiglu ? (N / 2) / gemv_swiglu_cols_per_block()
                               : (N + gemv_rows_per_block() - 1) / gemv_rows_per_block();
  const int grid = gemv_grid(hit * per, d->num_sms);
  cudaError_t e = launch_gemv(fmt, swiglu, p, grid, as_stream(stream));
  if (e == cudaErrorInvalidConfiguration)
    return fail(GNF4_ERR_CUDA, "grouped GEMV: the decode table does not fit above the kernel's shared data");
  if (e != cudaSuccess) return cuda_fail(e, "grouped GEMV launch");
  note_launch(kPathGemv);
  return GNF4_OK;
}

// GEMV with the top-k combine in its epilogue.
gnf4_status grouped_gemv_combine(int fmt, const void* a, const uint8_t* w, const void* scales,
                                 const int32_t* offsets, const int32_t* counts, int E, int N, int K, int M, void* y,
                                 const int32_t* sorted_to_flat, const int32_t* flat_to_sorted, const float* weights,
                                 int T, int k, void* out, int32_t* counters, void* stream) {
  // every shape rule before any pointer
  if (T < 0 || k < 1) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "T=%d / k=%d invalid", T, k);
  if ((long long)T * k >= (1LL << 31)) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "T*k too large");
  GNF4_TRY(check_grouped(fmt, a, w, scales, offsets, counts, E, N, K, M, y));
  if (T == 0) return GNF4_OK;
  GNF4_TRY(check_ptr(offsets, "offsets", 4, false));
  GNF4_TRY(check_ptr(counts, "counts", 4, false));
  GNF4_TRY(check_ptr(flat_to_sorted, "flat_to_sorted", 4));
  GNF4_TRY(check_ptr(weights, "weights", 4));
  GNF4_TRY(check_ptr(out, "out", 16));
  GNF4_TRY(check_ptr(counters, "counters", 4));
  if (M > 0) GNF4_TRY(check_ptr(sorted_to_flat, "sorted_to_flat", 4));
  DeviceState* d = nullptr;
  GNF4_TRY(device_state(&d));
  GroupedArgs p{static_cast<const __nv_bfloat16*>(a), w, scales, offsets, counts,
                static_cast<__nv_bfloat16*>(y), d->err, E, N, K, M};
  CombineArgs c{sorted_to_flat, flat_to_sorted, weights, static_cast<__nv_bfloat16*>(out), counters, T, k};
  const long long hit = E < M ? E : M;
  const long long per = (N + gemv_rows_per_block() - 1) / gemv_rows_per_block();
  // at least one CTA, so tokens without a valid pair still get their zero row
  const int grid = M > 0 ? gemv_grid(hit * per, d->num_sms) : 1;
  cudaError_t e = launch_gemv(fmt, false, p, grid, as_stream(stream), &c);
  if (e == cudaErrorInvalidConfiguration)
    return fail(GNF4_ERR_CUDA, "grouped GEMV + combine: the decode table does not fit above the kernel's shared data");
  if (e != cudaSuccess) return cuda_fail(e, "grouped GEMV + combine launch");
  note_launch(kPathGemv);
  return GNF4_OK;
}

// GEMM with the top-k combine after each unit's epilogue.
gnf4_status grouped_gemm_combine(int fmt, const void* a, const uint8_t* w, const void* scales,
                                 const int32_t* offsets, const int32_t* counts, int E, int N, int K, int M, void* y,
                                 const int32_t* sorted_to_flat, const int32_t* flat_to_sorted, const float* weights,
                                 int T, int k, void* out, int32_t* counters, void* stream) {
  if (T < 0 || k < 1) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "T=%d / k=%d invalid", T, k);
  if ((long long)T * k >= (1LL << 31)) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "T*k too large");
  GNF4_TRY(check_grouped(fmt, a, w, scales, offsets, counts, E, N, K, M, y));
  if (T == 0) return GNF4_OK;
  GNF4_TRY(check_ptr(flat_to_sorted, "flat_to_sorted", 4));
  GNF4_TRY(check_ptr(weights, "weights", 4));
  GNF4_TRY(check_ptr(out, "out", 16));
  if (M == 0) {  // no routed row, so no valid pair: every output row is zero
    cudaError_t e = cudaMemsetAsync(out, 0, (size_t)T * (size_t)N * 2, as_stream(stream));
    if (e != cudaSuccess) return cuda_fail(e, "zeroing out");
    note_launch(kPathOther);
    return GNF4_OK;
  }
  GNF4_TRY(check_ptr(sorted_to_flat, "sorted_to_flat", 4));
  GNF4_TRY(check_ptr(counters, "counters", 4));
  CombineArgs c{sorted_to_flat, flat_to_sorted, weights, static_cast<__nv_bfloat16*>(out), counters, T, k};
  return grouped_gemm(fmt, false, a, w, scales, offsets, counts, E, N, K, M, y, stream, 0, &c);
}

// dY [M, N] bf16 and the [E, N, K/2] stack -> dX [M, K] bf16.
gnf4_status grouped_dgrad(int fmt, const void* dy, const uint8_t* w, const void* scales, const int32_t* offsets,
                          const int32_t* counts, int E, int N, int K, int M, void* dx, void* stream) {
  GNF4_TRY(check_grouped(fmt, dy, w, scales, offsets, counts, E, N, K, M, dx));
  if (M == 0) return GNF4_OK;
  DeviceState* d = nullptr;
  GNF4_TRY(device_state(&d));
  CUtensorMap tm_y, tm_w;
  GNF4_TRY(encode_act_map(&tm_y, dy, M, N, dgrad_tc_rows_per_unit()));
  GNF4_TRY(encode_weight_map(&tm_w, w, E, N, K, dgrad_tc_k_per_unit() / 2, dgrad_tc_n_per_stage()));
  GroupedArgs p{static_cast<const __nv_bfloat16*>(dy), w, scales, offsets, counts,
                static_cast<__nv_bfloat16*>(dx), d->err, E, N, K, M};
  const long long rpu = dgrad_tc_rows_per_unit(), kpu = dgrad_tc_k_per_unit();
  const long long units = ((M + rpu - 1) / rpu + (E < M ? E : M)) * ((K + kpu - 1) / kpu);
  if (units >= (1LL << 31)) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "M=%d, K=%d give too many work units", M, K);
  const int grid = (int)(units < d->num_sms ? units : d->num_sms);
  cudaError_t e = launch_dgrad_tc(fmt, tm_y, tm_w, p, grid, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "grouped dgrad launch");
  note_launch(kPathDecode);
  return GNF4_OK;
}

// Native W4A8 GEMM: e4m3 codes [M, K] by TMA (32- and 128-row boxes of 128 codes), the e2m1 stack as
// [E*N] x (K/128) x 128 codes expanded by the TMA unit into the padded 16-codes-per-16-bytes layout, and
// for K % 128 == 64 a second view of codes [K-128, K) of every row.
// lo_codes / lo_scales non-null: the two-term mode (a_codes / a_scales are the hi term).
gnf4_status grouped_gemm_w4a8(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* lo_codes,
                              const uint8_t* lo_scales, const uint8_t* w, const uint8_t* w_scales,
                              const int32_t* offsets, const int32_t* counts, int E, int N, int K, int M, void* y,
                              void* stream, int max_rows = 1 << 30) {
  const bool split = lo_codes != nullptr || lo_scales != nullptr;
  if (E < 1 || E > kMaxExperts) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "E=%d outside [1, %d]", E, kMaxExperts);
  if (N < 1 || N % 8 != 0) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "N=%d must be a positive multiple of 8", N);
  if (K < 128 || K % 64 != 0 || K > 65536)
    return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "K=%d must be a multiple of 64 in [128, 65536] for W4A8", K);
  if (M < 0) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "M=%d is negative", M);
  if ((long long)E * N >= (1LL << 31)) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "E*N too large");
  if ((offsets == nullptr) == (counts == nullptr))
    return fail(GNF4_ERR_INVALID_ARG, "pass exactly one of offsets [E+1] and counts [E]");
  if (M == 0) return GNF4_OK;
  GNF4_TRY(check_ptr(a_codes, split ? "hi_codes" : "a_codes", 16));
  GNF4_TRY(check_ptr(a_scales, split ? "hi_scales" : "a_scales", 2));
  if (split) {
    GNF4_TRY(check_ptr(lo_codes, "lo_codes", 16));
    GNF4_TRY(check_ptr(lo_scales, "lo_scales", 2));
  }
  GNF4_TRY(check_ptr(w, "w", 32));
  GNF4_TRY(check_ptr(w_scales, "w_scales", 2));
  GNF4_TRY(check_ptr(offsets, "offsets", 4, false));
  GNF4_TRY(check_ptr(counts, "counts", 4, false));
  GNF4_TRY(check_ptr(y, "y", 16));
  DeviceState* d = nullptr;
  GNF4_TRY(device_state(&d));
  auto fn = encode_fn();
  if (!fn) return fail(GNF4_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  CUtensorMap tm_a, tm_a_big, tm_w, tm_w_tail;
  {
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)K};
    cuuint32_t estr[2] = {1, 1};
    for (int big = 0; big < 2; ++big) {
      // single term: 32- and 128-row boxes of the codes; two terms: 32-row boxes of hi and of lo
      const uint8_t* src = (split && big) ? lo_codes : a_codes;
      cuuint32_t box[2] = {128, (cuuint32_t)((big && !split) ? gemm_mx_rows_per_unit(0) : gemm_mx_small_box_rows())};
      CUresult r = fn(big ? &tm_a_big : &tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(src), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) return fail(GNF4_ERR_CUDA, "e4m3 tensor map encode failed (CUresult %d)", (int)r);
    }
  }
  const cuuint64_t rows = (cuuint64_t)E * (cuuint64_t)N, rb = (cuuint64_t)(K / 2);
  const cuuint32_t wrows = (cuuint32_t)gemm_mx_weight_rows_per_unit();
  {
    cuuint64_t dims[3] = {128, (cuuint64_t)(K / 128), rows};
    cuuint64_t strides[2] = {64, rb};
    cuuint32_t box[3] = {128, 1, wrows};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(&tm_w, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 3, const_cast<uint8_t*>(w), dims, strides, box,
                    estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(GNF4_ERR_CUDA, "e2m1 tensor map encode failed (CUresult %d)", (int)r);
  }
  if (K % 128 != 0) {
    cuuint64_t dims[2] = {128, rows};
    cuuint64_t strides[1] = {rb};
    cuuint32_t box[2] = {128, wrows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(&tm_w_tail, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<uint8_t*>(w + (K - 128) / 2),
                    dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(GNF4_ERR_CUDA, "e2m1 tail tensor map encode failed (CUresult %d)", (int)r);
  } else {
    tm_w_tail = tm_w;  // never used
  }
  const long long nwt = (N + (long long)wrows - 1) / wrows;
  const long long rpu = gemm_mx_rows_per_unit(split ? 1 : 0);
  const long long units = ((M + rpu - 1) / rpu + (E < M ? E : M)) * nwt;
  if (units >= (1LL << 31)) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "M=%d, N=%d give too many work units", M, N);
  const int grid = (int)(units < d->num_sms ? units : d->num_sms);
  cudaError_t e = launch_gemm_mx(split ? 1 : 0, tm_a, tm_a_big, tm_w, tm_w_tail, a_scales,
                                 split ? lo_scales : nullptr, w_scales, offsets, counts,
                                 static_cast<__nv_bfloat16*>(y), d->err, E, N, K, M, grid, as_stream(stream),
                                 max_rows);
  if (e != cudaSuccess) return cuda_fail(e, "W4A8 grouped GEMM launch");
  note_launch(kPathNative);
  return GNF4_OK;
}

// Native W4A4 GEMM: both operands packed e2m1 bytes by TMA (128-byte swizzled boxes of 256 codes).
gnf4_status grouped_gemm_w4a4(const uint8_t* a_blocks, const uint8_t* a_scales, const uint8_t* w,
                              const uint8_t* w_scales, const int32_t* offsets, const int32_t* counts, int E, int N,
                              int K, int M, void* y, void* stream) {
  if (E < 1 || E > kMaxExperts) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "E=%d outside [1, %d]", E, kMaxExperts);
  if (N < 1 || N % 8 != 0) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "N=%d must be a positive multiple of 8", N);
  if (K < 256 || K % 64 != 0 || K > 65536)
    return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "K=%d must be a multiple of 64 in [256, 65536] for W4A4", K);
  if (M < 0) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "M=%d is negative", M);
  if ((long long)E * N >= (1LL << 31)) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "E*N too large");
  if ((offsets == nullptr) == (counts == nullptr))
    return fail(GNF4_ERR_INVALID_ARG, "pass exactly one of offsets [E+1] and counts [E]");
  if (M == 0) return GNF4_OK;
  GNF4_TRY(check_ptr(a_blocks, "a_blocks", 16));
  GNF4_TRY(check_ptr(a_scales, "a_scales", 2));
  GNF4_TRY(check_ptr(w, "w", 16));
  GNF4_TRY(check_ptr(w_scales, "w_scales", 2));
  GNF4_TRY(check_ptr(offsets, "offsets", 4, false));
  GNF4_TRY(check_ptr(counts, "counts", 4, false));
  GNF4_TRY(check_ptr(y, "y", 16));
  DeviceState* d = nullptr;
  GNF4_TRY(device_state(&d));
  auto fn = encode_fn();
  if (!fn) return fail(GNF4_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  CUtensorMap tm_a, tm_a_big, tm_w;
  {
    cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)M};
    cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
    cuuint32_t estr[2] = {1, 1};
    for (int big = 0; big < 2; ++big) {
      cuuint32_t box[2] = {128, (cuuint32_t)(big ? gemm_mx_rows_per_unit(2) : gemm_mx_small_box_rows())};
      CUresult r = fn(big ? &tm_a_big : &tm_a, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(a_blocks), dims,
                      strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
      if (r != CUDA_SUCCESS) return fail(GNF4_ERR_CUDA, "e2m1 activation tensor map encode failed (CUresult %d)", (int)r);
    }
  }
  {
    cuuint64_t dims[3] = {(cuuint64_t)(K / 2), (cuuint64_t)N, (cuuint64_t)E};
    cuuint64_t strides[2] = {(cuuint64_t)(K / 2), (cuuint64_t)N * (cuuint64_t)(K / 2)};
    cuuint32_t box[3] = {128, (cuuint32_t)gemm_mx_weight_rows_per_unit(), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(&tm_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<uint8_t*>(w), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(GNF4_ERR_CUDA, "e2m1 weight tensor map encode failed (CUresult %d)", (int)r);
  }
  const long long nwt = (N + (long long)gemm_mx_weight_rows_per_unit() - 1) / gemm_mx_weight_rows_per_unit();
  const long long rpu = gemm_mx_rows_per_unit(2);
  const long long units = ((M + rpu - 1) / rpu + (E < M ? E : M)) * nwt;
  if (units >= (1LL << 31)) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "M=%d, N=%d give too many work units", M, N);
  const int grid = (int)(units < d->num_sms ? units : d->num_sms);
  cudaError_t e = launch_gemm_mx(2, tm_a, tm_a_big, tm_w, tm_w, a_scales, nullptr, w_scales, offsets, counts,
                                 static_cast<__nv_bfloat16*>(y), d->err, E, N, K, M, grid, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "W4A4 grouped GEMM launch");
  note_launch(kPathNative);
  return GNF4_OK;
}

// Workspace of the MXFP4 GEMM's native path: the two-term MXFP8 split of the
// activations as hi codes [M, K], lo codes [M, K], hi scales [M, K/32] and lo
// scales [M, K/32], each part 16-byte aligned.
struct SplitWorkspace {
  size_t hi, lo, hi_scales, lo_scales, total;
};
SplitWorkspace split_workspace(int M, int K) {
  const size_t codes = (size_t)M * (size_t)K;  // a multiple of 64: K % 64 == 0
  const size_t sc = ((size_t)M * (size_t)(K / 32) + 15) & ~size_t(15);
  return {0, codes, 2 * codes, 2 * codes + sc, 2 * codes + 2 * sc};
}

// Shapes on which the native path runs (the two-term GEMM's rules).
bool native_mxfp4_applies(int E, int N, int K) { return K >= 128 && K % 64 == 0 && (long long)E * N < (1LL << 31); }

// Groups of at most gemm_mx_rows_per_unit(two-term) rows on the native
// two-term path (one unit per weight tile), larger groups on the decode path.
gnf4_status grouped_gemm_mxfp4_ws(const void* a, const uint8_t* w, const uint8_t* scales, const int32_t* offsets,
                                  const int32_t* counts, int E, int N, int K, int M, void* y, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  GNF4_TRY(check_grouped(1, a, w, scales, offsets, counts, E, N, K, M, y));
  if (M == 0) return GNF4_OK;
  if (workspace == nullptr || !native_mxfp4_applies(E, N, K))
    return grouped_gemm(1, false, a, w, scales, offsets, counts, E, N, K, M, y, stream);
  const SplitWorkspace L = split_workspace(M, K);
  if (workspace_bytes < L.total)
    return fail(GNF4_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu bytes needed", workspace_bytes,
                L.total);
  GNF4_TRY(check_ptr(workspace, "workspace", 16));
  GNF4_TRY(check_ptr(w, "w (native path: 32-byte alignment)", 32));
  DeviceState* d = nullptr;
  GNF4_TRY(device_state(&d));
  const int thr = gemm_mx_rows_per_unit(1);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  cudaError_t e = launch_quant_mxfp8_split_rows(static_cast<const __nv_bfloat16*>(a), K, offsets, counts, E, M, thr,
                                                d->err, ws + L.hi, ws + L.hi_scales, ws + L.lo, ws + L.lo_scales,
                                                d->num_sms, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "MXFP8 split quantiser (small groups) launch");
  note_launch(kPathOther);
  GNF4_TRY(grouped_gemm_w4a8(ws + L.hi, ws + L.hi_scales, ws + L.lo, ws + L.lo_scales, w, scales, offsets, counts, E,
                             N, K, M, y, stream, thr));
  if (M > thr)  // some group may hold more rows
    GNF4_TRY(grouped_gemm(1, false, a, w, scales, offsets, counts, E, N, K, M, y, stream, thr + 1));
  return GNF4_OK;
}

// The fused gate_up + SwiGLU calls take I (the output width); the stack has 2I rows.
gnf4_status check_swiglu_width(int I) {
  if (I < 64 || I % 64 != 0 || I > (1 << 29))
    return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "I=%d must be a positive multiple of 64 (gate_up stack of 2I rows)", I);
  return GNF4_OK;
}

// Fused gate_up + SwiGLU: the [E, 2I, K/2] gate_up stack -> h [M, I].
gnf4_status grouped_swiglu(bool gemv, int fmt, const void* a, const uint8_t* w_gate_up, const void* scales,
                           const int32_t* offsets, const int32_t* counts, int E, int I, int K, int M, void* h,
                           void* stream) {
  GNF4_TRY(check_swiglu_width(I));
  return gemv ? grouped_gemv(fmt, true, a, w_gate_up, scales, offsets, counts, E, 2 * I, K, M, h, stream)
              : grouped_gemm(fmt, true, a, w_gate_up, scales, offsets, counts, E, 2 * I, K, M, h, stream);
}

}  // namespace

void set_last_error(const char* msg) { snprintf(t_last_error, sizeof(t_last_error), "%s", msg); }

// ------------------------------------------------------------- engagement
namespace {

struct EntryCounters {
  std::atomic<uint64_t> calls{0}, refused{0}, engaged{0}, rows{0}, decode{0}, native{0}, gemv{0};
};

constexpr int kEntries = static_cast<int>(Entry::count);
EntryCounters g_counters[kEntries];
const char* const kEntryNames[kEntries] = {
#define GNF4_ENTRY_NAME(n) "gnf4_" #n,
    GNF4_COUNTED_ENTRIES(GNF4_ENTRY_NAME)
#undef GNF4_ENTRY_NAME
};

thread_local int t_call_depth = 0;
thread_local unsigned t_call_paths = 0;  // families the current outermost call enqueued

void add(std::atomic<uint64_t>& c, uint64_t v) { c.fetch_add(v, std::memory_order_relaxed); }

}  // namespace

CallScope::CallScope(Entry e, long long rows) : entry_(e), rows_(rows), outer_(t_call_depth++ == 0) {
  if (outer_) t_call_paths = 0;
}

CallScope::~CallScope() { --t_call_depth; }

gnf4_status CallScope::operator()(gnf4_status s) {
  if (!outer_) return s;
  EntryCounters& c = g_counters[static_cast<int>(entry_)];
  add(c.calls, 1);
  if (s != GNF4_OK) add(c.refused, 1);
  if (t_call_paths != 0) {
    add(c.engaged, 1);
    add(c.rows, rows_ > 0 ? (uint64_t)rows_ : 0);
    if (t_call_paths & kPathDecode) add(c.decode, 1);
    if (t_call_paths & kPathNative) add(c.native, 1);
    if (t_call_paths & kPathGemv) add(c.gemv, 1);
  }
  return s;
}

void note_launch(unsigned path) { t_call_paths |= path; }

}  // namespace gnf4

using namespace gnf4;

extern "C" {

const char* gnf4_last_error(void) { return t_last_error; }

const char* gnf4_version(void) { return "libgnf4 0.1.0 (sm_100a)"; }

gnf4_status gnf4_call_stats_get(const char* entry, gnf4_call_stats* out, int reset) {
  if (out == nullptr) return fail(GNF4_ERR_INVALID_ARG, "out is NULL");
  int first = 0, last = kEntries;
  if (entry != nullptr) {
    while (first < kEntries && strcmp(kEntryNames[first], entry) != 0) ++first;
    if (first == kEntries) return fail(GNF4_ERR_INVALID_ARG, "'%s' is not a counted entry point", entry);
    last = first + 1;
  }
  gnf4_call_stats sum = {};
  for (int i = first; i < last; ++i) {
    EntryCounters& c = g_counters[i];
    auto take = [reset](std::atomic<uint64_t>& v) {
      return reset ? v.exchange(0, std::memory_order_relaxed) : v.load(std::memory_order_relaxed);
    };
    sum.calls += take(c.calls);
    sum.refused += take(c.refused);
    sum.engaged += take(c.engaged);
    sum.rows += take(c.rows);
    sum.decode_path += take(c.decode);
    sum.native_path += take(c.native);
    sum.gemv_path += take(c.gemv);
  }
  *out = sum;
  return GNF4_OK;
}

const char* gnf4_call_stats_name(int i) { return i >= 0 && i < kEntries ? kEntryNames[i] : nullptr; }

gnf4_status gnf4_device_errors(uint32_t* flags, int clear) {
  if (flags == nullptr) return fail(GNF4_ERR_INVALID_ARG, "flags is NULL");
  DeviceState* d = nullptr;
  GNF4_TRY(device_state(&d));
  unsigned v = 0;
  cudaError_t e = cudaMemcpy(&v, d->err, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "reading the device error word");
  if (clear) {
    const unsigned zero = 0;
    e = cudaMemcpy(d->err, &zero, sizeof(zero), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device error word");
  }
  *flags = v;
  return GNF4_OK;
}

gnf4_status gnf4_selftest_bounded_wait(unsigned long long limit_cycles, void* stream) {
  if (limit_cycles < 1 || limit_cycles > (1ull << 32))
    return fail(GNF4_ERR_INVALID_ARG, "limit_cycles=%llu outside [1, 2^32]", limit_cycles);
  DeviceState* d = nullptr;
  GNF4_TRY(device_state(&d));
  cudaError_t e = launch_bounded_wait_probe(d->err, (long long)limit_cycles, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "bounded-wait probe launch");
  return GNF4_OK;
}

size_t gnf4_route_workspace_bytes(int T, int k, int E) {
  if (T < 0 || k < 1 || E < 1) return 0;
  return route_workspace_bytes(T, k, E);
}

static gnf4_status route_permute_impl(const int32_t* topk_ids, const void* x, int T, int k, int E, int K,
                                      int32_t* offsets, int32_t* sorted_to_flat, int32_t* flat_to_sorted,
                                      void* x_sorted, void* workspace, size_t workspace_bytes, int32_t* bad_id_count,
                                      void* stream) {
  if (T < 0) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "T=%d is negative", T);
  if (E < 1 || E > 4096) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "E=%d outside [1, 4096]", E);
  if (k < 1 || k > E) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "k=%d outside [1, E=%d]", k, E);
  if (K < 8 || K % 8 != 0) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "K=%d must be a positive multiple of 8", K);
  if ((long long)T * k > (1LL << 30)) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "T*k too large");
  GNF4_TRY(check_ptr(offsets, "offsets", 4));
  GNF4_TRY(check_ptr(bad_id_count, "bad_id_count", 4, false));
  if (T > 0) {
    GNF4_TRY(check_ptr(topk_ids, "topk_ids", 4));
    GNF4_TRY(check_ptr(x, "x", 16));
    GNF4_TRY(check_ptr(sorted_to_flat, "sorted_to_flat", 4));
    GNF4_TRY(check_ptr(flat_to_sorted, "flat_to_sorted", 4));
    GNF4_TRY(check_ptr(x_sorted, "x_sorted", 16));
  }
  const size_t need = route_workspace_bytes(T, k, E);
  if (need > 0) {
    if (workspace_bytes < need)
      return fail(GNF4_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu bytes needed",
                  workspace_bytes, need);
    GNF4_TRY(check_ptr(workspace, "workspace", 16));
  }
  DeviceState* d = nullptr;
  GNF4_TRY(device_state(&d));
  cudaError_t e = launch_route(topk_ids, static_cast<const __nv_bfloat16*>(x), T, k, E, K, offsets,
                               sorted_to_flat, flat_to_sorted, static_cast<__nv_bfloat16*>(x_sorted), workspace,
                               bad_id_count, d->num_sms, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "route_permute launch");
  note_launch(kPathOther);
  return GNF4_OK;
}

gnf4_status gnf4_route_permute(const int32_t* topk_ids, const void* x, int T, int k, int E, int K,
                               int32_t* offsets, int32_t* sorted_to_flat, int32_t* flat_to_sorted, void* x_sorted,
                               void* workspace, size_t workspace_bytes, int32_t* bad_id_count, void* stream) {
  CallScope call(Entry::route_permute, (long long)T * k);
  return call(route_permute_impl(topk_ids, x, T, k, E, K, offsets, sorted_to_flat, flat_to_sorted, x_sorted, workspace,
                                 workspace_bytes, bad_id_count, stream));
}

static gnf4_status route_topk_permute_impl(const float* logits, const float* bias, int T, int E, int k,
                                           const void* x, int K, int32_t* topk_ids, float* topk_weights,
                                           int32_t* offsets,
                                           int32_t* sorted_to_flat, int32_t* flat_to_sorted, void* x_sorted,
                                           void* workspace, size_t workspace_bytes, void* stream) {
  if (T < 0) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "T=%d is negative", T);
  if (E < 1 || E > 4096) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "E=%d outside [1, 4096]", E);
  if (k < 1 || k > E || k > kMaxRouterTopK)
    return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "k=%d outside [1, min(E=%d, %d)]", k, E, kMaxRouterTopK);
  if (K < 8 || K % 8 != 0) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "K=%d must be a positive multiple of 8", K);
  if ((long long)T * k > (1LL << 30)) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "T*k too large");
  GNF4_TRY(check_ptr(offsets, "offsets", 4));
  GNF4_TRY(check_ptr(bias, "bias", 4, false));
  if (T > 0) {
    GNF4_TRY(check_ptr(logits, "logits", 4));
    GNF4_TRY(check_ptr(x, "x", 16));
    GNF4_TRY(check_ptr(topk_ids, "topk_ids", 4));
    GNF4_TRY(check_ptr(topk_weights, "topk_weights", 4));
    GNF4_TRY(check_ptr(sorted_to_flat, "sorted_to_flat", 4));
    GNF4_TRY(check_ptr(flat_to_sorted, "flat_to_sorted", 4));
    GNF4_TRY(check_ptr(x_sorted, "x_sorted", 16));
  }
  const size_t need = route_workspace_bytes(T, k, E);
  if (need > 0) {
    if (workspace_bytes < need)
      return fail(GNF4_ERR_INVALID_ARG, "workspace of %zu bytes is smaller than the %zu bytes needed",
                  workspace_bytes, need);
    GNF4_TRY(check_ptr(workspace, "workspace", 16));
  }
  DeviceState* d = nullptr;
  GNF4_TRY(device_state(&d));
  cudaError_t e = launch_route_topk(logits, bias, T, E, k, static_cast<const __nv_bfloat16*>(x), K, topk_ids,
                                    topk_weights, offsets, sorted_to_flat, flat_to_sorted,
                                    static_cast<__nv_bfloat16*>(x_sorted), workspace, d->num_sms,
                                    as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "route_topk_permute launch");
  note_launch(kPathOther);
  return GNF4_OK;
}

gnf4_status gnf4_route_topk_permute(const float* logits, const float* bias, int T, int E, int k, const void* x, int K,
                                    int32_t* topk_ids, float* topk_weights, int32_t* offsets,
                                    int32_t* sorted_to_flat, int32_t* flat_to_sorted, void* x_sorted,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  CallScope call(Entry::route_topk_permute, (long long)T * k);
  return call(route_topk_permute_impl(logits, bias, T, E, k, x, K, topk_ids, topk_weights, offsets, sorted_to_flat,
                                      flat_to_sorted, x_sorted, workspace, workspace_bytes, stream));
}

gnf4_status gnf4_grouped_gemm_nf4(const void* a, const uint8_t* w, const float* absmax, const int32_t* offsets,
                                  const int32_t* counts, int E, int N, int K, int M, void* y, void* stream) {
  CallScope call(Entry::grouped_gemm_nf4, (long long)M);
  return call(grouped_gemm(0, false, a, w, absmax, offsets, counts, E, N, K, M, y, stream));
}

gnf4_status gnf4_grouped_gemm_mxfp4(const void* a, const uint8_t* w, const uint8_t* scales, const int32_t* offsets,
                                    const int32_t* counts, int E, int N, int K, int M, void* y, void* stream) {
  CallScope call(Entry::grouped_gemm_mxfp4, (long long)M);
  return call(grouped_gemm(1, false, a, w, scales, offsets, counts, E, N, K, M, y, stream));
}

size_t gnf4_grouped_gemm_mxfp4_workspace_bytes(int M, int K) {
  if (M < 1 || K < 128 || K % 64 != 0 || K > 65536) return 0;
  return split_workspace(M, K).total;
}

int gnf4_grouped_gemm_mxfp4_native_max_rows(void) { return gemm_mx_rows_per_unit(1); }

gnf4_status gnf4_grouped_gemm_mxfp4_ws(const void* a, const uint8_t* w, const uint8_t* scales,
                                       const int32_t* offsets, const int32_t* counts, int E, int N, int K, int M,
                                       void* y, void* workspace, size_t workspace_bytes, void* stream) {
  CallScope call(Entry::grouped_gemm_mxfp4_ws, (long long)M);
  return call(grouped_gemm_mxfp4_ws(a, w, scales, offsets, counts, E, N, K, M, y, workspace, workspace_bytes, stream));
}

gnf4_status gnf4_grouped_gemv_nf4(const void* a, const uint8_t* w, const float* absmax, const int32_t* offsets,
                                  const int32_t* counts, int E, int N, int K, int M, void* y, void* stream) {
  CallScope call(Entry::grouped_gemv_nf4, (long long)M);
  return call(grouped_gemv(0, false, a, w, absmax, offsets, counts, E, N, K, M, y, stream));
}

gnf4_status gnf4_grouped_gemv_mxfp4(const void* a, const uint8_t* w, const uint8_t* scales, const int32_t* offsets,
                                    const int32_t* counts, int E, int N, int K, int M, void* y, void* stream) {
  CallScope call(Entry::grouped_gemv_mxfp4, (long long)M);
  return call(grouped_gemv(1, false, a, w, scales, offsets, counts, E, N, K, M, y, stream));
}

static gnf4_status combine_impl(const void* y, const int32_t* flat_to_sorted, const float* weights, int T, int k, int N,
                                void* out, void* stream) {
  if (T < 0 || k < 1) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "T=%d / k=%d invalid", T, k);
  if ((long long)T * k >= (1LL << 31)) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "T*k too large");
  if (N < 8 || N % 8 != 0) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "N=%d must be a positive multiple of 8", N);
  if (T == 0) return GNF4_OK;
  GNF4_TRY(check_ptr(y, "y", 16));
  GNF4_TRY(check_ptr(flat_to_sorted, "flat_to_sorted", 4));
  GNF4_TRY(check_ptr(weights, "weights", 4));
  GNF4_TRY(check_ptr(out, "out", 16));
  DeviceState* d = nullptr;
  GNF4_TRY(device_state(&d));
  cudaError_t e = launch_combine(static_cast<const __nv_bfloat16*>(y), flat_to_sorted, weights, T, k, N,
                                 static_cast<__nv_bfloat16*>(out), d->num_sms, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "combine launch");
  note_launch(kPathOther);
  return GNF4_OK;
}

gnf4_status gnf4_combine(const void* y, const int32_t* flat_to_sorted, const float* weights, int T, int k, int N,
                         void* out, void* stream) {
  CallScope call(Entry::combine, (long long)T * k);
  return call(combine_impl(y, flat_to_sorted, weights, T, k, N, out, stream));
}

static gnf4_status dequant(int fmt, const uint8_t* w, const void* scales, int64_t rows, int K, float* out,
                           void* stream) {
  const int kq = fmt == 0 ? 64 : 32;
  if (rows < 0 || K < kq || K % kq != 0)
    return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "rows=%lld / K=%d invalid (K %% %d == 0 required)", (long long)rows, K,
                kq);
  if (rows == 0) return GNF4_OK;
  GNF4_TRY(check_ptr(w, "w", 1));
  GNF4_TRY(check_ptr(scales, fmt == 0 ? "absmax" : "scales", fmt == 0 ? 4 : 1));
  GNF4_TRY(check_ptr(out, "out", 8));
  DeviceState* d = nullptr;
  GNF4_TRY(device_state(&d));
  cudaError_t e = launch_dequant(fmt, w, scales, rows, K, out, d->num_sms, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "dequant launch");
  note_launch(kPathOther);
  return GNF4_OK;
}

gnf4_status gnf4_dequant_nf4_f32(const uint8_t* w, const float* absmax, int64_t rows, int K, float* out,
                                 void* stream) {
  CallScope call(Entry::dequant_nf4_f32, (long long)rows);
  return call(dequant(0, w, absmax, rows, K, out, stream));
}

gnf4_status gnf4_dequant_mxfp4_f32(const uint8_t* w, const uint8_t* scales, int64_t rows, int K, float* out,
                                   void* stream) {
  CallScope call(Entry::dequant_mxfp4_f32, (long long)rows);
  return call(dequant(1, w, scales, rows, K, out, stream));
}

}  // extern "C"

extern "C" {

gnf4_status gnf4_grouped_dgrad_nf4(const void* dy, const uint8_t* w, const float* absmax, const int32_t* offsets,
                                   const int32_t* counts, int E, int N, int K, int M, void* dx, void* stream) {
  CallScope call(Entry::grouped_dgrad_nf4, (long long)M);
  return call(grouped_dgrad(0, dy, w, absmax, offsets, counts, E, N, K, M, dx, stream));
}

gnf4_status gnf4_grouped_dgrad_mxfp4(const void* dy, const uint8_t* w, const uint8_t* scales, const int32_t* offsets,
                                     const int32_t* counts, int E, int N, int K, int M, void* dx, void* stream) {
  CallScope call(Entry::grouped_dgrad_mxfp4, (long long)M);
  return call(grouped_dgrad(1, dy, w, scales, offsets, counts, E, N, K, M, dx, stream));
}

gnf4_status gnf4_grouped_gemm_nf4_swiglu(const void* a, const uint8_t* w_gate_up, const float* absmax,
                                         const int32_t* offsets, const int32_t* counts, int E, int I, int K, int M,
                                         void* h, void* stream) {
  CallScope call(Entry::grouped_gemm_nf4_swiglu, (long long)M);
  return call(grouped_swiglu(false, 0, a, w_gate_up, absmax, offsets, counts, E, I, K, M, h,
                             stream));
}

size_t gnf4_combine_counters_bytes(int T, int N) {
  if (T < 0 || N < 1) return 0;
  return gemv_combine_counter_bytes(T, N);
}

gnf4_status gnf4_grouped_gemv_nf4_combine(const void* a, const uint8_t* w, const float* absmax,
                                          const int32_t* offsets, const int32_t* counts, int E, int N, int K, int M,
                                          void* y, const int32_t* sorted_to_flat, const int32_t* flat_to_sorted,
                                          const float* weights, int T, int k, void* out, int32_t* counters,
                                          void* stream) {
  CallScope call(Entry::grouped_gemv_nf4_combine, (long long)M);
  return call(grouped_gemv_combine(0, a, w, absmax, offsets, counts, E, N, K, M, y, sorted_to_flat, flat_to_sorted,
                                   weights, T, k, out, counters, stream));
}

gnf4_status gnf4_grouped_gemv_mxfp4_combine(const void* a, const uint8_t* w, const uint8_t* scales,
                                            const int32_t* offsets, const int32_t* counts, int E, int N, int K, int M,
                                            void* y, const int32_t* sorted_to_flat, const int32_t* flat_to_sorted,
                                            const float* weights, int T, int k, void* out, int32_t* counters,
                                            void* stream) {
  CallScope call(Entry::grouped_gemv_mxfp4_combine, (long long)M);
  return call(grouped_gemv_combine(1, a, w, scales, offsets, counts, E, N, K, M, y, sorted_to_flat, flat_to_sorted,
                                   weights, T, k, out, counters, stream));
}

gnf4_status gnf4_grouped_gemm_nf4_combine(const void* a, const uint8_t* w, const float* absmax,
                                          const int32_t* offsets, const int32_t* counts, int E, int N, int K, int M,
                                          void* y, const int32_t* sorted_to_flat, const int32_t* flat_to_sorted,
                                          const float* weights, int T, int k, void* out, int32_t* counters,
                                          void* stream) {
  CallScope call(Entry::grouped_gemm_nf4_combine, (long long)M);
  return call(grouped_gemm_combine(0, a, w, absmax, offsets, counts, E, N, K, M, y, sorted_to_flat, flat_to_sorted,
                                   weights, T, k, out, counters, stream));
}

gnf4_status gnf4_grouped_gemm_mxfp4_combine(const void* a, const uint8_t* w, const uint8_t* scales,
                                            const int32_t* offsets, const int32_t* counts, int E, int N, int K, int M,
                                            void* y, const int32_t* sorted_to_flat, const int32_t* flat_to_sorted,
                                            const float* weights, int T, int k, void* out, int32_t* counters,
                                            void* stream) {
  CallScope call(Entry::grouped_gemm_mxfp4_combine, (long long)M);
  return call(grouped_gemm_combine(1, a, w, scales, offsets, counts, E, N, K, M, y, sorted_to_flat, flat_to_sorted,
                                   weights, T, k, out, counters, stream));
}

static gnf4_status quantize_mxfp8_impl(const void* x, int M, int K, uint8_t* codes, uint8_t* scales, void* stream) {
  if (M < 0) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "M=%d is negative", M);
  if (K < 32 || K % 32 != 0) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "K=%d must be a positive multiple of 32", K);
  if (M == 0) return GNF4_OK;
  GNF4_TRY(check_ptr(x, "x", 16));
  GNF4_TRY(check_ptr(codes, "codes", 16));
  GNF4_TRY(check_ptr(scales, "scales", 1));
  DeviceState* d = nullptr;
  GNF4_TRY(device_state(&d));
  cudaError_t e = launch_quant_mxfp8(static_cast<const __nv_bfloat16*>(x), (long long)M * K, codes, scales, nullptr,
                                     nullptr, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "MXFP8 quantiser launch");
  note_launch(kPathOther);
  return GNF4_OK;
}

gnf4_status gnf4_quantize_mxfp8(const void* x, int M, int K, uint8_t* codes, uint8_t* scales, void* stream) {
  CallScope call(Entry::quantize_mxfp8, (long long)M);
  return call(quantize_mxfp8_impl(x, M, K, codes, scales, stream));
}

gnf4_status gnf4_grouped_gemm_w4a8(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* w,
                                   const uint8_t* w_scales, const int32_t* offsets, const int32_t* counts, int E,
                                   int N, int K, int M, void* y, void* stream) {
  CallScope call(Entry::grouped_gemm_w4a8, (long long)M);
  return call(
      grouped_gemm_w4a8(a_codes, a_scales, nullptr, nullptr, w, w_scales, offsets, counts, E, N, K, M, y, stream));
}

static gnf4_status quantize_mxfp4_act_impl(const void* x, int M, int K, uint8_t* blocks, uint8_t* scales,
                                           void* stream) {
  if (M < 0) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "M=%d is negative", M);
  if (K < 32 || K % 32 != 0) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "K=%d must be a positive multiple of 32", K);
  if (M == 0) return GNF4_OK;
  GNF4_TRY(check_ptr(x, "x", 16));
  GNF4_TRY(check_ptr(blocks, "blocks", 4));
  GNF4_TRY(check_ptr(scales, "scales", 1));
  DeviceState* d = nullptr;
  GNF4_TRY(device_state(&d));
  cudaError_t e = launch_quant_mxfp4_act(static_cast<const __nv_bfloat16*>(x), (long long)M * K, blocks, scales,
                                         as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "MXFP4 activation quantiser launch");
  note_launch(kPathOther);
  return GNF4_OK;
}

gnf4_status gnf4_quantize_mxfp4_act(const void* x, int M, int K, uint8_t* blocks, uint8_t* scales, void* stream) {
  CallScope call(Entry::quantize_mxfp4_act, (long long)M);
  return call(quantize_mxfp4_act_impl(x, M, K, blocks, scales, stream));
}

gnf4_status gnf4_grouped_gemm_w4a4(const uint8_t* a_blocks, const uint8_t* a_scales, const uint8_t* w,
                                   const uint8_t* w_scales, const int32_t* offsets, const int32_t* counts, int E,
                                   int N, int K, int M, void* y, void* stream) {
  CallScope call(Entry::grouped_gemm_w4a4, (long long)M);
  return call(grouped_gemm_w4a4(a_blocks, a_scales, w, w_scales, offsets, counts, E, N, K, M, y, stream));
}

static gnf4_status quantize_mxfp8_split_impl(const void* x, int M, int K, uint8_t* hi_codes, uint8_t* hi_scales,
                                             uint8_t* lo_codes, uint8_t* lo_scales, void* stream) {
  if (M < 0) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "M=%d is negative", M);
  if (K < 32 || K % 32 != 0) return fail(GNF4_ERR_UNSUPPORTED_SHAPE, "K=%d must be a positive multiple of 32", K);
  if (M == 0) return GNF4_OK;
  GNF4_TRY(check_ptr(x, "x", 16));
  GNF4_TRY(check_ptr(hi_codes, "hi_codes", 16));
  GNF4_TRY(check_ptr(hi_scales, "hi_scales", 1));
  GNF4_TRY(check_ptr(lo_codes, "lo_codes", 16));
  GNF4_TRY(check_ptr(lo_scales, "lo_scales", 1));
  DeviceState* d = nullptr;
  GNF4_TRY(device_state(&d));
  cudaError_t e = launch_quant_mxfp8(static_cast<const __nv_bfloat16*>(x), (long long)M * K, hi_codes, hi_scales,
                                     lo_codes, lo_scales, as_stream(stream));
  if (e != cudaSuccess) return cuda_fail(e, "MXFP8 split quantiser launch");
  note_launch(kPathOther);
  return GNF4_OK;
}

gnf4_status gnf4_quantize_mxfp8_split(const void* x, int M, int K, uint8_t* hi_codes, uint8_t* hi_scales,
                                      uint8_t* lo_codes, uint8_t* lo_scales, void* stream) {
  CallScope call(Entry::quantize_mxfp8_split, (long long)M);
  return call(quantize_mxfp8_split_impl(x, M, K, hi_codes, hi_scales, lo_codes, lo_scales, stream));
}

static gnf4_status grouped_gemm_w4a8x2_impl(const uint8_t* hi_codes, const uint8_t* hi_scales, const uint8_t* lo_codes,
                                            const uint8_t* lo_scales, const uint8_t* w, const uint8_t* w_scales,
                                            const int32_t* offsets, const int32_t* counts, int E, int N, int K, int M,
                                            void* y, void* stream) {
  if (lo_codes == nullptr || lo_scales == nullptr) return fail(GNF4_ERR_INVALID_ARG, "lo_codes / lo_scales is NULL");
  return grouped_gemm_w4a8(hi_codes, hi_scales, lo_codes, lo_scales, w, w_scales, offsets, counts, E, N, K, M, y,
                           stream);
}

gnf4_status gnf4_grouped_gemm_w4a8x2(const uint8_t* hi_codes, const uint8_t* hi_scales, const uint8_t* lo_codes,
                                     const uint8_t* lo_scales, const uint8_t* w, const uint8_t* w_scales,
                                     const int32_t* offsets, const int32_t* counts, int E, int N, int K, int M,
                                     void* y, void* stream) {
  CallScope call(Entry::grouped_gemm_w4a8x2, (long long)M);
  return call(grouped_gemm_w4a8x2_impl(hi_codes, hi_scales, lo_codes, lo_scales, w, w_scales, offsets, counts, E, N, K,
                                       M, y, stream));
}

gnf4_status gnf4_grouped_gemm_mxfp4_swiglu(const void* a, const uint8_t* w_gate_up, const uint8_t* scales,
                                           const int32_t* offsets, const int32_t* counts, int E, int I, int K, int M,
                                           void* h, void* stream) {
  CallScope call(Entry::grouped_gemm_mxfp4_swiglu, (long long)M);
  return call(grouped_swiglu(false, 1, a, w_gate_up, scales, offsets, counts, E, I, K, M, h,
                             stream));
}

gnf4_status gnf4_grouped_gemv_nf4_swiglu(const void* a, const uint8_t* w_gate_up, const float* absmax,
                                         const int32_t* offsets, const int32_t* counts, int E, int I, int K, int M,
                                         void* h, void* stream) {
  CallScope call(Entry::grouped_gemv_nf4_swiglu, (long long)M);
  return call(grouped_swiglu(true, 0, a, w_gate_up, absmax, offsets, counts, E, I, K, M, h,
                             stream));
}

gnf4_status gnf4_grouped_gemv_mxfp4_swiglu(const void* a, const uint8_t* w_gate_up, const uint8_t* scales,
                                           const int32_t* offsets, const int32_t* counts, int E, int I, int K, int M,
                                           void* h, void* stream) {
  CallScope call(Entry::grouped_gemv_mxfp4_swiglu, (long long)M);
  return call(grouped_swiglu(true, 1, a, w_gate_up, scales, offsets, counts, E, I, K, M, h,
                             stream));
}

}  // extern "C"
