// internal.h -- launchers shared between the C-ABI layer and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <cuda_bf16.h>

#include <atomic>
#include <utility>

#include "gnf4.h"

namespace gnf4 {

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel of the stream is still finishing.  Every kernel
// launched this way executes griddep_wait() (common.cuh) before it reads or
// writes any global memory that earlier work in the stream uses.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Raises a kernel's dynamic shared-memory limit to `bytes`, once per device
// (`done` is the kernel's flag array; a racing second call is harmless, and
// devices past 64 set the attribute on every call).
template <typename Kernel>
cudaError_t set_smem_limit_once(Kernel kernel, int bytes, std::atomic<bool> (&done)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool tracked = dev >= 0 && dev < 64;
  if (tracked && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && tracked) done[dev].store(true, std::memory_order_release);
  return e;
}

// Arguments of the grouped GEMM / GEMV kernels (device pointers).
struct GroupedArgs {
  const __nv_bfloat16* a;  // [M, K]
  const uint8_t* w;        // [E, N, K/2]
  const void* scales;      // absmax fp32 [E, N, K/64] or e8m0 [E, N, K/32]
  const int* offsets;      // [E+1] or null
  const int* counts;       // [E] or null
  __nv_bfloat16* y;        // [M, N]
  unsigned* err;           // device error word
  int E, N, K, M;
  int min_rows = 0;  // tcgen05 GEMM: groups with fewer rows are left to another kernel (rows of y not written)
};

// gemm_tc.cu
size_t gemm_tc_smem_bytes();
int gemm_tc_rows_per_unit();         // token rows per unit
int gemm_tc_weight_rows_per_unit();  // weight rows per unit (a CTA pair)
int gemm_tc_weight_box_rows();       // weight rows per CTA (tm_w box)
int gemm_tc_grid(long long units, int num_sms);  // CTAs (whole pairs) for `units` units
int gemm_tc_out_box_rows();          // tokens per output store (tm_y box rows)
int gemm_tc_small_box_rows();  // activation rows per box for groups of at most this many rows (tm_a)
int gemm_tc_big_box_rows();    // activation rows per box otherwise (tm_a_big)
// swiglu: p.w is a gate_up stack [E, N = 2I, K/2] (tm_w its 5-D gate/up view) and p.y the [M, I] output h.
// tm_y: the output [M, N] (SwiGLU: [M, I]) bf16 in boxes of 128 (SwiGLU: 64) columns x gemm_tc_out_box_rows() rows.
struct CombineArgs;
// combine (not with swiglu): also out[t] = sum_j w[t,j] y[f2s[t*k+j]] after each unit (counters per 128 columns).
cudaError_t launch_gemm_tc(int fmt, bool swiglu, const CUtensorMap& tm_a, const CUtensorMap& tm_a_big,
                           const CUtensorMap& tm_w, const CUtensorMap& tm_y, const GroupedArgs& p, int grid,
                           cudaStream_t stream, const CombineArgs* combine = nullptr);

// Fused top-k combine in the GEMV / GEMM epilogue (device pointers).
struct CombineArgs {
  const int* s2f;     // sorted_to_flat [M]
  const int* f2s;     // flat_to_sorted [T*k]
  const float* w;     // weights [T, k]
  __nv_bfloat16* out; // [T, N]
  int* cnt;           // [T, ceil(N/64)] counters (the GEMM uses [T, ceil(N/128)]), zero before and after a call
  int T, k;
};

// gemv.cu
// swiglu: p.w is a gate_up stack [E, N = 2I, K/2] and p.y the [M, I] output h.
// combine (not with swiglu): also out[t] = sum_j w[t,j] y[f2s[t*k+j]] in the epilogue.
cudaError_t launch_gemv(int fmt, bool swiglu, const GroupedArgs& p, int grid, cudaStream_t stream,
                        const CombineArgs* combine = nullptr);
size_t gemv_combine_counter_bytes(int T, int N);
int gemv_rows_per_block();
int gemv_swiglu_cols_per_block();
// CTAs for a GEMV launch over `units` (expert, 64-row) units.
int gemv_grid(long long units, int num_sms);

// dgrad.cu: p.w is the [E, N, K/2] stack, p.a = dY [M, N], p.y = dX [M, K]
cudaError_t launch_dgrad_tc(int fmt, const CUtensorMap& tm_y, const CUtensorMap& tm_w, const GroupedArgs& p,
                            int grid, cudaStream_t stream);
size_t dgrad_tc_smem_bytes();
int dgrad_tc_rows_per_unit();
int dgrad_tc_k_per_unit();
int dgrad_tc_n_per_stage();

// mx.cu: native block-scaled MXFP4 modes.  mode 0 = W4A8 (MXFP8 activations,
// kind::mxf8f6f4), 1 = two-term MXFP8 (hi + lo), 2 = W4A4 (MXFP4 activations,
// kind::mxf4).
// lo_codes / lo_scales non-null: the two-term split (hi into codes / scales)
cudaError_t launch_quant_mxfp8(const __nv_bfloat16* x, long long elems, uint8_t* codes, uint8_t* scales,
                               uint8_t* lo_codes, uint8_t* lo_scales, cudaStream_t stream);
cudaError_t launch_quant_mxfp4_act(const __nv_bfloat16* x, long long elems, uint8_t* blocks, uint8_t* scales,
                                   cudaStream_t stream);
// Modes 0 / 2: tm_a / tm_a_big = the activation codes in 32- / 128-row boxes of 128 bytes; mode 1: tm_a = hi
// codes, tm_a_big = lo codes, both in 32-row boxes.  tm_w: modes 0 / 1 the [E*N] x (K/128) x 128-code view of
// the e2m1 stack in 16-byte slots, tm_w_tail its codes [K-128, K) (K % 128 == 64); mode 2 the [E, N, K/2] bytes
// in 128-byte x 128-row boxes.
cudaError_t launch_gemm_mx(int mode, const CUtensorMap& tm_a, const CUtensorMap& tm_a_big, const CUtensorMap& tm_w,
                           const CUtensorMap& tm_w_tail, const uint8_t* a_scales, const uint8_t* lo_scales,
                           const uint8_t* w_scales, const int* offsets, const int* counts, __nv_bfloat16* y,
                           unsigned* err, int E, int N, int K, int M, int grid, cudaStream_t stream,
                           int max_rows = 1 << 30);  // groups of more rows are skipped (rows of y not written)
// The two-term split of the rows of the groups with at most max_rows rows only (other rows not written);
// offsets / counts as the grouped GEMM.  Persistent grid of num_sms * 8 CTAs.
cudaError_t launch_quant_mxfp8_split_rows(const __nv_bfloat16* x, int K, const int* offsets, const int* counts,
                                          int E, int M, int max_rows, unsigned* err, uint8_t* hi_codes,
                                          uint8_t* hi_scales, uint8_t* lo_codes, uint8_t* lo_scales, int num_sms,
                                          cudaStream_t stream);
size_t gemm_mx_smem_bytes(int mode);
int gemm_mx_rows_per_unit(int mode);
int gemm_mx_k_per_stage(int mode);
int gemm_mx_weight_rows_per_unit();
int gemm_mx_small_box_rows();

// route.cu
size_t route_workspace_bytes(int T, int k, int E);
cudaError_t launch_route(const int32_t* topk_ids, const __nv_bfloat16* x, int T, int k, int E, int K,
                         int32_t* offsets, int32_t* sorted_to_flat, int32_t* flat_to_sorted,
                         __nv_bfloat16* x_sorted, void* workspace, int32_t* bad_id_count, int num_sms,
                         cudaStream_t stream);

// Router epilogue (top-k of logits + bias, softmax weights) followed by the routing above.
cudaError_t launch_route_topk(const float* logits, const float* bias, int T, int E, int k, const __nv_bfloat16* x,
                              int K, int32_t* topk_ids, float* topk_weights, int32_t* offsets,
                              int32_t* sorted_to_flat, int32_t* flat_to_sorted, __nv_bfloat16* x_sorted,
                              void* workspace, int num_sms, cudaStream_t stream);
constexpr int kMaxRouterTopK = 32;

// combine.cu
cudaError_t launch_combine(const __nv_bfloat16* y, const int32_t* flat_to_sorted, const float* weights, int T,
                           int k, int N, __nv_bfloat16* out, int num_sms, cudaStream_t stream);

// selftest.cu: one bounded wait on a barrier nothing arrives on
cudaError_t launch_bounded_wait_probe(unsigned* err, long long limit_cycles, cudaStream_t stream);

// api.cu: sets the text gnf4_last_error() returns on this thread
void set_last_error(const char* msg);

// api.cu: engagement counters, one record per entry point that enqueues work.
#define GNF4_COUNTED_ENTRIES(X)                                                                              \
  X(route_permute) X(route_permute_static) X(route_topk_permute) X(grouped_gemm_nf4) X(grouped_gemm_mxfp4) \
  X(grouped_gemm_mxfp4_ws) X(grouped_gemv_nf4) X(grouped_gemv_mxfp4) X(grouped_dgrad_nf4)                \
  X(grouped_dgrad_mxfp4) X(grouped_gemm_nf4_swiglu) X(grouped_gemm_mxfp4_swiglu)                          \
  X(grouped_gemv_nf4_swiglu) X(grouped_gemv_mxfp4_swiglu) X(grouped_gemv_nf4_combine)                     \
  X(grouped_gemv_mxfp4_combine) X(grouped_gemm_nf4_combine) X(grouped_gemm_mxfp4_combine)                 \
  X(quantize_mxfp8) X(quantize_mxfp8_split) X(quantize_mxfp4_act) X(grouped_gemm_w4a8)                    \
  X(grouped_gemm_w4a8x2) X(grouped_gemm_w4a4) X(combine) X(dequant_nf4_f32) X(dequant_mxfp4_f32)

enum class Entry : int {
#define GNF4_ENTRY_ENUM(n) n,
  GNF4_COUNTED_ENTRIES(GNF4_ENTRY_ENUM)
#undef GNF4_ENTRY_ENUM
      count
};

// Kernel families a call can launch (the counters' *_path fields).
enum : unsigned { kPathDecode = 1u, kPathNative = 2u, kPathGemv = 4u, kPathOther = 8u };

// One counted call: the outermost scope on a thread records it when the
// status passes through operator(); nested scopes (an entry point called by
// another) record nothing of their own.
class CallScope {
 public:
  CallScope(Entry e, long long rows);
  ~CallScope();
  gnf4_status operator()(gnf4_status s);
  CallScope(const CallScope&) = delete;
  CallScope& operator=(const CallScope&) = delete;

 private:
  Entry entry_;
  long long rows_;
  bool outer_;
};

// Marks that the current call enqueued work of the given family.
void note_launch(unsigned path);

// dequant.cu
cudaError_t launch_dequant(int fmt, const uint8_t* w, const void* scales, int64_t rows, int K, float* out,
                           int num_sms, cudaStream_t stream);

}  // namespace gnf4
