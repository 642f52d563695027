// combine.cu -- top-k weighted scatter of expert outputs back to tokens
// (grouped-nf4-gemm index.json, problems_solved[5] "top-k combine";
// releases v0.2.6: the caller's "weighting, unsorting").
//   out[t, n] = sum_{j<k} weights[t, j] * y[flat_to_sorted[t*k + j], n]
// fp32 sum in order j = 0..k-1, one bf16 rounding at the end.  One thread
// produces 8 consecutive outputs of a token with 16-byte loads and stores.
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace gnf4 {
namespace {

__global__ void __launch_bounds__(256) combine_kernel(const uint4* y, const int32_t* f2s, const float* w, int T,
                                                      int k, int N8, uint4* out) {
  griddep_launch_dependents();
  griddep_wait();
  const int rows_y = T * k;
  const size_t total = (size_t)T * N8;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)(i / N8);
    const int v = (int)(i - (size_t)t * N8);
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < k; ++j) {
      const int p = __ldg(f2s + (size_t)t * k + j);
      if (p < 0 || p >= rows_y) continue;  // dropped pair (or out of range)
      const float wj = __ldg(w + (size_t)t * k + j);
      const uint4 q = __ldg(y + (size_t)p * N8 + v);
      const uint32_t qq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        acc[2 * h] = fmaf(wj, __uint_as_float(qq[h] << 16), acc[2 * h]);
        acc[2 * h + 1] = fmaf(wj, __uint_as_float(qq[h] & 0xFFFF0000u), acc[2 * h + 1]);
      }
    }
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * h], acc[2 * h + 1]);
      o[h] = *reinterpret_cast<uint32_t*>(&b);
    }
    out[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

}  // namespace

cudaError_t launch_combine(const __nv_bfloat16* y, const int32_t* flat_to_sorted, const float* weights, int T,
                           int k, int N, __nv_bfloat16* out, int num_sms, cudaStream_t stream) {
  const int N8 = N / 8;
  const size_t total = (size_t)T * N8;
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  const size_t want = (total + threads - 1) / threads;
  const int grid = (int)(want < (size_t)num_sms * 16 ? want : (size_t)num_sms * 16);
  return launch_pdl(combine_kernel, dim3(grid), dim3(threads), 0, stream, reinterpret_cast<const uint4*>(y),
                    flat_to_sorted, weights, T, k, N8, reinterpret_cast<uint4*>(out));
}

}  // namespace gnf4
