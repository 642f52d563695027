// dequant.cu -- fp32 decode of packed rows (test support: the bit-exact check
// of the decode that the pages' dequant_ref performs; grouped-nf4-gemm 0.33.1
// on PyPI, "Try it on CPU right now", examples 1 and 2).
//   NF4:   out[r, k] = NF4[code] * absmax[r, k/64]   (element 2i = high nibble)
//   MXFP4: out[r, k] = e2m1[code] * 2^(s[r, k/32]-127) (element 2i = low nibble)
// One IEEE fp32 multiply per element, round to nearest, subnormals kept.
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace gnf4 {
namespace {

template <int FMT>
__global__ void __launch_bounds__(256) dequant_kernel(const uint8_t* w, const void* scales, int64_t rows, int K,
                                                      float* out) {
  const int64_t nbytes = rows * (int64_t)(K / 2);
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nbytes; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = i / (K / 2);
    const int kb = (int)(i - r * (K / 2));  // byte within the row: elements 2kb, 2kb+1
    const uint32_t b = w[i];
    float v0, v1;
    if (FMT == 0) {
      const float am = reinterpret_cast<const float*>(scales)[r * (K / 64) + (2 * kb) / 64];
      v0 = __fmul_rn(kNf4Code[b >> 4], am);
      v1 = __fmul_rn(kNf4Code[b & 15u], am);
    } else {
      const float sc = e8m0_to_f32(reinterpret_cast<const uint8_t*>(scales)[r * (K / 32) + (2 * kb) / 32]);
      v0 = __fmul_rn(e2m1_value(b & 15u), sc);
      v1 = __fmul_rn(e2m1_value(b >> 4), sc);
    }
    reinterpret_cast<float2*>(out)[i] = make_float2(v0, v1);
  }
}

}  // namespace

cudaError_t launch_dequant(int fmt, const uint8_t* w, const void* scales, int64_t rows, int K, float* out,
                           int num_sms, cudaStream_t stream) {
  const int64_t nbytes = rows * (int64_t)(K / 2);
  if (nbytes == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t want = (nbytes + threads - 1) / threads;
  const int grid = (int)(want < (int64_t)num_sms * 16 ? want : (int64_t)num_sms * 16);
  if (fmt == 0)
    dequant_kernel<0><<<grid, threads, 0, stream>>>(w, scales, rows, K, out);
  else
    dequant_kernel<1><<<grid, threads, 0, stream>>>(w, scales, rows, K, out);
  return cudaGetLastError();
}

}  // namespace gnf4
