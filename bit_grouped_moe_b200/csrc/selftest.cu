// selftest.cu -- exercises the failure-detection path of the pipelines'
// bounded waits without a GPU fault.
//
// Every mbarrier wait in the GEMM / GEMV / dgrad pipelines gives up after a
// cycle limit, raises GNF4_DEVERR_TIMEOUT in the device error word and lets
// the kernel return.  This kernel runs that same wait on a barrier nothing
// ever arrives on, with a short limit chosen by the caller, so a test can see
// the status appear and the context stay usable.
#include "common.cuh"
#include "internal.h"

namespace gnf4 {
namespace {

__global__ void bounded_wait_probe_kernel(unsigned* err, long long limit_cycles) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // expects one arrival; none is ever made
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_for(&bar, 0, err, &abort_flag, limit_cycles);
}

}  // namespace

cudaError_t launch_bounded_wait_probe(unsigned* err, long long limit_cycles, cudaStream_t stream) {
  bounded_wait_probe_kernel<<<1, 32, 0, stream>>>(err, limit_cycles);
  return cudaGetLastError();
}

}  // namespace gnf4
