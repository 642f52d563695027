// route_static.cu -- gnf4_route_permute_static: the routing call for callers
// that cannot allocate device memory.
//
// Some callers are not allowed to allocate: a plugin running inside an
// inference engine whose device memory is budgeted and owned by the host
// process, or latency-critical code that must not pay for cudaMalloc's
// implicit device synchronisation.  For them this entry point runs the same
// routing as gnf4_route_permute with its scratch in a fixed array that is
// part of the library image on every GPU that loads libgnf4.
//
// The array's name means something different on each side: device code may
// name it directly, but in host code it is only a host-side stand-in for the
// symbol, not a device address.  The device address is obtained once per
// device with cudaGetSymbolAddress and passed to the kernels as a plain
// pointer.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "gnf4.h"
#include "internal.h"

namespace gnf4 {
namespace {

constexpr size_t kStaticRouteScratchBytes = GNF4_ROUTE_STATIC_SCRATCH_BYTES;

// Scratch of the allocation-free routing call, one copy per device, held
// for the life of the process.
static __device__ __align__(256) unsigned char g_route_scratch[kStaticRouteScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

}  // namespace
}  // namespace gnf4

static gnf4_status route_permute_static_impl(const int32_t* topk_ids, const void* x, int T, int k, int E,
                                             int K, int32_t* offsets, int32_t* sorted_to_flat,
                                             int32_t* flat_to_sorted, void* x_sorted, int32_t* bad_id_count,
                                             void* stream) {
  using namespace gnf4;
  // the size check needs no device
  if (T >= 0 && k >= 1 && E >= 1) {
    const size_t need = gnf4_route_workspace_bytes(T, k, E);
    if (need > kStaticRouteScratchBytes) {
      char msg[256];
      snprintf(msg, sizeof(msg),
               "gnf4_route_permute_static: T=%d, k=%d, E=%d need %zu scratch bytes, more than the %zu-byte "
               "static array; use gnf4_route_permute with a caller-provided workspace",
               T, k, E, need, kStaticRouteScratchBytes);
      set_last_error(msg);
      return GNF4_ERR_UNSUPPORTED_SHAPE;
    }
  }
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    char msg[256];
    snprintf(msg, sizeof(msg), "gnf4_route_permute_static: no usable current device (%s)", cudaGetErrorString(e));
    set_last_error(msg);
    return GNF4_ERR_CUDA;
  }
  void* scratch = nullptr;
  {
    // set-up on the first call on this device, with this device current
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (g_scratch_ptr[dev] == nullptr) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_route_scratch);
      if (e != cudaSuccess || p == nullptr) {
        char msg[256];
        snprintf(msg, sizeof(msg), "gnf4_route_permute_static: cudaGetSymbolAddress failed (%s)",
                 cudaGetErrorString(e));
        set_last_error(msg);
        return GNF4_ERR_CUDA;
      }
      g_scratch_ptr[dev] = p;
    }
    scratch = g_scratch_ptr[dev];
  }
  // Nothing in the scratch has to start at zero: the routing kernels write
  // every word they later read.
  return gnf4_route_permute(topk_ids, x, T, k, E, K, offsets, sorted_to_flat, flat_to_sorted, x_sorted, scratch,
                            kStaticRouteScratchBytes, bad_id_count, stream);
}

extern "C" gnf4_status gnf4_route_permute_static(const int32_t* topk_ids, const void* x, int T, int k, int E,
                                                 int K, int32_t* offsets, int32_t* sorted_to_flat,
                                                 int32_t* flat_to_sorted, void* x_sorted, int32_t* bad_id_count,
                                                 void* stream) {
  gnf4::CallScope call(gnf4::Entry::route_permute_static, (long long)T * k);
  return call(route_permute_static_impl(topk_ids, x, T, k, E, K, offsets, sorted_to_flat, flat_to_sorted, x_sorted,
                                        bad_id_count, stream));
}
