// route.cu -- sort (token, slot) pairs into per-expert row groups and gather
// the activations (grouped-nf4-gemm releases, v0.2.6 "The patch point": the
// argsort of the top-k ids, the gather x[idxs // k] and tokens_per_expert).
//
// A stable counting sort in four short launches, with no host sync and no
// atomics on global memory:
//   1. hist:    each 256-pair chunk counts its pairs per expert (shared
//               memory) and writes the counts row hist[chunk][0..E);
//   2. scan:    one block turns hist into each chunk's first output row per
//               expert and writes offsets[0..E] and the dropped-id count;
//   3. scatter: each chunk ranks its pairs within an expert in flat order
//               (warp match + running per-expert counters, warps in order),
//               giving sorted_to_flat / flat_to_sorted;
//   4. gather:  x_sorted[r] = x[sorted_to_flat[r] / k] with 16-byte copies;
//               rows past offsets[E] are zeroed.
// Ids outside [0, E) are counted and dropped, never used as an index
// (releases v0.3.0, "Also": model-global ids read out of bounds silently).
//
// Decode-sized calls (at most 256 pairs) take a single launch instead: every
// block repeats the whole (tiny) sort in shared memory, block 0 writes the
// routing outputs and all blocks share the gather.  Same results, bit for bit.
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace gnf4 {
namespace {

constexpr int kChunk = 256;  // pairs per histogram chunk
constexpr int kMaxRouteExperts = 4096;

__global__ void __launch_bounds__(kChunk) route_hist_kernel(const int32_t* ids, int M, int E, int32_t* hist,
                                                            int32_t* badc) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ int cnt[kMaxRouteExperts];
  __shared__ int nbad;
  const int tid = threadIdx.x, c = blockIdx.x;
  for (int i = tid; i < E; i += kChunk) cnt[i] = 0;
  if (tid == 0) nbad = 0;
  __syncthreads();
  const int f = c * kChunk + tid;
  if (f < M) {
    const int e = ids[f];
    if (e >= 0 && e < E)
      atomicAdd(&cnt[e], 1);
    else
      atomicAdd(&nbad, 1);
  }
  __syncthreads();
  for (int i = tid; i < E; i += kChunk) hist[(size_t)c * E + i] = cnt[i];
  if (tid == 0) badc[c] = nbad;
}

__global__ void __launch_bounds__(1024) route_scan_kernel(int32_t* hist, const int32_t* badc, int nchunk, int E,
                                                          int32_t* offsets, int32_t* bad_out) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ int tot[kMaxRouteExperts];
  __shared__ int wsum[32];
  const int tid = threadIdx.x;
  // per expert: running count over chunks (coalesced across experts)
  for (int e = tid; e < E; e += blockDim.x) {
    int run = 0;
    for (int c = 0; c < nchunk; ++c) {
      const int v = hist[(size_t)c * E + e];
      hist[(size_t)c * E + e] = run;
      run += v;
    }
    tot[e] = run;
  }
  __syncthreads();
  // exclusive scan of tot over experts: each thread takes a contiguous slice
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int lo = min(E, tid * per), hi = min(E, lo + per);
  int mine = 0;
  for (int e = lo; e < hi; ++e) mine += tot[e];
  // block-wide exclusive scan of `mine`
  const int lane = tid & 31, wid = tid >> 5;
  int incl = mine;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += v;
  }
  if (lane == 31) wsum[wid] = incl;
  __syncthreads();
  if (wid == 0) {
    int w = (lane < (int)(blockDim.x >> 5)) ? wsum[lane] : 0;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, w, d);
      if (lane >= d) w += v;
    }
    wsum[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  int base = incl - mine + (wid > 0 ? wsum[wid - 1] : 0);
  for (int e = lo; e < hi; ++e) {
    const int t = tot[e];
    tot[e] = base;  // now the exclusive prefix
    base += t;
  }
  // the owner of the last expert ends with the number of valid pairs
  if (lo < hi && hi == E) offsets[E] = base;
  __syncthreads();
  for (int e = tid; e < E; e += blockDim.x) offsets[e] = tot[e];
  if (tid == 0 && bad_out != nullptr) {
    int bad = 0;
    for (int c = 0; c < nchunk; ++c) bad += badc[c];
    *bad_out = bad;
  }
  // chunk bases: hist[c][e] += offsets[e]
  for (size_t i = tid; i < (size_t)nchunk * E; i += blockDim.x) hist[i] += tot[i % E];
}

__global__ void __launch_bounds__(kChunk) route_scatter_kernel(const int32_t* ids, int M, int E,
                                                               const int32_t* hist, int32_t* s2f,
                                                               int32_t* f2s) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ int run[kMaxRouteExperts];
  const int tid = threadIdx.x, c = blockIdx.x, lane = tid & 31, wid = tid >> 5;
  for (int i = tid; i < E; i += kChunk) run[i] = 0;
  __syncthreads();
  const int f = c * kChunk + tid;
  const int e = (f < M) ? ids[f] : -1;
  const bool valid = (f < M) && e >= 0 && e < E;
  const unsigned lt = (1u << lane) - 1u;
  int pos = -1;
  for (int w = 0; w < kChunk / 32; ++w) {
    if (wid == w) {
      const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
      const int before = valid ? run[e] : 0;
      __syncwarp();
      if (valid) {
        pos = hist[(size_t)c * E + e] + before + __popc(peers & lt);
        if ((peers & lt) == 0u) run[e] = before + __popc(peers);  // lowest lane of the peer set
      }
    }
    __syncthreads();
  }
  if (f < M) {
    f2s[f] = valid ? pos : -1;
    if (valid) s2f[pos] = f;
  }
}

__global__ void route_gather_kernel(const uint4* x, int K8, int k, const int32_t* offsets, int E, int M,
                                    int32_t* s2f, uint4* xs) {
  griddep_launch_dependents();
  griddep_wait();
  const int nvalid = offsets[E];
  const size_t total = (size_t)M * K8;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(i / K8);
    const int v = (int)(i - (size_t)r * K8);
    if (r < nvalid) {
      const int f = s2f[r];
      // a pair index outside [0, M) would mean a broken permutation: never
      // dereference it, write zeros instead
      xs[i] = (f >= 0 && f < M) ? x[(size_t)(f / k) * K8 + v] : make_uint4(0u, 0u, 0u, 0u);
    } else {
      xs[i] = make_uint4(0u, 0u, 0u, 0u);
      if (v == 0) s2f[r] = -1;
    }
  }
}


// ---------------------------------------------------------------- router epilogue
// Top-k of score = logit + bias (fp32) per token and the softmax of the
// selected raw logits (grouped-nf4-gemm index.json, problems_solved[5]:
// router softmax and top-k among the decode tail folded into one launch).

// Selection order: NaN scores after every number, larger scores first, ties
// to the lower expert index; an index < 0 is "no candidate".
__device__ __forceinline__ bool sel_before(float a, int ia, float b, int ib) {
  if (ib < 0) return ia >= 0;
  if (ia < 0) return false;
  const bool na = a != a, nb = b != b;
  if (na != nb) return nb;
  if (!na && a != b) return a > b;
  return ia < ib;
}

// One warp, one token: lane j < k ends with the j-th selected expert in
// *id and its weight in *w.  Lane l scans experts l, l+32, ...; the experts
// it has lost to the selection are bits of four words (E <= 4096).
__device__ __forceinline__ void router_warp(const float* row, const float* bias, int E, int k, int lane, int* id,
                                            float* w) {
  uint32_t tk0 = 0u, tk1 = 0u, tk2 = 0u, tk3 = 0u;
  int mine = -1;
  for (int j = 0; j < k; ++j) {
    float bv = 0.f;
    int bi = -1;
    for (int c = 0, e = lane; e < E; ++c, e += 32) {
      const uint32_t word = c < 32 ? tk0 : (c < 64 ? tk1 : (c < 96 ? tk2 : tk3));
      if ((word >> (c & 31)) & 1u) continue;
      const float sc = bias != nullptr ? row[e] + bias[e] : row[e];
      if (sel_before(sc, e, bv, bi)) {
        bv = sc;
        bi = e;
      }
    }
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, bv, d);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, d);
      if (sel_before(ov, oi, bv, bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (bi >= 0 && (bi & 31) == lane) {
      const int c = bi >> 5;
      const uint32_t bit = 1u << (c & 31);
      if (c < 32) tk0 |= bit;
      else if (c < 64) tk1 |= bit;
      else if (c < 96) tk2 |= bit;
      else tk3 |= bit;
    }
    if (lane == j) mine = bi;
  }
  // softmax over the selected raw logits (a NaN logit makes every weight NaN)
  const float l = lane < k ? row[mine] : -INFINITY;
  float m = l;
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) {
    const float o = __shfl_xor_sync(0xffffffffu, m, d);
    if (m == m && (o != o || o > m)) m = o;
  }
  const float ex = lane < k ? expf(l - m) : 0.f;
  float sum = ex;
#pragma unroll
  for (int d = 16; d >= 1; d >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, d);
  *id = mine;
  *w = ex / sum;
}

__global__ void __launch_bounds__(256) router_kernel(const float* logits, const float* bias, int T, int E, int k,
                                                     int32_t* ids, float* weights) {
  griddep_launch_dependents();
  griddep_wait();
  const int t = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (t >= T) return;  // uniform over the warp
  int id;
  float w;
  router_warp(logits + (size_t)t * E, bias, E, k, lane, &id, &w);
  if (lane < k) {
    ids[(size_t)t * k + lane] = id;
    weights[(size_t)t * k + lane] = w;
  }
}

// Single-launch routing for M <= kChunk pairs: each block sorts all pairs in
// shared memory (same counting sort, same ranks), block 0 writes offsets and
// permutations, and block b gathers rows b, b + gridDim.x, ...
// With logits != nullptr the block first runs the router epilogue for all
// T = M / k tokens (ids into shared memory; block 0 also writes ids and
// weights out) and sorts those ids.
__global__ void __launch_bounds__(kChunk) route_small_kernel(const int32_t* ids, int M, int E, const uint4* x,
                                                             int K8, int k, int32_t* offsets, int32_t* s2f,
                                                             int32_t* f2s, int32_t* bad_out, uint4* xs,
                                                             const float* logits, const float* bias,
                                                             int32_t* ids_out, float* w_out) {
  griddep_launch_dependents();
  griddep_wait();
  __shared__ int cnt[kMaxRouteExperts];
  __shared__ int s2f_sm[kChunk];
  __shared__ int ids_sm[kChunk];
  __shared__ int wsum[kChunk / 32];
  __shared__ int nbad, nvalid_sm;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  for (int i = tid; i < E; i += kChunk) cnt[i] = 0;
  if (tid == 0) nbad = 0;
  if (logits != nullptr) {
    for (int t = wid; t * k < M; t += kChunk / 32) {  // uniform over the warp
      int id;
      float w;
      router_warp(logits + (size_t)t * E, bias, E, k, lane, &id, &w);
      if (lane < k) {
        ids_sm[t * k + lane] = id;
        if (blockIdx.x == 0) {
          ids_out[t * k + lane] = id;
          w_out[t * k + lane] = w;
        }
      }
    }
  }
  __syncthreads();
  const int e = (tid < M) ? (logits != nullptr ? ids_sm[tid] : ids[tid]) : -1;
  const bool valid = tid < M && e >= 0 && e < E;
  if (valid) atomicAdd(&cnt[e], 1);
  else if (tid < M) atomicAdd(&nbad, 1);
  __syncthreads();
  // exclusive scan of cnt over experts: each thread a contiguous slice
  const int per = (E + kChunk - 1) / kChunk;
  const int lo = min(E, tid * per), hi = min(E, lo + per);
  int mine = 0;
  for (int i = lo; i < hi; ++i) mine += cnt[i];
  int incl = mine;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += v;
  }
  if (lane == 31) wsum[wid] = incl;
  __syncthreads();
  int base = incl - mine;
  for (int w = 0; w < wid; ++w) base += wsum[w];
  __syncthreads();  // every thread has read its slice of cnt
  for (int i = lo; i < hi; ++i) {
    const int c = cnt[i];
    cnt[i] = base;  // exclusive prefix = first row of expert i
    base += c;
  }
  if (lo < hi && hi == E) nvalid_sm = base;
  if (E == 0 && tid == 0) nvalid_sm = 0;
  __syncthreads();
  // stable rank within the expert: warps in order, lanes by match
  const unsigned lt = (1u << lane) - 1u;
  int pos = -1;
  for (int w = 0; w < kChunk / 32; ++w) {
    if (wid == w) {
      const unsigned peers = __match_any_sync(0xffffffffu, valid ? e : -1);
      const int before = valid ? cnt[e] : 0;
      __syncwarp();
      if (valid) {
        pos = before + __popc(peers & lt);
        if ((peers & lt) == 0u) cnt[e] = before + __popc(peers);
      }
    }
    __syncthreads();
  }
  if (valid) s2f_sm[pos] = tid;
  __syncthreads();
  const int nvalid = nvalid_sm;
  if (blockIdx.x == 0) {
    if (tid < M) {
      f2s[tid] = valid ? pos : -1;
      s2f[tid] = tid < nvalid ? s2f_sm[tid] : -1;
    }
    // offsets: cnt now holds each expert's end row = the next expert's start
    for (int i = tid; i < E; i += kChunk) offsets[i + 1] = cnt[i];
    if (tid == 0) {
      offsets[0] = 0;
      if (bad_out != nullptr) *bad_out = nbad;
    }
  }
  for (int r = blockIdx.x; r < M; r += gridDim.x) {
    uint4* dst = xs + (size_t)r * K8;
    if (r < nvalid) {
      const uint4* src = x + (size_t)(s2f_sm[r] / k) * K8;
      for (int v = tid; v < K8; v += kChunk) dst[v] = src[v];
    } else {
      for (int v = tid; v < K8; v += kChunk) dst[v] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

}  // namespace

size_t route_workspace_bytes(int T, int k, int E) {
  const size_t M = (size_t)T * (size_t)k;
  const size_t nchunk = (M + kChunk - 1) / kChunk;
  size_t b = nchunk * (size_t)E * 4 + nchunk * 4;
  return (b + 255) & ~(size_t)255;
}

cudaError_t launch_route(const int32_t* topk_ids, const __nv_bfloat16* x, int T, int k, int E, int K,
                         int32_t* offsets, int32_t* sorted_to_flat, int32_t* flat_to_sorted,
                         __nv_bfloat16* x_sorted, void* workspace, int32_t* bad_id_count, int num_sms,
                         cudaStream_t stream) {
  const int M = T * k;
  if (M > 0 && M <= kChunk) {
    const int grid = M < 2 * num_sms ? M : 2 * num_sms;
    return launch_pdl(route_small_kernel, dim3(grid), dim3(kChunk), 0, stream, topk_ids, M, E,
                      reinterpret_cast<const uint4*>(x), K / 8, k, offsets, sorted_to_flat, flat_to_sorted,
                      bad_id_count, reinterpret_cast<uint4*>(x_sorted), (const float*)nullptr,
                      (const float*)nullptr, (int32_t*)nullptr, (float*)nullptr);
  }
  const int nchunk = (M + kChunk - 1) / kChunk;
  int32_t* hist = reinterpret_cast<int32_t*>(workspace);
  int32_t* badc = hist + (size_t)nchunk * E;
  if (M > 0) {
    cudaError_t e = launch_pdl(route_hist_kernel, dim3(nchunk), dim3(kChunk), 0, stream, topk_ids, M, E, hist, badc);
    if (e != cudaSuccess) return e;
  }
  {
    cudaError_t e = launch_pdl(route_scan_kernel, dim3(1), dim3(1024), 0, stream, hist, badc, nchunk, E, offsets,
                               bad_id_count);
    if (e != cudaSuccess) return e;
  }
  if (M > 0) {
    cudaError_t e = launch_pdl(route_scatter_kernel, dim3(nchunk), dim3(kChunk), 0, stream, topk_ids, M, E,
                               (const int32_t*)hist, sorted_to_flat, flat_to_sorted);
    if (e != cudaSuccess) return e;
    const int K8 = K / 8;
    const size_t total = (size_t)M * K8;
    const int threads = 256;
    const size_t want = (total + threads - 1) / threads;
    const int grid = (int)(want < (size_t)num_sms * 16 ? want : (size_t)num_sms * 16);
    e = launch_pdl(route_gather_kernel, dim3(grid), dim3(threads), 0, stream, reinterpret_cast<const uint4*>(x), K8,
                   k, (const int32_t*)offsets, E, M, sorted_to_flat, reinterpret_cast<uint4*>(x_sorted));
    if (e != cudaSuccess) return e;
  }
  return cudaGetLastError();
}

cudaError_t launch_route_topk(const float* logits, const float* bias, int T, int E, int k, const __nv_bfloat16* x,
                              int K, int32_t* topk_ids, float* topk_weights, int32_t* offsets,
                              int32_t* sorted_to_flat, int32_t* flat_to_sorted, __nv_bfloat16* x_sorted,
                              void* workspace, int num_sms, cudaStream_t stream) {
  const int M = T * k;
  if (M > 0 && M <= kChunk) {
    const int grid = M < 2 * num_sms ? M : 2 * num_sms;
    return launch_pdl(route_small_kernel, dim3(grid), dim3(kChunk), 0, stream, (const int32_t*)topk_ids, M, E,
                      reinterpret_cast<const uint4*>(x), K / 8, k, offsets, sorted_to_flat, flat_to_sorted,
                      (int32_t*)nullptr, reinterpret_cast<uint4*>(x_sorted), logits, bias, topk_ids, topk_weights);
  }
  if (M > 0) {
    cudaError_t e = launch_pdl(router_kernel, dim3((T + 7) / 8), dim3(256), 0, stream, logits, bias, T, E, k,
                               topk_ids, topk_weights);
    if (e != cudaSuccess) return e;
  }
  return launch_route(topk_ids, x, T, k, E, K, offsets, sorted_to_flat, flat_to_sorted, x_sorted, workspace,
                      nullptr, num_sms, stream);
}

}  // namespace gnf4
