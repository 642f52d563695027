// gemv.cu -- grouped 4-bit expert GEMV for decode (at most 8 rows per group).
//
// Decode steps are bandwidth-bound: the weights of the routed experts are the
// bytes that must stream from HBM (grouped-nf4-gemm index.json,
// problems_solved[2]).  The pages' decode GEMV re-streams the weights once per
// row (same page, limitations); here every weight byte is read once and used
// for all of its group's rows.
//
// Work unit = one warp x (expert e, 16 consecutive weight rows, all of K).
// The warp streams its 16 rows with 8-byte loads (each 32-byte sector of a
// row is fully used by 4 lanes), decodes every packed byte with a lookup in
// a lane-private copy of the pair table (two bf16 codes per byte), and feeds
// the bf16 codes straight into m16n8k16 warp MMAs whose 8 columns are the
// group's (<= 8) activation rows.  The MMA does the k-reduction that a
// CUDA-core GEMV would do with warp shuffles.
//   * NF4: codes enter the MMA unscaled; each 64-k block is accumulated on
//     its own and folded in with its fp32 absmax (exact fp32 scaling).
//   * MXFP4: codes are scaled by their power of two in bf16 before the MMA
//     (exact), so the whole K accumulates in one fragment.
// Lane (g, t) = (lane / 4, lane % 4) owns weight rows g and g+8 of the warp's
// 16 and, within every 64-k chunk, the 16 consecutive k in [16t, 16t+16).
// The MMA's k index is a permutation of these physical k; the activation
// fragment uses the same permutation, so the contraction is unchanged.
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace gnf4 {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRowsPerWarp = 16;
constexpr int kMaxRows = 8;
constexpr int kUnroll = 4;  // 64-k chunks whose loads are issued together

struct GemvSmem {
  uint32_t lut[kLutWords];
  int off[kMaxExperts + 1];
  int upre[kMaxExperts + 1];
  int scratch[kMaxExperts];
};

template <int FMT>
__global__ void __launch_bounds__(kThreads, 2) gemv_kernel(GroupedArgs p) {
  extern __shared__ uint8_t smem_raw[];
  GemvSmem& s = *reinterpret_cast<GemvSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;

  if (!load_groups(p.offsets, p.counts, p.E, p.M, s.off, s.scratch, p.err)) return;
  const int nsl = (p.N + kRowsPerWarp - 1) / kRowsPerWarp;
  block_exclusive_scan(p.E, s.upre, s.scratch, [&](int e) { return (s.off[e + 1] > s.off[e]) ? nsl : 0; });
  const int U = s.upre[p.E];
  if ((int)blockIdx.x * kWarps >= U) return;
  build_pair_lut<FMT>(s.lut, tid, kThreads);
  __syncthreads();

  const uint32_t lut_lane = smem_u32(s.lut) + (uint32_t)lane * 4u;
  const int K = p.K;
  const int nchunk = (K + 63) / 64;
  const size_t row_bytes = (size_t)K / 2;

  for (int u = blockIdx.x * kWarps + warp; u < U; u += gridDim.x * kWarps) {
    const int e = find_group(s.upre, p.E, u);
    const int sl = u - s.upre[e];
    const int r0 = s.off[e], rows = s.off[e + 1] - r0;
    if (rows > kMaxRows) {
      if (lane == 0 && sl == 0) atomicOr(p.err, GNF4_DEVERR_GEMV_ROWS);
      continue;
    }
    const int nA = sl * kRowsPerWarp + g, nB = nA + 8;
    const bool vA = nA < p.N, vB = nB < p.N, vT = g < rows;
    const uint8_t* wA = p.w + ((size_t)e * p.N + (vA ? nA : 0)) * row_bytes + 8 * t;
    const uint8_t* wB = p.w + ((size_t)e * p.N + (vB ? nB : 0)) * row_bytes + 8 * t;
    const __nv_bfloat16* xr = p.a + (size_t)(r0 + (vT ? g : 0)) * K + 16 * t;
    const size_t sA = ((size_t)e * p.N + (vA ? nA : 0)), sB = ((size_t)e * p.N + (vB ? nB : 0));

    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int c0 = 0; c0 < nchunk; c0 += kUnroll) {
      uint2 qa[kUnroll], qb[kUnroll];
      uint4 xa[kUnroll], xb[kUnroll];
      uint32_t sa[kUnroll], sb[kUnroll];
#pragma unroll
      for (int d = 0; d < kUnroll; ++d) {
        const int c = c0 + d;
        const bool inK = (c < nchunk) && (c * 64 + 16 * t < K);
        qa[d] = (inK && vA) ? ldg_nc_u64(wA + (size_t)c * 32) : make_uint2(0u, 0u);
        qb[d] = (inK && vB) ? ldg_nc_u64(wB + (size_t)c * 32) : make_uint2(0u, 0u);
        if (inK && vT) {
          xa[d] = ldg_u128(xr + (size_t)c * 64);
          xb[d] = ldg_u128(xr + (size_t)c * 64 + 8);
        } else {
          xa[d] = make_uint4(0u, 0u, 0u, 0u);
          xb[d] = make_uint4(0u, 0u, 0u, 0u);
        }
        if (FMT == 0) {
          const float* am = reinterpret_cast<const float*>(p.scales);
          sa[d] = (inK && vA) ? __float_as_uint(__ldg(am + sA * (size_t)(K / 64) + c)) : 0u;
          sb[d] = (inK && vB) ? __float_as_uint(__ldg(am + sB * (size_t)(K / 64) + c)) : 0u;
        } else {
          const uint8_t* sc = reinterpret_cast<const uint8_t*>(p.scales);
          const int blk = 2 * c + (t >> 1);
          sa[d] = (inK && vA) ? e8m0_to_bf16x2(__ldg(sc + sA * (size_t)(K / 32) + blk)) : 0u;
          sb[d] = (inK && vB) ? e8m0_to_bf16x2(__ldg(sc + sB * (size_t)(K / 32) + blk)) : 0u;
        }
      }
#pragma unroll
      for (int d = 0; d < kUnroll; ++d) {
        if (c0 + d >= nchunk) break;
        uint32_t pa[8], pb[8];
        const uint32_t wa[2] = {qa[d].x, qa[d].y}, wb[2] = {qb[d].x, qb[d].y};
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          pa[4 * i + 0] = lds_u32(lut_lane + ((wa[i] << 7) & 0x7F80u));
          pa[4 * i + 1] = lds_u32(lut_lane + ((wa[i] >> 1) & 0x7F80u));
          pa[4 * i + 2] = lds_u32(lut_lane + ((wa[i] >> 9) & 0x7F80u));
          pa[4 * i + 3] = lds_u32(lut_lane + ((wa[i] >> 17) & 0x7F80u));
          pb[4 * i + 0] = lds_u32(lut_lane + ((wb[i] << 7) & 0x7F80u));
          pb[4 * i + 1] = lds_u32(lut_lane + ((wb[i] >> 1) & 0x7F80u));
          pb[4 * i + 2] = lds_u32(lut_lane + ((wb[i] >> 9) & 0x7F80u));
          pb[4 * i + 3] = lds_u32(lut_lane + ((wb[i] >> 17) & 0x7F80u));
        }
        const uint32_t xv[8] = {xa[d].x, xa[d].y, xa[d].z, xa[d].w, xb[d].x, xb[d].y, xb[d].z, xb[d].w};
        if (FMT == 0) {
          float blk[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_bf16_16816(blk, pa[2 * j], pb[2 * j], pa[2 * j + 1], pb[2 * j + 1], xv[2 * j], xv[2 * j + 1]);
          const float amA = __uint_as_float(sa[d]), amB = __uint_as_float(sb[d]);
          acc[0] = fmaf(blk[0], amA, acc[0]);
          acc[1] = fmaf(blk[1], amA, acc[1]);
          acc[2] = fmaf(blk[2], amB, acc[2]);
          acc[3] = fmaf(blk[3], amB, acc[3]);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            pa[i] = bf16x2_mul(pa[i], sa[d]);
            pb[i] = bf16x2_mul(pb[i], sb[d]);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_bf16_16816(acc, pa[2 * j], pb[2 * j], pa[2 * j + 1], pb[2 * j + 1], xv[2 * j], xv[2 * j + 1]);
        }
      }
    }
    // acc[0..1]: weight row nA, tokens 2t, 2t+1; acc[2..3]: row nB.
    const int t0 = 2 * t, t1 = 2 * t + 1;
    if (vA) {
      if (t0 < rows) p.y[(size_t)(r0 + t0) * p.N + nA] = __float2bfloat16_rn(acc[0]);
      if (t1 < rows) p.y[(size_t)(r0 + t1) * p.N + nA] = __float2bfloat16_rn(acc[1]);
    }
    if (vB) {
      if (t0 < rows) p.y[(size_t)(r0 + t0) * p.N + nB] = __float2bfloat16_rn(acc[2]);
      if (t1 < rows) p.y[(size_t)(r0 + t1) * p.N + nB] = __float2bfloat16_rn(acc[3]);
    }
  }
}

}  // namespace

int gemv_warps_per_block() { return kWarps; }
int gemv_rows_per_warp() { return kRowsPerWarp; }

template <int FMT>
static cudaError_t launch_gemv_t(const GroupedArgs& p, int grid, cudaStream_t stream) {
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemv_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sizeof(GemvSmem));
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  gemv_kernel<FMT><<<grid, kThreads, sizeof(GemvSmem), stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gemv(int fmt, const GroupedArgs& p, int grid, cudaStream_t stream) {
  return fmt == 0 ? launch_gemv_t<0>(p, grid, stream) : launch_gemv_t<1>(p, grid, stream);
}

}  // namespace gnf4
