// gemv.cu -- grouped 4-bit expert GEMV for decode (at most 8 rows per group).
//
// Decode steps are bandwidth-bound: the weights of the routed experts are the
// bytes that must stream from HBM (grouped-nf4-gemm index.json,
// problems_solved[2]).  The pages' decode GEMV re-streams the weights once per
// row (same page, limitations); here every weight byte is read once and used
// for all of its group's rows.
//
// Work unit = one CTA x (expert e, 64 consecutive weight rows).  The 8 warps
// split K: warp w takes a contiguous range of 128-k "double chunks" and
// computes the partial sums of all 64 rows (four m16 tiles) for the group's
// <= 8 rows (the MMA's 8 columns); a fixed-order shared-memory reduction over
// the warps finishes the unit.  Per double chunk a lane loads 16 bytes (32
// codes) of each of its 8 weight rows with one 16-byte load each, decodes
// every byte with one PRMT (which builds the table address) and one shared
// load from a lane-private copy of the pair table, multiplies the bf16 pair
// by the row's block scale, and feeds the pairs to m16n8k16 warp MMAs.  The
// MMA does the k reduction that a CUDA-core GEMV would do with shuffles.
//
// Lane (g, t) = (lane / 4, lane % 4) owns rows g and g+8 of every tile and,
// in every double chunk, the 32 consecutive k in [32t, 32t+32) (one NF4
// block, one MXFP4 block).  The MMA's k index is a permutation of these
// physical k; the activation fragment uses the same permutation.
//   * MXFP4: e2m1 x 2^(e-127) is exact in bf16.
//   * NF4: the code is rounded to bf16, then multiplied by bf16(absmax) and
//     rounded again (relative error <= ~3 * 2^-9 per weight); sums are fp32.
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace gnf4 {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kRows = 64;        // weight rows per unit (4 m16 tiles)
constexpr int kMaxTokens = 8;    // rows of a group = MMA columns
constexpr int kDK = 128;         // k per double chunk

struct GemvSmem {
  uint32_t lut[kLut256Words];                 // 64 KB pair table, 256-byte entry stride
  float red[kWarps][4][32][4];                // 16 KB cross-warp partial sums
  int off[kMaxExperts + 1];
  int upre[kMaxExperts + 1];
  int scratch[kMaxExperts];
};

template <int FMT>
__global__ void __launch_bounds__(kThreads, 2) gemv_kernel(GroupedArgs p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  GemvSmem& s = *reinterpret_cast<GemvSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;

  if (!load_groups(p.offsets, p.counts, p.E, p.M, s.off, s.scratch, p.err)) return;
  const int nblk = (p.N + kRows - 1) / kRows;
  block_exclusive_scan(p.E, s.upre, s.scratch, [&](int e) { return (s.off[e + 1] > s.off[e]) ? nblk : 0; });
  const int U = s.upre[p.E];
  if ((int)blockIdx.x >= U) return;
  build_pair_lut256<FMT>(s.lut, tid, kThreads);
  __syncthreads();

  const uint32_t lut = smem_u32(s.lut);
  const uint32_t lane4 = (uint32_t)lane * 4u;
  const int K = p.K;
  const int ndk = (K + kDK - 1) / kDK;
  const int d_lo = (warp * ndk) / kWarps, d_hi = ((warp + 1) * ndk) / kWarps;
  const size_t row_bytes = (size_t)K / 2;
  const int nsc = FMT == 0 ? K / 64 : K / 32;  // scales per weight row

  for (int u = blockIdx.x; u < U; u += gridDim.x) {
    const int e = find_group(s.upre, p.E, u);
    const int jb = u - s.upre[e];
    const int r0 = s.off[e], rows = s.off[e + 1] - r0;
    if (rows > kMaxTokens) {  // uniform over the CTA
      if (tid == 0 && jb == 0) atomicOr(p.err, GNF4_DEVERR_GEMV_ROWS);
      continue;
    }
    // this lane's 8 weight rows: q = 2*tile + half -> row jb*64 + g + 8q
    const int n0 = jb * kRows + g;
    const size_t rr0 = (size_t)e * p.N + (size_t)n0;
    const uint8_t* wbase = p.w + rr0 * row_bytes;
    const size_t sbase = rr0 * (size_t)nsc;
    const int nvalid_q = (p.N - n0 + 7) / 8;  // rows n0 + 8q < N  <=>  q < nvalid_q
    const bool tv = g < rows;
    const __nv_bfloat16* xrow = p.a + (size_t)(r0 + (tv ? g : 0)) * K;

    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

    for (int d = d_lo; d < d_hi; ++d) {
      const int k0 = d * kDK + 32 * t;
      const bool inK = k0 < K;
      uint4 wq[8];
      uint32_t sc[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const bool ok = inK && q < nvalid_q;
        const size_t roff = (size_t)(8 * q);
        wq[q] = ok ? ldg_nc_u128(wbase + roff * row_bytes + (k0 >> 1)) : make_uint4(0u, 0u, 0u, 0u);
        if (FMT == 0) {
          const float am =
              ok ? __ldg(reinterpret_cast<const float*>(p.scales) + sbase + roff * (size_t)nsc + (k0 >> 6)) : 0.f;
          sc[q] = f32_to_bf16x2_rn(am);
        } else {
          sc[q] = ok ? e8m0_to_bf16x2(
                           __ldg(reinterpret_cast<const uint8_t*>(p.scales) + sbase + roff * (size_t)nsc + (k0 >> 5)))
                     : 0u;
        }
      }
      uint4 xa[4];
#pragma unroll
      for (int v = 0; v < 4; ++v)
        xa[v] = (tv && inK) ? ldg_u128(xrow + k0 + 8 * v) : make_uint4(0u, 0u, 0u, 0u);
      const uint32_t xp[16] = {xa[0].x, xa[0].y, xa[0].z, xa[0].w, xa[1].x, xa[1].y, xa[1].z, xa[1].w,
                               xa[2].x, xa[2].y, xa[2].z, xa[2].w, xa[3].x, xa[3].y, xa[3].z, xa[3].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint32_t pa[16], pb[16];
        decode16_lut256(lut, lane4, wq[2 * i], sc[2 * i], pa);
        decode16_lut256(lut, lane4, wq[2 * i + 1], sc[2 * i + 1], pb);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          mma_bf16_16816(acc[i], pa[2 * j], pb[2 * j], pa[2 * j + 1], pb[2 * j + 1], xp[2 * j], xp[2 * j + 1]);
      }
    }
    // fixed-order reduction over the warps
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) s.red[warp][i][lane][j] = acc[i][j];
    __syncthreads();
    for (int o = tid; o < 4 * 32 * 4; o += kThreads) {
      const int i = o >> 7, l = (o >> 2) & 31, j = o & 3;
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) v += s.red[w][i][l][j];
      const int n = jb * kRows + 16 * i + (l >> 2) + 8 * (j >> 1);
      const int tok = 2 * (l & 3) + (j & 1);
      if (n < p.N && tok < rows) p.y[(size_t)(r0 + tok) * p.N + n] = __float2bfloat16_rn(v);
    }
    __syncthreads();
  }
}

}  // namespace

int gemv_rows_per_block() { return kRows; }

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
