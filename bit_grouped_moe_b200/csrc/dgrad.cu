// dgrad.cu -- data gradient of the grouped 4-bit projection on tcgen05 (sm_100a):
//     dX[r, k] = sum_n dY[r, n] * W_e[n, k]     for the rows r of every expert e
// (grouped-nf4-gemm index.json, system_manifest.owns: "grouped packed GEMM (NF4
// and native MXFP4) and its dgrad"; entrypoints: nf4_grouped:dgrad_4bit_grouped),
// on the same packed stacks the forward call reads; fp32 accumulation, bf16 out.
//
// The contraction runs over the weight rows n.  A stage covers 64 of them:
//  * the dY tile [128 rows r][64 n] bf16 arrives by TMA in the 128B-swizzled
//    K-major layout (the MMA's A operand);
//  * the packed weight block [64 n][64 bytes = 128 k] arrives by TMA;
//  * the four warps decode it through the pair table and write it TRANSPOSED
//    as [128 k][64 n] bf16 in the same 128B-swizzled K-major layout (the MMA's
//    B operand), so both operands use the plain K-major descriptor.
// D[r, k] accumulates in TMEM (lane = row r, column = k).  Work unit = (expert
// e, chunk of <= 128 of its rows, 128-wide k tile); a persistent grid strides
// over the units.  Two stage buffers: the TMA of stage s+1 and the MMAs of
// stage s-1 overlap the decode of stage s.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace gnf4 {
namespace {

constexpr int kThreads = 128;
constexpr int kBR = 128;                   // rows per unit (MMA M)
constexpr int kBKt = 128;                  // k per unit (MMA N)
constexpr int kBN = 64;                    // n per stage (four k-steps of 16)
constexpr int kYBytes = kBR * kBN * 2;     // 16 KB
constexpr int kTBytes = kBKt * kBN * 2;    // 16 KB
constexpr int kWBytes = kBN * kBKt / 2;    // 4 KB
constexpr int kTmemCols = kBKt;

struct DSmem {
  uint8_t y[2][kYBytes];    // dY tiles (1024-aligned for the 128-byte swizzle)
  uint8_t t[2][kTBytes];    // decoded W^T tiles
  uint8_t w[2][kWBytes];    // packed weight blocks
  uint32_t lut[kLut256Words];
  int off[kMaxExperts + 1];
  int upre[kMaxExperts + 1];
  int scratch[kMaxExperts];
  uint64_t full[2], mdone[2], accf, drain;
  uint32_t tmem_base;
  int abort;
};

struct DUnit {
  int e, kt, row0, rows;
};

__device__ __forceinline__ DUnit dunit_of(const DSmem& s, int E, int nkt, int u) {
  DUnit x;
  x.e = find_group(s.upre, E, u);
  const int local = u - s.upre[x.e];
  const int c = local / nkt;
  x.kt = local - c * nkt;
  x.row0 = s.off[x.e] + c * kBR;
  x.rows = min(kBR, s.off[x.e + 1] - x.row0);
  return x;
}

// D[tmem] (+)= A[smem] x B[smem]^T, kind::f16, both operands K-major.
__device__ __forceinline__ void tc_mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Byte offset of the 16-byte chunk c (8 bf16 of n) of row k in a 128B-swizzled
// K-major tile with 128-byte rows (8-row atoms of 1 KB).
__device__ __forceinline__ uint32_t sw128_chunk(int k, int c) {
  return (uint32_t)((k >> 3) * 1024 + (k & 7) * 128 + ((c ^ (k & 7)) << 4));
}

__device__ __forceinline__ void sts_u128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ uint32_t lds_u8(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

template <int FMT>
__global__ void __launch_bounds__(kThreads, 1)
    dgrad_tc_kernel(const __grid_constant__ CUtensorMap tm_y, const __grid_constant__ CUtensorMap tm_w,
                    GroupedArgs p) {
  extern __shared__ uint8_t smem_raw[];
  DSmem& s = *reinterpret_cast<DSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  unsigned* err = p.err;
  volatile int* abort = &s.abort;
  // p.N = weight rows (the contraction), p.K = weight columns (the output width)
  const int N = p.N, K = p.K;

  griddep_launch_dependents();
  build_pair_lut256<FMT>(s.lut, tid, kThreads);
  griddep_wait();
  if (!load_groups(p.offsets, p.counts, p.E, p.M, s.off, s.scratch, err)) return;
  const int nkt = (K + kBKt - 1) / kBKt;
  block_exclusive_scan(p.E, s.upre, s.scratch, [&](int e) { return ((s.off[e + 1] - s.off[e] + kBR - 1) / kBR) * nkt; });
  const int U = s.upre[p.E];
  if ((int)blockIdx.x >= U) return;  // uniform over the block
  const int ns = (N + kBN - 1) / kBN;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.mdone[i], 1);
    }
    mbar_init(&s.accf, 1);
    mbar_init(&s.drain, 1);
    s.abort = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_y);
    prefetch_tmap(&tm_w);
  }
  if (warp == 0) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  const uint32_t lut = smem_u32(s.lut);
  const uint32_t lane4 = (uint32_t)lane * 4u;
  const uint32_t idesc = idesc_bf16_m128((uint32_t)kBKt);
  const int nsc = FMT == 0 ? K / 64 : K / 32;  // scales per weight row

  // stage stream: stage g = (unit u, n-block sb); issue(g) loads it into buffer g & 1
  int issued = 0;  // thread 0: stages issued
  auto issue = [&](int u, int sb, int g) {
    ++issued;
    const DUnit x = dunit_of(s, p.E, nkt, u);
    const int b = g & 1;
    mbar_arrive_expect_tx(&s.full[b], kYBytes + kWBytes);
    tma_load_2d(s.y[b], &tm_y, &s.full[b], sb * kBN, x.row0);
    tma_load_3d(s.w[b], &tm_w, &s.full[b], x.kt * (kBKt / 2), sb * kBN, x.e);
  };

  int g = 0, uc = 0;  // stages consumed, units finished by this CTA
  bool ok = true;
  if (tid == 0) issue(blockIdx.x, 0, 0);
  for (int u = blockIdx.x; u < U; u += gridDim.x, ++uc) {
    const DUnit x = dunit_of(s, p.E, nkt, u);
    const int k0 = x.kt * kBKt;
    for (int sb = 0; sb < ns; ++sb, ++g) {
      const int b = g & 1;
      // producer: stage g+1 into the other buffer once the MMAs of stage g-1 are done with it
      if (tid == 0 && !*abort) {
        const int nu = sb + 1 < ns ? u : u + (int)gridDim.x;
        const int nsb = sb + 1 < ns ? sb + 1 : 0;
        if (nu < U) {
          if (g >= 1) ok = mbar_wait(&s.mdone[b ^ 1], ((g - 1) >> 1) & 1, err, abort);
          if (ok) issue(nu, nsb, g + 1);
        }
      }
      // this stage's tiles have landed, and the MMAs of stage g-2 no longer read t[b]
      if (!*abort) mbar_wait(&s.full[b], (g >> 1) & 1, err, abort);
      if (g >= 2 && !*abort) mbar_wait(&s.mdone[b], ((g - 2) >> 1) & 1, err, abort);

      // decode: item (kp, nb) = k pair kp (k = 2kp, 2kp+1 of the tile), n rows nb*8 .. nb*8+7
      const uint32_t wbase = smem_u32(s.w[b]);
      const uint32_t tbase = smem_u32(s.t[b]);
      const int n0 = sb * kBN;
#pragma unroll 1
      for (int j = 0; j < 4; ++j) {
        const int item = tid + kThreads * j;
        const int kp = item & 63, nb = item >> 6;
        const int kk = k0 + 2 * kp;  // first k of the pair
        const int kblk = min(FMT == 0 ? kk / 64 : kk / 32, nsc - 1);  // past K: any valid scale, never stored
        uint32_t pr[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int n = n0 + nb * 8 + i;
          const uint32_t byte = lds_u8(wbase + (uint32_t)((nb * 8 + i) * (kBKt / 2) + kp));
          uint32_t sc = 0u;  // rows past N contribute nothing
          if (n < N) {
            const size_t srow = ((size_t)x.e * N + (size_t)n) * (size_t)nsc + (size_t)kblk;
            sc = FMT == 0 ? f32_to_bf16x2_rn(__ldg(reinterpret_cast<const float*>(p.scales) + srow))
                          : e8m0_to_bf16x2(__ldg(reinterpret_cast<const uint8_t*>(p.scales) + srow));
          }
          pr[i] = bf16x2_mul(lut256_get(lut, byte, lane4, 0u), sc);
        }
        // row 2kp of W^T takes the low halves (even k), row 2kp+1 the high halves
        sts_u128(tbase + sw128_chunk(2 * kp, nb), prmt_b32(pr[0], pr[1], 0x5410u), prmt_b32(pr[2], pr[3], 0x5410u),
                 prmt_b32(pr[4], pr[5], 0x5410u), prmt_b32(pr[6], pr[7], 0x5410u));
        sts_u128(tbase + sw128_chunk(2 * kp + 1, nb), prmt_b32(pr[0], pr[1], 0x7632u),
                 prmt_b32(pr[2], pr[3], 0x7632u), prmt_b32(pr[4], pr[5], 0x7632u), prmt_b32(pr[6], pr[7], 0x7632u));
      }
      fence_proxy_async_smem();  // generic-proxy writes of t[b] before the MMA reads them
      __syncthreads();
      if (tid == 0 && !*abort) {
        tc_fence_after();
        const uint32_t ya = smem_u32(s.y[b]), ta = smem_u32(s.t[b]);
#pragma unroll
        for (int q = 0; q < kBN / 16; ++q)
          tc_mma_ss(tmem, sdesc_k_sw128(ya + q * 32), sdesc_k_sw128(ta + q * 32), idesc, (sb | q) != 0);
        tc_commit(&s.mdone[b]);
      }
    }
    // epilogue: lane = row, columns = k
    if (tid == 0 && !*abort) tc_commit(&s.accf);
    if (!*abort) mbar_wait(&s.accf, uc & 1, err, abort);
    tc_fence_after();
    const int r = warp * 32 + lane;
    const uint32_t t_lane = tmem + ((uint32_t)(warp * 32) << 16);
    for (int c = 0; c < kBKt / 32; ++c) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(t_lane + (uint32_t)(c * 32), v);
      tmem_wait_ld();
      const int kc = k0 + c * 32;
      if (r < x.rows && kc < K && !*abort) {
        __nv_bfloat16* dst = p.y + (size_t)(x.row0 + r) * K + kc;
        if (kc + 32 <= K) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 o;
            __nv_bfloat162 h0 = __floats2bfloat162_rn(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1]));
            __nv_bfloat162 h1 = __floats2bfloat162_rn(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3]));
            __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5]));
            __nv_bfloat162 h3 = __floats2bfloat162_rn(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7]));
            o.x = *reinterpret_cast<uint32_t*>(&h0);
            o.y = *reinterpret_cast<uint32_t*>(&h1);
            o.z = *reinterpret_cast<uint32_t*>(&h2);
            o.w = *reinterpret_cast<uint32_t*>(&h3);
            reinterpret_cast<uint4*>(dst)[q] = o;
          }
        } else {
          for (int i = 0; i < 32 && kc + i < K; ++i) dst[i] = __float2bfloat16_rn(__uint_as_float(v[i]));
        }
      }
    }
    tc_fence_before();
    __syncthreads();  // the accumulator is read before the next unit's first MMA
  }
  if (*abort && tid == 0) {
    // let issued MMAs retire and landing copies complete before the memory goes away
    tc_commit(&s.drain);
    mbar_drain(&s.drain, 0);
    for (int i = max(0, issued - 2); i < issued; ++i) mbar_drain(&s.full[i & 1], (uint32_t)(i >> 1) & 1u);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

size_t dgrad_tc_smem_bytes() { return sizeof(DSmem) + 1024; }
int dgrad_tc_rows_per_unit() { return kBR; }
int dgrad_tc_k_per_unit() { return kBKt; }
int dgrad_tc_n_per_stage() { return kBN; }

template <int FMT>
static cudaError_t launch_dgrad_t(const CUtensorMap& tm_y, const CUtensorMap& tm_w, const GroupedArgs& p, int grid,
                                  cudaStream_t stream) {
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaError_t e = cudaFuncSetAttribute(dgrad_tc_kernel<FMT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)dgrad_tc_smem_bytes());
    if (e != cudaSuccess) return e;
    configured[dev] = true;
  }
  return launch_pdl(dgrad_tc_kernel<FMT>, dim3(grid), dim3(kThreads), dgrad_tc_smem_bytes(), stream, tm_y, tm_w, p);
}

cudaError_t launch_dgrad_tc(int fmt, const CUtensorMap& tm_y, const CUtensorMap& tm_w, const GroupedArgs& p,
                            int grid, cudaStream_t stream) {
  return fmt == 0 ? launch_dgrad_t<0>(tm_y, tm_w, p, grid, stream) : launch_dgrad_t<1>(tm_y, tm_w, p, grid, stream);
}

}  // namespace gnf4
