// gemv.cu -- grouped 4-bit expert GEMV for decode (at most 8 rows per group).
//
// Decode steps are bandwidth-bound: the weights of the routed experts are the
// bytes that must stream from HBM (grouped-nf4-gemm index.json,
// problems_solved[2]).  The pages' decode GEMV re-streams the weights once per
// row (same page, limitations); here every weight byte is read once and used
// for all of its group's rows.
//
// Work unit = (expert e, 64 consecutive weight rows).  A CTA (one per SM,
// 16 warps) runs two units at a time, one per half of 8 warps; the 8 warps of
// a half split K: warp s takes a contiguous range of 128-k "items" and
// computes the partial sums of all 64 rows (four m16 tiles) for the group's
// <= 8 rows (the MMA's 8 columns); a fixed-order shared-memory reduction over
// the 8 warps finishes the unit.  Per item a lane holds 16 bytes (32 codes)
// of each of its 8 weight rows, decodes every byte with one PRMT, which
// builds the shared-memory address of a lane-private pair-table entry, and
// one shared load, multiplies the bf16 pair by the row's block scale, and
// feeds the pairs to m16n8k16 warp MMAs.  The MMA does the k reduction that
// a CUDA-core GEMV would do with shuffles.
//
// Fused combine (CMB): after a half has stored its unit's rows, each row
// counts its (token, 64-column block) in; the half that completes a token's
// last valid pair computes that token's 64 output columns with the same fp32
// fmaf sequence as the separate combine (pairs in slot order), so the fused
// output equals the unfused one bit for bit, and resets the counter for the
// next call.  Stores are published with a fence before the count; the
// completing half fences again before it reads the other rows through L2.
//
// Latency hiding: a warp's items form one stream across unit boundaries, and
// the loads of the next item are issued tile by tile while the current item
// is decoded (each tile's registers are refilled as soon as they have been
// decoded), so every warp always has about one item (4 KB) in flight without
// a second register set.
//
// The pair table (one copy per SM, 64 KB) starts at the first 64 KB boundary
// of the shared window above the kernel's other shared data (0x10000 unless
// static shared memory grows past the budget checked on the host): the PRMT
// that extracts a byte also inserts the table's base, so a lookup is exactly
// one PRMT and one shared load.
//
// Lane (g, t) = (lane / 4, lane % 4) owns rows g and g+8 of every tile and,
// in every item, the 32 consecutive k in [32t, 32t+32) (one NF4 half-block,
// one MXFP4 block).  The MMA's k index is a permutation of these physical k;
// the activation fragment uses the same permutation.
//   * MXFP4: e2m1 x 2^(e-127) is exact in bf16.
//   * NF4: the code is rounded to bf16, then multiplied by bf16(absmax) and
//     rounded again (relative error <= ~3 * 2^-9 per weight); sums are fp32.
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace gnf4 {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kSplit = 8;                 // warps per half = K-splits of a unit
constexpr int kRows = 64;                 // weight rows per unit (4 m16 tiles)
constexpr int kMaxTokens = 8;             // rows of a group = MMA columns
constexpr int kDK = 128;                  // k per item
constexpr int kSmemBytes = 0x20000;  // dynamic shared memory per CTA

// Everything but the pair table; lives below it.
struct GemvLow {
  float red[2][kSplit][4][32][4];  // 32 KB: partial sums per half and K-split
  int done[2][kMaxTokens];         // fused combine: tokens a half's unit completed (-1: none)
  int off[kMaxExperts + 1];
  int upre[kMaxExperts + 1];
  int scratch[kMaxExperts];
};

// f32 -> bf16 (round to nearest even, NaN kept quiet), duplicated in both halves.
__device__ __forceinline__ uint32_t cvt_bf16x2_dup(float f) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %1;" : "=r"(d) : "f"(f));
  return d;
}

// One pair-table lookup: byte j of `word` selects the entry; `lanesel` holds
// 4*lane in byte 0 and byte 2 of the table's 64 KB-aligned base in byte 2.
__device__ __forceinline__ uint32_t lut_lookup(uint32_t word, uint32_t lanesel, uint32_t j) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(prmt_b32(word, lanesel, 0x7604u | (j << 4))));
  return v;
}

__device__ __forceinline__ void half_barrier(int h) {
  asm volatile("bar.sync %0, %1;" ::"r"(1 + h), "r"(kThreads / 2) : "memory");
}

// Per-lane view of one unit: where this lane's rows, scales and activation row start.
struct UnitView {
  const uint8_t* w;            // weight row n0 (q = 0), byte 0
  const uint8_t* sc;           // first scale of row n0 (bytes)
  const __nv_bfloat16* x;      // activation row of token g (row 0 if g >= rows), k = 32t
  int qv;                      // rows n0 + 8q < N  <=>  q < qv
  bool tv;                     // token g exists
};

// Row layouts of a unit's 8 rows per lane (q = 0..7):
//   kModeClamp  rows n0 + 8q of a [E, N, K] stack, N % 8 == 0 (rows past N read row N-1, never stored)
//   kModeFull   rows n0 + 8q, N % 64 == 0
//   kModeSwiglu gate_up stack [E, 2I, K]: q < 4 are gate rows n0 + 8q, q >= 4 the matching up rows
//               I + n0 + 8(q-4), with n0 = 32 jb + g; the unit writes h columns [32 jb, 32 jb + 32)
constexpr int kModeClamp = 0, kModeFull = 1, kModeSwiglu = 2;

template <int FMT, int MODE>
__device__ __forceinline__ UnitView unit_view(const GemvLow& s, const GroupedArgs& p, int u, int g, int t) {
  const int e = find_group(s.upre, p.E, u);
  const int jb = u - s.upre[e];
  const int r0 = s.off[e], rows = s.off[e + 1] - r0;
  const int n0 = jb * (MODE == kModeSwiglu ? kRows / 2 : kRows) + g;
  const size_t row = (size_t)e * p.N + (size_t)n0;
  const int nsc = FMT == 0 ? p.K / 64 : p.K / 32;
  UnitView v;
  v.w = p.w + row * (size_t)(p.K / 2);
  v.sc = reinterpret_cast<const uint8_t*>(p.scales) + row * (size_t)nsc * (FMT == 0 ? 4u : 1u);
  v.tv = g < rows;
  v.x = p.a + (size_t)(r0 + (v.tv ? g : 0)) * p.K + 32 * t;
  v.qv = (p.N - n0 + 7) / 8;
  return v;
}

// Loads of one item for tile i (rows q = 2i, 2i+1): packed weights and raw scales.
// `rb` = packed bytes per weight row, `nsr` = scales per weight row, `gap` =
// I - 32 (kModeSwiglu: rows from the unit's last gate row block to its up rows).
template <int FMT, int MODE>
__device__ __forceinline__ void load_tile(const UnitView& v, int d, int t, int K, size_t rb, size_t nsr, int gap,
                                          int i, uint4 (&wq)[8], uint32_t (&sr)[8]) {
  const bool inK = d * kDK + 32 * t < K;
  const size_t kb = inK ? (size_t)(d * (kDK / 2) + 16 * t) : 0;  // outside K: any valid address
  const size_t si = inK ? (size_t)(FMT == 0 ? 2 * d + (t >> 1) : 4 * d + t) : 0;
#pragma unroll
  for (int hq = 0; hq < 2; ++hq) {
    const int q = 2 * i + hq;
    const int roff = MODE == kModeClamp ? 8 * min(q, v.qv - 1) : (MODE == kModeSwiglu && q >= 4 ? 8 * q + gap : 8 * q);
    wq[q] = ldg_nc_u128(v.w + (size_t)roff * rb + kb);
    if (FMT == 0)
      sr[q] = __ldg(reinterpret_cast<const unsigned int*>(v.sc + ((size_t)roff * nsr + si) * 4u));
    else
      sr[q] = __ldg(v.sc + (size_t)roff * nsr + si);
  }
}

__device__ __forceinline__ void load_acts(const UnitView& v, int d, int t, int K, uint4 (&xa)[4]) {
  const bool ok = v.tv && (d * kDK + 32 * t < K);
#pragma unroll
  for (int c = 0; c < 4; ++c) xa[c] = ok ? ldg_u128(v.x + d * kDK + 8 * c) : make_uint4(0u, 0u, 0u, 0u);
}

template <int FMT>
__device__ __forceinline__ uint32_t scale_pair(uint32_t raw) {
  return FMT == 0 ? cvt_bf16x2_dup(__uint_as_float(raw)) : e8m0_to_bf16x2(raw);
}

// Sum over the valid pairs of token t (sorted row inside [0, nvalid)).
__device__ __forceinline__ int valid_pairs(const CombineArgs& c, int t, int nvalid) {
  int need = 0;
  for (int j = 0; j < c.k; ++j) {
    const int r = __ldg(c.f2s + (size_t)t * c.k + j);
    need += (r >= 0 && r < nvalid) ? 1 : 0;
  }
  return need;
}

template <int FMT, int MODE, bool CMB>
__global__ void __launch_bounds__(kThreads, 1) gemv_kernel(GroupedArgs p, CombineArgs cmb) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  GemvLow& s = *reinterpret_cast<GemvLow*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int h = warp / kSplit, ks = warp % kSplit;

  // The table takes the first 64 KB boundary above GemvLow; the host refuses
  // to launch when the window cannot hold it (table_fits_once), so this
  // check only guards against a window placed differently than the host saw.
  const uint32_t base = smem_u32(smem_raw);
  const uint32_t lut_at = (base + (uint32_t)sizeof(GemvLow) + 0xFFFFu) & ~0xFFFFu;
  if (lut_at + (uint32_t)kLut256Bytes > base + (uint32_t)kSmemBytes) {
    if (tid == 0) atomicOr(p.err, GNF4_DEVERR_INTERNAL);
    return;
  }
  griddep_launch_dependents();
  // the pair table depends on nothing earlier in the stream: build it while
  // the previous kernel finishes (made visible by the barriers below)
  build_pair_lut256<FMT>(reinterpret_cast<uint32_t*>(smem_raw + (lut_at - base)), tid, kThreads);
  griddep_wait();
  if (!load_groups(p.offsets, p.counts, p.E, p.M, s.off, s.scratch, p.err)) return;
  const int nblk = MODE == kModeSwiglu ? (p.N / 2) / (kRows / 2) : (p.N + kRows - 1) / kRows;
  block_exclusive_scan(p.E, s.upre, s.scratch, [&](int e) { return (s.off[e + 1] > s.off[e]) ? nblk : 0; });
  const int U = s.upre[p.E];
  if (CMB && blockIdx.x == 0) {  // tokens without a valid pair get a zero row (no unit ever completes them)
    const int nvalid = s.off[p.E];
    for (int t = tid; t < cmb.T; t += kThreads)
      if (valid_pairs(cmb, t, nvalid) == 0)
        for (int n = 0; n < p.N; ++n) cmb.out[(size_t)t * p.N + n] = __float2bfloat16_rn(0.f);
  }
  if (2 * (int)blockIdx.x >= U) return;  // uniform over the CTA

  const int K = p.K;
  const int ndk = (K + kDK - 1) / kDK;
  const int d_lo = (ks * ndk) / kSplit, d_hi = ((ks + 1) * ndk) / kSplit;
  const size_t rb = (size_t)(K / 2);                              // packed bytes per weight row
  const size_t nsr = (size_t)(FMT == 0 ? K / 64 : K / 32);         // scales per weight row
  const int gap = p.N / 2 - kRows / 2;                             // kModeSwiglu only
  const int ustride = 2 * (int)gridDim.x;
  int u = 2 * (int)blockIdx.x + h;

  // first item of this warp's stream
  uint4 wq[8], xa[4];
  uint32_t sr[8];
  UnitView cur{};
  if (u < U) {
    cur = unit_view<FMT, MODE>(s, p, u, g, t);
    if (d_lo < d_hi) {
#pragma unroll
      for (int i = 0; i < 4; ++i) load_tile<FMT, MODE>(cur, d_lo, t, K, rb, nsr, gap, i, wq, sr);
      load_acts(cur, d_lo, t, K, xa);
    }
  }
  __syncthreads();

  const uint32_t lanesel = (uint32_t)lane * 4u | (lut_at & 0x00FF0000u);

  for (; u < U; u += ustride) {  // uniform over the half
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;

    for (int d = d_lo; d < d_hi; ++d) {
      // The next item of this warp's stream is (u, d+1), or the first item of
      // the next unit.  The current item's loads were issued one iteration
      // ago, so `cur` can already describe the unit of the next item.
      const bool last = d + 1 == d_hi;
      const int dn = last ? d_lo : d + 1;
      const bool has_next = !last || u + ustride < U;
      if (last && has_next) cur = unit_view<FMT, MODE>(s, p, u + ustride, g, t);
      uint4 xn[4];
      if (has_next) load_acts(cur, dn, t, K, xn);

      const uint32_t xp[16] = {xa[0].x, xa[0].y, xa[0].z, xa[0].w, xa[1].x, xa[1].y, xa[1].z, xa[1].w,
                               xa[2].x, xa[2].y, xa[2].z, xa[2].w, xa[3].x, xa[3].y, xa[3].z, xa[3].w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint32_t s0 = scale_pair<FMT>(sr[2 * i]), s1 = scale_pair<FMT>(sr[2 * i + 1]);
        const uint32_t w0[4] = {wq[2 * i].x, wq[2 * i].y, wq[2 * i].z, wq[2 * i].w};
        const uint32_t w1[4] = {wq[2 * i + 1].x, wq[2 * i + 1].y, wq[2 * i + 1].z, wq[2 * i + 1].w};
        // MMA step j takes bytes 2j, 2j+1 of both rows (word j/2, bytes 2(j%2) and 2(j%2)+1)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t b0 = 2u * (uint32_t)(j & 1);
          const uint32_t a0 = bf16x2_mul(lut_lookup(w0[j >> 1], lanesel, b0), s0);
          const uint32_t a1 = bf16x2_mul(lut_lookup(w1[j >> 1], lanesel, b0), s1);
          const uint32_t a2 = bf16x2_mul(lut_lookup(w0[j >> 1], lanesel, b0 + 1u), s0);
          const uint32_t a3 = bf16x2_mul(lut_lookup(w1[j >> 1], lanesel, b0 + 1u), s1);
          mma_bf16_16816(acc[i], a0, a1, a2, a3, xp[2 * j], xp[2 * j + 1]);
        }
        if (has_next) load_tile<FMT, MODE>(cur, dn, t, K, rb, nsr, gap, i, wq, sr);
      }
      if (has_next) {
#pragma unroll
        for (int c = 0; c < 4; ++c) xa[c] = xn[c];
      }
    }

    // fixed-order reduction over the half's 8 warps
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<float4*>(&s.red[h][ks][i][lane][0]) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
    half_barrier(h);
    {
      const int e = find_group(s.upre, p.E, u);
      const int jb = u - s.upre[e];
      const int r0 = s.off[e], rows = s.off[e + 1] - r0;
      const int ht = tid & (kThreads / 2 - 1);
      if (rows > kMaxTokens) {
        if (ht == 0 && jb == 0) atomicOr(p.err, GNF4_DEVERR_GEMV_ROWS);
      } else if (MODE == kModeSwiglu) {
        // tiles 0, 1 hold gate rows, tiles 2, 3 the matching up rows
        const int I = p.N / 2;
        for (int o = ht; o < 2 * 32 * 4; o += kThreads / 2) {
          const int i = o >> 7, l = (o >> 2) & 31, j = o & 3;
          float vg = 0.f, vu = 0.f;
#pragma unroll
          for (int w = 0; w < kSplit; ++w) {
            vg += s.red[h][w][i][l][j];
            vu += s.red[h][w][i + 2][l][j];
          }
          const int col = jb * (kRows / 2) + 16 * i + (l >> 2) + 8 * (j >> 1);
          const int tok = 2 * (l & 3) + (j & 1);
          if (tok < rows) p.y[(size_t)(r0 + tok) * I + col] = __float2bfloat16_rn(silu_mul(vg, vu));
        }
      } else {
        for (int o = ht; o < 4 * 32 * 4; o += kThreads / 2) {
          const int i = o >> 7, l = (o >> 2) & 31, j = o & 3;
          float v = 0.f;
#pragma unroll
          for (int w = 0; w < kSplit; ++w) v += s.red[h][w][i][l][j];
          const int n = jb * kRows + 16 * i + (l >> 2) + 8 * (j >> 1);
          const int tok = 2 * (l & 3) + (j & 1);
          if (n < p.N && tok < rows) p.y[(size_t)(r0 + tok) * p.N + n] = __float2bfloat16_rn(v);
        }
        if (CMB) {
          // The half's stores happen before the barrier; the counting thread's
          // fence (cumulative) publishes them at GPU scope before its count.
          half_barrier(h);
          const int nvalid = s.off[p.E];
          if (ht < kMaxTokens) {
            int t = -1;
            if (ht < rows) {
              const int f = __ldg(cmb.s2f + r0 + ht);
              if (f >= 0 && f < cmb.T * cmb.k) {
                const int tk = f / cmb.k;
                int* ctr = cmb.cnt + (size_t)tk * nblk + jb;
                __threadfence();
                if (atomicAdd(ctr, 1) == valid_pairs(cmb, tk, nvalid) - 1) {
                  __threadfence();  // the other units' rows of tk are visible to this half from here on
                  t = tk;
                  *ctr = 0;  // every pair of this block is in: ready for the next call
                }
              }
            }
            s.done[h][ht] = t;
          }
          half_barrier(h);
          for (int o = ht; o < kMaxTokens * kRows; o += kThreads / 2) {
            const int t = s.done[h][o / kRows];
            const int n = jb * kRows + (o % kRows);
            if (t < 0 || n >= p.N) continue;
            float acc = 0.f;
            for (int j0 = 0; j0 < cmb.k; j0 += 8) {  // 8 independent row loads, then the fmaf chain in slot order
              float yv[8], wv[8];
              bool okv[8];
#pragma unroll
              for (int jj = 0; jj < 8; ++jj) {
                const int j = j0 + jj;
                const int r = j < cmb.k ? __ldg(cmb.f2s + (size_t)t * cmb.k + j) : -1;
                const bool ok = r >= 0 && r < nvalid;  // else a dropped pair
                const unsigned short yb =
                    ok ? __ldcg(reinterpret_cast<const unsigned short*>(p.y) + (size_t)r * p.N + n) : (unsigned short)0;
                yv[jj] = __uint_as_float((uint32_t)yb << 16);
                wv[jj] = ok ? __ldg(cmb.w + (size_t)t * cmb.k + j) : 0.f;
                okv[jj] = ok;
              }
#pragma unroll
              for (int jj = 0; jj < 8; ++jj)
                if (okv[jj]) acc = fmaf(wv[jj], yv[jj], acc);
            }
            cmb.out[(size_t)t * p.N + n] = __float2bfloat16_rn(acc);
          }
        }
      }
    }
    half_barrier(h);
  }
}

}  // namespace

int gemv_grid(long long units, int num_sms) {
  const long long ctas = (units + 1) / 2;  // two units at a time per CTA
  return (int)(ctas < num_sms ? ctas : num_sms);
}

// Host side of the pair-table placement: the dynamic window starts after the
// device's reserved and the kernel's static shared memory (at most 1 KB of
// alignment more), and the table needs GemvLow below the 64 KB boundary.
// Checked once per device; a launch the table cannot fit is refused with
// cudaErrorInvalidConfiguration before anything is enqueued.
template <typename Kernel>
static cudaError_t table_fits_once(Kernel kernel, std::atomic<int> (&state)[64]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool tracked = dev >= 0 && dev < 64;
  if (tracked) {
    const int st = state[dev].load(std::memory_order_acquire);
    if (st != 0) return st > 0 ? cudaSuccess : cudaErrorInvalidConfiguration;
  }
  cudaFuncAttributes fa;
  if ((e = cudaFuncGetAttributes(&fa, kernel)) != cudaSuccess) return e;
  int reserved = 0;
  if ((e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, dev)) != cudaSuccess) return e;
  const size_t start = ((size_t)reserved + fa.sharedSizeBytes + 1023) & ~(size_t)1023;
  const bool fits = start + sizeof(GemvLow) <= 0x10000u;
  if (tracked) state[dev].store(fits ? 1 : -1, std::memory_order_release);
  return fits ? cudaSuccess : cudaErrorInvalidConfiguration;
}

template <int FMT, int MODE, bool CMB>
static cudaError_t launch_gemv_t(const GroupedArgs& p, const CombineArgs& c, int grid, cudaStream_t stream) {
  static std::atomic<bool> configured[64];
  static std::atomic<int> placed[64];
  cudaError_t e = table_fits_once(gemv_kernel<FMT, MODE, CMB>, placed);
  if (e != cudaSuccess) return e;
  e = set_smem_limit_once(gemv_kernel<FMT, MODE, CMB>, kSmemBytes, configured);
  if (e != cudaSuccess) return e;
  return launch_pdl(gemv_kernel<FMT, MODE, CMB>, dim3(grid), dim3(kThreads), (size_t)kSmemBytes, stream, p, c);
}

template <int FMT>
static cudaError_t launch_gemv_f(bool swiglu, const GroupedArgs& p, const CombineArgs* c, int grid,
                                 cudaStream_t stream) {
  const CombineArgs none{};
  if (swiglu) return launch_gemv_t<FMT, kModeSwiglu, false>(p, none, grid, stream);
  if (c != nullptr)
    return p.N % kRows == 0 ? launch_gemv_t<FMT, kModeFull, true>(p, *c, grid, stream)
                            : launch_gemv_t<FMT, kModeClamp, true>(p, *c, grid, stream);
  return p.N % kRows == 0 ? launch_gemv_t<FMT, kModeFull, false>(p, none, grid, stream)
                          : launch_gemv_t<FMT, kModeClamp, false>(p, none, grid, stream);
}

cudaError_t launch_gemv(int fmt, bool swiglu, const GroupedArgs& p, int grid, cudaStream_t stream,
                        const CombineArgs* combine) {
  return fmt == 0 ? launch_gemv_f<0>(swiglu, p, combine, grid, stream)
                  : launch_gemv_f<1>(swiglu, p, combine, grid, stream);
}

size_t gemv_combine_counter_bytes(int T, int N) { return (size_t)T * (size_t)((N + kRows - 1) / kRows) * 4; }

int gemv_rows_per_block() { return kRows; }
int gemv_swiglu_cols_per_block() { return kRows / 2; }

}  // namespace gnf4
