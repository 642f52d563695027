// mx.cu -- the native block-scaled MXFP4 modes on tcgen05, and the
// activation quantisers that feed them:
//   W4A8     MXFP8 activations x MXFP4 weights   (kind::mxf8f6f4, K = 32 per MMA)
//   two-term hi + lo MXFP8 activations x MXFP4     (same MMA; both terms stacked
//            in one B operand): the accuracy of bf16 activations
//   W4A4     MXFP4 activations x MXFP4 weights   (kind::mxf4, K = 64 per MMA)
//
// bw24 v0.9.0 release notes (Features, "f8f4 tile piece 1"; Documentation,
// "prefill arc design"): W4A8-FP8 multiplies native e2m1 weights by e4m3
// activations in one block-scaled MMA.  grouped-nf4-gemm index.json,
// system_manifest.owns: the grouped GEMM runs on native MXFP4.
//
// Quantisers (OCP MX v1.0): the 32 consecutive k of one row share an e8m0
// scale 2^X.  MXFP8 E4M3: X = floor(log2(amax)) - 8, elements x * 2^-X
// rounded to the nearest e4m3 value, ties to even, saturating at +-448
// (cvt.rn.satfinite); the two-term split uses X = floor(log2(amax)) - 7 for
// hi and for the exact residual lo (one binade of headroom: nothing
// saturates).  MXFP4: X = floor(log2(amax)) - 2, e2m1 saturating at +-6.  An
// all-zero block gets scale byte 0.
//
// GEMM design (B200):
//  * D^T[n, r] = W_e[n, :] . A[r, :]: the 128 weight rows of a tile are the
//    MMA's M, the rows (tokens) of the group its N, as in the bf16 path.
//  * Both operands go straight from global memory into 128B-swizzled shared
//    memory by TMA.  For kind::mxf8f6f4 the packed e2m1 weights are expanded
//    by the TMA unit itself into the layout the MMA reads (16 codes in 8
//    bytes followed by 8 bytes of padding, so 128 codes fill one 128-byte
//    row); kind::mxf4 reads them packed (256 codes per row).  The SM decodes
//    nothing: no lookup table and no bf16 copy of a weight exist anywhere.
//  * Block scales: per stage a loader warp copies the e8m0 scales of the
//    tile's 128 weight rows and of the group's rows into shared memory in the
//    layout tcgen05.cp reads (row m at byte 16*(m%32) + 4*(m/32), one byte
//    per 32-k block), moves them to the stage's own TMEM columns with
//    tcgen05.cp.32x128b.warpx4 and commits the copies to the stage's full
//    barrier; the MMAs of the stage select their scale bytes with their
//    scale-factor ids.  The MMA thread only waits, issues four MMAs and
//    commits: it is the one serial thread of the pipeline.
//  * K not a multiple of the stage's k: the last stage reads [K - kBK, K)
//    and skips the MMAs already covered, so no box reads past a row.
//  * Warp roles (14 warps): 0 and 12 = TMA producers (alternate stages: one
//    issuing thread alone caps the stream), 1 = TMEM owner + MMA issuer,
//    13 = stage poller (tests the full barriers and publishes a count of
//    complete stages that the MMA thread reads with a load-acquire),
//    4..7 = epilogue (warp w reads TMEM lanes 32*(w%4)..+31, i.e. weight
//    rows), 2, 3 and 8.. = scale loaders, one per ring slot, so the global
//    loads of every stage in the ring are in flight at once.  Two TMEM
//    accumulators let the epilogue of one unit overlap the next.
//  * A block-scaled M=128 MMA occupies the SM's tensor pipe for about 160
//    cycles whatever N is (measured), so small groups stream weights at a
//    fixed rate per MMA: K = 64 per MMA (W4A4) streams twice as fast, and
//    the two-term form's second term rides in the same MMAs.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"
#include "internal.h"

namespace gnf4 {
namespace {

// ------------------------------------------------------------------ quantiser

constexpr int kQThreads = 256;

__device__ __forceinline__ uint32_t cvt_e4m3x2(float hi, float lo) {
  uint16_t pr;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pr) : "f"(hi), "f"(lo));
  return pr;
}

// e4m3 pair (low byte = first element) -> two floats, exactly (through f16).
__device__ __forceinline__ float2 e4m3x2_to_f32(uint32_t pr) {
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((uint16_t)pr));
  const __half2 hh = *reinterpret_cast<const __half2*>(&h);
  return __half22float2(hh);
}

// Exact power of two 2^e for e in [-126, 127].
__device__ __forceinline__ float exp2i(int e) { return __uint_as_float((uint32_t)(e + 127) << 23); }

// floor(log2(a)) of a positive float given by its bits (subnormals included).
__device__ __forceinline__ int ilog2_f32(uint32_t b) {
  return (b >> 23) != 0 ? (int)(b >> 23) - 127 : (31 - __clz((int)b)) - 149;
}

// One thread quantises octet o (8 consecutive k, 16 bytes of bf16); the 4
// lanes of a 32-k block (lanes 4i..4i+3 of the warp, all 32 lanes calling)
// agree on its amax with two shuffles.  TOP = 8: the OCP rule (exponent
// floor(log2 amax) - 8).  SPLIT: the two-term split with one binade of
// headroom (exponent floor(log2 amax) - 7 for both terms): hi of x, then lo
// of the exact residual x - hi.  ok = false: the lane joins the shuffles only.
template <bool SPLIT>
__device__ __forceinline__ void quant_octet(const __nv_bfloat16* __restrict__ x, long long o, bool ok, int lane,
                                            uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                            uint8_t* __restrict__ lo_codes, uint8_t* __restrict__ lo_scales) {
  constexpr int kTop = SPLIT ? 7 : 8;
  const uint4 v = ok ? ldg_nc_u128(x + o * 8) : make_uint4(0u, 0u, 0u, 0u);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  // |bf16| compares like its bit pattern with the sign cleared
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) m = max(m, max(w[i] & 0x7FFFu, (w[i] >> 16) & 0x7FFFu));
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
  // floor(log2(amax)) is the bf16 exponent field - 127; zero and subnormal
  // amax clamp to the smallest scale
  const int ef = (int)(m >> 7);
  const int X = ef == 0 ? -127 : max(ef - 127 - kTop, -127);
  const float inv = __uint_as_float((uint32_t)(127 - X) << 23);  // 2^-X, a normal float for every X here
  float xv[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    xv[2 * i] = __fmul_rn(__uint_as_float(w[i] << 16), inv);  // exact: a power-of-two scaling
    xv[2 * i + 1] = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), inv);
  }
  uint32_t out[2];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t pr = cvt_e4m3x2(xv[2 * i + 1], xv[2 * i]);
    if (i & 1)
      out[i >> 1] |= pr << 16;
    else
      out[i >> 1] = pr;
  }
  if (ok) {
    *reinterpret_cast<uint2*>(codes + o * 8) = make_uint2(out[0], out[1]);
    if ((lane & 3) == 0) scales[o >> 2] = (uint8_t)(X + 127);
  }
  if (SPLIT) {
    // residual in the scaled domain: exact in fp32 (x has 8 significant bits,
    // hi is x rounded to 4 of them, or to the 2^-9 grid below 2^-6)
    float r[8];
    uint32_t rm = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 h = e4m3x2_to_f32((out[i >> 1] >> (16 * (i & 1))) & 0xFFFFu);
      r[2 * i] = __fsub_rn(xv[2 * i], h.x);
      r[2 * i + 1] = __fsub_rn(xv[2 * i + 1], h.y);
      rm = max(rm, max(__float_as_uint(r[2 * i]) & 0x7FFFFFFFu, __float_as_uint(r[2 * i + 1]) & 0x7FFFFFFFu));
    }
    rm = max(rm, __shfl_xor_sync(0xffffffffu, rm, 1));
    rm = max(rm, __shfl_xor_sync(0xffffffffu, rm, 2));
    // lo exponent in absolute terms: floor(log2(max|r| * 2^X)) - 7, clamped
    const int XL = rm == 0 ? -127 : min(max(ilog2_f32(rm) + X - kTop, -127), 127);
    const int d = X - XL;  // >= 0: lo value = r * 2^d, split in two exact steps
    const int d1 = min(d, 126);
    const float m1 = exp2i(d1), m2 = exp2i(d - d1);
    uint32_t lo[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a = __fmul_rn(__fmul_rn(r[2 * i], m1), m2);
      const float b = __fmul_rn(__fmul_rn(r[2 * i + 1], m1), m2);
      const uint32_t pr = cvt_e4m3x2(b, a);
      if (i & 1)
        lo[i >> 1] |= pr << 16;
      else
        lo[i >> 1] = pr;
    }
    if (ok) {
      *reinterpret_cast<uint2*>(lo_codes + o * 8) = make_uint2(lo[0], lo[1]);
      if ((lane & 3) == 0) lo_scales[o >> 2] = (uint8_t)(XL + 127);
    }
  }
}

template <bool SPLIT>
__global__ void __launch_bounds__(kQThreads) quant_mxfp8_kernel(const __nv_bfloat16* __restrict__ x,
                                                                long long octets, uint8_t* __restrict__ codes,
                                                                uint8_t* __restrict__ scales,
                                                                uint8_t* __restrict__ lo_codes,
                                                                uint8_t* __restrict__ lo_scales) {
  griddep_launch_dependents();
  griddep_wait();
  const long long o = (long long)blockIdx.x * kQThreads + threadIdx.x;
  quant_octet<SPLIT>(x, o, o < octets, (int)(threadIdx.x & 31), codes, scales, lo_codes, lo_scales);
}

// The same quantiser over the rows of the groups with at most max_rows rows
// only (the rows the native two-term GEMM reads when it takes the small
// groups); other rows are not written.  Persistent grid: one warp per
// 32-octet chunk of a row at a time, the rows of the selected groups
// enumerated through an exclusive scan of their sizes.
template <bool SPLIT>
__global__ void __launch_bounds__(kQThreads) quant_mxfp8_rows_kernel(const __nv_bfloat16* __restrict__ x, int K,
                                                                     const int* offsets, const int* counts, int E,
                                                                     int M, int max_rows, unsigned* err,
                                                                     uint8_t* __restrict__ codes,
                                                                     uint8_t* __restrict__ scales,
                                                                     uint8_t* __restrict__ lo_codes,
                                                                     uint8_t* __restrict__ lo_scales) {
  __shared__ int off[kMaxExperts + 1], pre[kMaxExperts + 1], scratch[kMaxExperts];
  griddep_launch_dependents();
  griddep_wait();
  if (!load_groups(offsets, counts, E, M, off, scratch, err)) return;
  block_exclusive_scan(E, pre, scratch, [&](int e) {
    const int r = off[e + 1] - off[e];
    return r <= max_rows ? r : 0;
  });
  const int R = pre[E];
  const int lane = threadIdx.x & 31, wpb = kQThreads / 32;
  const int per_row = K / 8;  // octets; a multiple of 4 (K % 32 == 0), so blocks never straddle rows
  const int cpr = (per_row + 31) / 32;  // 32-octet chunks per row
  // one warp per (row, chunk): a row is spread over warps, so no warp walks
  // a long row's chunks one load latency after another
  const long long items = (long long)R * cpr;
  for (long long c = (long long)blockIdx.x * wpb + (threadIdx.x >> 5); c < items; c += (long long)gridDim.x * wpb) {
    const int rr = (int)(c / cpr), b = (int)(c - (long long)rr * cpr) * 32;
    const int g = find_group(pre, E, rr);
    const long long row = off[g] + (rr - pre[g]);
    quant_octet<SPLIT>(x, row * per_row + b + lane, b + lane < per_row, lane, codes, scales, lo_codes, lo_scales);
  }
}

// MXFP4 activations (the W4A4 mode): the OCP rule of the weights, exponent
// floor(log2(amax)) - 2, e2m1 round to nearest even saturating at +-6,
// element 2i in the low nibble.  One thread packs 8 k into 4 bytes.
__global__ void __launch_bounds__(kQThreads) quant_mxfp4_act_kernel(const __nv_bfloat16* __restrict__ x,
                                                                    long long octets, uint8_t* __restrict__ blocks,
                                                                    uint8_t* __restrict__ scales) {
  griddep_launch_dependents();
  griddep_wait();
  const long long o = (long long)blockIdx.x * kQThreads + threadIdx.x;
  const bool ok = o < octets;
  const uint4 v = ok ? ldg_nc_u128(x + o * 8) : make_uint4(0u, 0u, 0u, 0u);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) m = max(m, max(w[i] & 0x7FFFu, (w[i] >> 16) & 0x7FFFu));
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = max(m, __shfl_xor_sync(0xffffffffu, m, 2));
  const int ef = (int)(m >> 7);
  const int X = ef == 0 ? -127 : max(ef - 127 - 2, -127);
  const float inv = __uint_as_float((uint32_t)(127 - X) << 23);
  float xv[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    xv[2 * i] = __fmul_rn(__uint_as_float(w[i] << 16), inv);
    xv[2 * i + 1] = __fmul_rn(__uint_as_float(w[i] & 0xFFFF0000u), inv);
  }
  uint32_t packed;
  asm("{\n\t.reg .b8 q0, q1, q2, q3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 q3, %8, %7;\n\t"
      "mov.b32 %0, {q0, q1, q2, q3};\n\t}"
      : "=r"(packed)
      : "f"(xv[0]), "f"(xv[1]), "f"(xv[2]), "f"(xv[3]), "f"(xv[4]), "f"(xv[5]), "f"(xv[6]), "f"(xv[7]));
  if (ok) {
    reinterpret_cast<uint32_t*>(blocks)[o] = packed;
    if ((threadIdx.x & 3) == 0) scales[o >> 2] = (uint8_t)(X + 127);
  }
}

// ------------------------------------------------------------------ GEMM

// Modes of the native kernel:
//   kW4A8  MXFP8 activations x MXFP4 weights, kind::mxf8f6f4 (K = 32 per MMA)
//   kSplit two-term MXFP8 activations: a unit takes at most 96 rows of a
//          group; its B operand stacks the hi rows (nbx = ceil(rows / 32)
//          boxes of 32 rows) over the lo rows (nbx more boxes), so one MMA
//          with N = 64 * nbx multiplies both terms and the epilogue adds the
//          two halves of the accumulator
//   kW4A4  MXFP4 activations x MXFP4 weights, kind::mxf4 (K = 64 per MMA,
//          both operands packed two codes per byte; two scale bytes per row
//          per MMA)
constexpr int kW4A8 = 0, kSplit = 1, kW4A4 = 2;

template <int MODE>
struct Geo {
  static constexpr int kBT = MODE == kSplit ? 96 : 128;         // rows (tokens) per unit
  static constexpr int kBK = MODE == kW4A4 ? 256 : 128;         // k per stage (128-byte rows in shared memory)
  static constexpr int kMmaK = MODE == kW4A4 ? 64 : 32;         // k per MMA
  static constexpr int kStages = MODE == kSplit ? 5 : 6;
  static constexpr int kAccW = MODE == kSplit ? 192 : 128;      // accumulator columns per buffer
  static constexpr int kARows = MODE == kSplit ? 192 : 128;     // activation rows per stage in shared memory
  static constexpr int kSfBlocks = MODE == kW4A4 ? 2 : 1;       // 4-scale blocks per row per stage
  static constexpr int kSfwWords = 128 * kSfBlocks;             // weight scale words per stage
  static constexpr int kSfaWords = MODE == kSplit ? 256 : 128 * kSfBlocks;  // activation scale words per stage
  static constexpr int kSfCols = 4 * (kSfwWords + kSfaWords) / 128;        // TMEM scale columns per stage
};

constexpr int kBW = 128;  // weight rows per unit = MMA M
constexpr int kBox = 32;  // activation rows per small TMA box
constexpr int kEpiWarp0 = 4;
constexpr int kProd2 = 12;  // second TMA producer warp
constexpr int kPoller = 13;  // tests the stage barriers for the MMA thread
constexpr int kThreads = 14 * 32;
constexpr int kWStageBytes = kBW * 128;  // one 128-byte row per weight row and stage
constexpr int kTmemCols = 512;

// bytes the TMA delivers for a stage's weights: packed codes, two per byte
template <int MODE>
constexpr int w_stage_tx() { return kBW * Geo<MODE>::kBK / 2; }

// scale-loader index of a warp (its ring slot), or -1: warps 2, 3, 8, 9, ...
template <int MODE>
__device__ __forceinline__ int loader_index(int warp) {
  return warp == 2 || warp == 3 ? warp - 2 : (warp >= 8 && warp < 8 + Geo<MODE>::kStages - 2 ? warp - 6 : -1);
}

template <int MODE>
struct MxSmem {
  using G = Geo<MODE>;
  uint8_t w[G::kStages][kWStageBytes];  // 1024-aligned (offset 0)
  uint8_t a[G::kStages][G::kARows * 128];
  uint32_t sfw[G::kStages][G::kSfwWords];  // weight scales of the stage, tcgen05.cp layout
  uint32_t sfa[G::kStages][G::kSfaWords];  // activation scales of the stage
  int off[kMaxExperts + 1];
  int upre[kMaxExperts + 1];
  int scratch[kMaxExperts];
  uint64_t full[G::kStages], empty[G::kStages];  // full: TMA bytes + producer arrival + the scale copies' commit
  uint64_t ldone[G::kStages];                    // abort path only: a loader's scale copies have retired
  uint64_t accf[2], acce[2];
  uint64_t mdone;  // abort path only: every issued MMA has retired
  uint32_t tmem_base;
  uint32_t sready;  // stages whose operands and scales are complete (the poller counts, the MMA thread reads)
  int abort;
};
#define GNF4_MX_CHECK(M)                                                                               \
  static_assert(sizeof(MxSmem<M>) + 1024 <= 227 * 1024, "shared memory budget");                       \
  static_assert(2 * Geo<M>::kAccW + Geo<M>::kSfCols * Geo<M>::kStages <= kTmemCols, "TMEM budget");    \
  static_assert(Geo<M>::kStages <= 6, "scale loaders are warps 2, 3, 8..11");
GNF4_MX_CHECK(kW4A8)
GNF4_MX_CHECK(kSplit)
GNF4_MX_CHECK(kW4A4)
#undef GNF4_MX_CHECK

struct MxArgs {
  const uint8_t* sa;   // activation scales e8m0 [M, K/32] (kSplit: of the hi term; the codes come by TMA)
  const uint8_t* sl;   // kSplit: lo-term scales [M, K/32]
  const uint8_t* sw;   // e8m0 [E, N, K/32]
  const int* offsets;  // [E+1] or null
  const int* counts;   // [E] or null
  __nv_bfloat16* y;    // [M, N]
  unsigned* err;
  int E, N, K, M;
  int max_rows;  // groups with more rows are left to another kernel (their rows of y are not written)
};

struct Unit {
  int e, j, row0, rows;
};

// Partial accumulators per unit (single-term modes): the MMAs of a unit of
// at most 32 (64) rows rotate over 4 (2) accumulators of 32 (64) columns;
// the epilogue adds them in a fixed order.
__device__ __forceinline__ int acc_split(int rows) { return rows <= 32 ? 4 : (rows <= 64 ? 2 : 1); }

template <int MODE>
__device__ __forceinline__ Unit unit_of(const MxSmem<MODE>& s, int E, int u) {
  constexpr int kBT = Geo<MODE>::kBT;
  Unit x;
  x.e = find_group(s.upre, E, u);
  const int local = u - s.upre[x.e];
  const int rows_e = s.off[x.e + 1] - s.off[x.e];
  const int nch = (rows_e + kBT - 1) / kBT;
  x.j = local / nch;
  const int c = local - x.j * nch;
  x.row0 = s.off[x.e] + c * kBT;
  x.rows = min(kBT, s.off[x.e + 1] - x.row0);
  return x;
}

// Shared-memory descriptor of a 32-row x 16-byte scale block (no swizzle;
// 8-row core matrices 128 bytes apart; one 16-byte column, so the leading
// byte offset is unused).
__device__ __forceinline__ uint64_t sdesc_scales(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(128u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  return d;
}

// 32 lanes x 128 bits from shared memory into TMEM, replicated to all four
// 32-lane quarters.
__device__ __forceinline__ void tc_copy_scales(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Instruction descriptor of a block-scaled MMA: operand formats fa / fb, e8m0
// scales, both K-major, M = 128, N = n (multiple of 16); scale-factor ids sf
// (the first byte of the MMA's scales inside their 32-bit TMEM column).
__device__ __forceinline__ uint32_t idesc_mx(uint32_t fa, uint32_t fb, uint32_t n, uint32_t sf) {
  return (sf << 4) | (fa << 7) | (fb << 10) | ((n >> 3) << 17) | (1u << 23) | ((128u >> 4) << 24) | (sf << 29);
}

// A = e2m1 (format 5), B = e4m3 (format 0), K = 32.
__device__ __forceinline__ void tc_mma_mxf8f6f4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// A = B = e2m1 (format 1), packed, K = 64, one e8m0 scale per 32 k.
__device__ __forceinline__ void tc_mma_mxf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// 4 scale bytes starting at an even byte address (two 2-byte loads).
__device__ __forceinline__ uint32_t ld_scales4(const uint8_t* p) {
  const uint16_t* q = reinterpret_cast<const uint16_t*>(p);
  return (uint32_t)__ldg(q) | ((uint32_t)__ldg(q + 1) << 16);
}

__device__ __forceinline__ void sts_u128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// kW4A8 / kW4A4: tm_a / tm_a_big are the activation codes in 32- / 128-row
// boxes (kW4A4: packed bytes).  kSplit: tm_a = hi codes, tm_a_big = lo codes,
// both in 32-row boxes.  tm_w: kW4A8 / kSplit the [E*N] x (K/128) x 128-code
// view expanded to 16-byte slots (16U4_ALIGN16B), tm_w_tail the codes
// [K-128, K) of every row; kW4A4 the [E, N, K/2] bytes in 128-byte boxes.
template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_mx_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_a_big,
                   const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_w_tail,
                   MxArgs p) {
  using G = Geo<MODE>;
  constexpr int kStages = G::kStages;
  constexpr bool SPLIT = MODE == kSplit;
  extern __shared__ uint8_t smem_raw[];
  MxSmem<MODE>& s =
      *reinterpret_cast<MxSmem<MODE>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  unsigned* err = p.err;
  volatile int* abort = &s.abort;

  griddep_launch_dependents();
  griddep_wait();
  if (!load_groups(p.offsets, p.counts, p.E, p.M, s.off, s.scratch, err)) return;
  const int nwt = (p.N + kBW - 1) / kBW;
  block_exclusive_scan(p.E, s.upre, s.scratch, [&](int e) {
    const int r = s.off[e + 1] - s.off[e];
    return r <= p.max_rows ? ((r + G::kBT - 1) / G::kBT) * nwt : 0;
  });
  const int U = s.upre[p.E];
  if ((int)blockIdx.x >= U) return;  // uniform over the block
  const int K = p.K;
  const int nk = (K + G::kBK - 1) / G::kBK;
  // the last stage reads [K - kBK, K) and skips the MMAs already covered
  auto stage_k0 = [&](int kt) { return min(kt * G::kBK, K - G::kBK); };

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&s.full[i], 2);
      mbar_init(&s.empty[i], 1);
      mbar_init(&s.ldone[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.accf[i], 1);
      mbar_init(&s.acce[i], 4);
    }
    mbar_init(&s.mdone, 1);
    s.sready = 0;
    s.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_a_big);
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_w_tail);
  }
  if (warp == 1) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  const int sf_col0 = 2 * G::kAccW;

  if (warp == 0 || warp == kProd2) {
    // ------------------------------------------------------------ TMA producers
    const int pi = warp == 0 ? 0 : 1;
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
        const Unit x = unit_of<MODE>(s, p.E, u);
        const bool big = x.rows > kBox;
        const int nbx = (x.rows + kBox - 1) / kBox;  // kSplit: 32-row boxes per term
        const int wrow = x.e * p.N + x.j * kBW;
        for (int kt = 0; kt < nk; ++kt, ++it) {
          if ((it & 1) != pi) continue;
          const int st = it % kStages, use = it / kStages;
          if (it >= kStages && !(ok = mbar_wait(&s.empty[st], (use - 1) & 1, err, abort))) break;
          const int k0 = stage_k0(kt);
          const int abytes = SPLIT ? 2 * nbx * kBox * 128 : (big ? G::kBT : kBox) * 128;
          mbar_arrive_expect_tx(&s.full[st], w_stage_tx<MODE>() + abytes);
          if (MODE == kW4A4)
            tma_load_3d(s.w[st], &tm_w, &s.full[st], k0 / 2, x.j * kBW, x.e);
          else if (k0 != kt * G::kBK)
            tma_load_2d(s.w[st], &tm_w_tail, &s.full[st], 0, wrow);
          else
            tma_load_3d(s.w[st], &tm_w, &s.full[st], 0, kt, wrow);
          const int ax = MODE == kW4A4 ? k0 / 2 : k0;  // activation bytes: packed in kW4A4
          if (SPLIT) {
            for (int b = 0; b < nbx; ++b) {
              tma_load_2d(s.a[st] + b * kBox * 128, &tm_a, &s.full[st], ax, x.row0 + b * kBox);
              tma_load_2d(s.a[st] + (nbx + b) * kBox * 128, &tm_a_big, &s.full[st], ax, x.row0 + b * kBox);
            }
          } else {
            tma_load_2d(s.a[st], big ? &tm_a_big : &tm_a, &s.full[st], ax, x.row0);
          }
        }
      }
      if (!ok)  // drain loads still in flight before shared memory goes away
        for (int i = max(0, it - kStages); i < it; ++i)
          if ((i & 1) == pi) mbar_drain(&s.full[i % kStages], (i / kStages) & 1);
    }
  } else if (loader_index<MODE>(warp) >= 0) {
    // ------------------------------------------------------------ scale loaders
    // Loader i fills ring slot i only.  Lane l serves rows l + 32c of the
    // weight tile (c < 4) and of the activation operand (c < 4, or < 8 for the
    // stacked hi / lo rows of kSplit); per row it copies 4 scale bytes per
    // 4-scale block of the stage (kW4A4: two blocks).  Rows outside the tile
    // or the group get scale 2^0 (their products are never stored).
    const int li = loader_index<MODE>(warp);
    const int nsb = K / 32;
    const uint8_t* swb = p.sw;
    int it = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < U && ok; u += gridDim.x) {
      const Unit x = unit_of<MODE>(s, p.E, u);
      const int hrows = kBox * ((x.rows + kBox - 1) / kBox);  // kSplit: hi rows of the stacked operand
      for (int kt = 0; kt < nk; ++kt, ++it) {
        const int st = it % kStages, use = it / kStages;
        if (st != li) continue;
        if (it >= kStages && !(ok = mbar_wait(&s.empty[st], (use - 1) & 1, err, abort))) break;
        const int b0 = stage_k0(kt) / 32;  // even: K % 64 == 0
#pragma unroll
        for (int bl = 0; bl < G::kSfBlocks; ++bl) {
          uint32_t wv[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const int n = x.j * kBW + lane + 32 * c;
            wv[c] = n < p.N ? ld_scales4(swb + ((size_t)x.e * p.N + (size_t)n) * (size_t)nsb + b0 + 4 * bl)
                            : 0x7F7F7F7Fu;
          }
          sts_u128(smem_u32(&s.sfw[st][bl * 128 + lane * 4]), wv[0], wv[1], wv[2], wv[3]);
        }
        constexpr int kARowsSf = SPLIT ? 256 : 128;  // activation rows with a scale block
#pragma unroll
        for (int bl = 0; bl < G::kSfaWords / 128; ++bl) {
          uint32_t av[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            // kSplit: block bl covers stacked rows 128 bl + ..; kW4A4: scale block bl of rows 0..127
            const int m = (SPLIT ? bl * 128 : 0) + lane + 32 * c;
            const bool lo_row = SPLIT && m >= hrows;
            const int rr = lo_row ? m - hrows : m;
            const uint8_t* src = lo_row ? p.sl : p.sa;
            const int boff = MODE == kW4A4 ? 4 * bl : 0;
            av[c] = (rr < x.rows && m < kARowsSf) ? ld_scales4(src + (size_t)(x.row0 + rr) * (size_t)nsb + b0 + boff)
                                                  : 0x7F7F7F7Fu;
          }
          sts_u128(smem_u32(&s.sfa[st][bl * 128 + lane * 4]), av[0], av[1], av[2], av[3]);
        }
        fence_proxy_async_smem();  // the tensor core reads these through the async proxy
        __syncwarp();
        if (lane == 0) {
          const uint32_t col = tmem + (uint32_t)(sf_col0 + G::kSfCols * st);
#pragma unroll
          for (int bl = 0; bl < G::kSfwWords / 128; ++bl)
            tc_copy_scales(col + 4u * (uint32_t)bl, sdesc_scales(smem_u32(&s.sfw[st][bl * 128])));
#pragma unroll
          for (int bl = 0; bl < G::kSfaWords / 128; ++bl)
            tc_copy_scales(col + 4u * (uint32_t)(G::kSfwWords / 128 + bl),
                           sdesc_scales(smem_u32(&s.sfa[st][bl * 128])));
          tc_commit(&s.full[st]);
        }
      }
    }
    if (!ok && lane == 0) {  // abort: the copies already issued retire before TMEM is released
      tc_commit(&s.ldone[li]);
      mbar_drain(&s.ldone[li], 0);
    }
  } else if (warp == kPoller) {
    // ------------------------------------------------------------ stage poller
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x)
        for (int kt = 0; kt < nk; ++kt, ++it) {
          if (!(ok = mbar_wait(&s.full[it % kStages], (uint32_t)(it / kStages) & 1u, err, abort))) break;
          st_release_shared(&s.sready, (uint32_t)(it + 1));
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, uc = 0;
      uint32_t ready = 0;  // stages the poller had counted complete at the last read
      bool ok = true;
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x, ++uc) {
        const Unit x = unit_of<MODE>(s, p.E, u);
        const int ab = uc & 1;
        if (uc >= 2 && !(ok = mbar_wait(&s.acce[ab], ((uc >> 1) - 1) & 1, err, abort))) break;
        tc_fence_after();
        const uint32_t n_mma =
            SPLIT ? (uint32_t)(2 * kBox * ((x.rows + kBox - 1) / kBox)) : (uint32_t)((x.rows + 15) & ~15);
        const uint32_t d_tmem = tmem + (uint32_t)(ab * G::kAccW);
        const int nsplit = SPLIT ? 1 : acc_split(x.rows);
        const uint32_t sub_w = (uint32_t)(G::kAccW / nsplit);
        for (int kt = 0; kt < nk; ++kt, ++it) {
          const int st = it % kStages;
          const uint32_t ph = (uint32_t)(it / kStages) & 1u;
          (void)ph;
          // The poller warp tests the stage barriers and counts complete
          // stages; this thread re-reads the count only after using up the
          // last value.  An mbarrier test here costs ~220 cycles while MMAs
          // are in flight (measured), enough to let the tensor pipe run dry.
          if ((int)ready <= it) ready = ld_acquire_shared(&s.sready);
          if ((int)ready <= it) {
            const long long t0 = clock64();
            while ((int)(ready = ld_acquire_shared(&s.sready)) <= it) {
              if (*abort) {
                ok = false;
                break;
              }
              if (clock64() - t0 > kSpinLimitCycles) {
                atomicOr(err, GNF4_DEVERR_TIMEOUT);
                *abort = 1;
                ok = false;
                break;
              }
            }
            if (!ok) break;
          }
          tc_fence_after();
          const uint32_t t_sfw = tmem + (uint32_t)(sf_col0 + G::kSfCols * st);
          const uint32_t t_sfa = t_sfw + 4u * (uint32_t)(G::kSfwWords / 128);
          const uint32_t w_addr = smem_u32(s.w[st]), a_addr = smem_u32(s.a[st]);
          const int j0 = (kt * G::kBK - stage_k0(kt)) / G::kMmaK;
          constexpr int kSteps = G::kBK / G::kMmaK;  // 4 MMAs per stage, 32 bytes of each row apiece
          for (int j = j0; j < kSteps; ++j) {
            const int q = kt * kSteps + j;  // MMA step of the unit (every unit has at least 4)
            const uint32_t d = d_tmem + (uint32_t)(q % nsplit) * sub_w;
            const uint64_t da = sdesc_k_sw128(w_addr + 32 * j), db = sdesc_k_sw128(a_addr + 32 * j);
            const uint32_t acc = q >= nsplit;
            if (MODE == kW4A4) {
              // two scales per row per MMA: column set j / 2, bytes 2 (j % 2) and 2 (j % 2) + 1
              const uint32_t sf = 2u * (uint32_t)(j & 1), cs = 4u * (uint32_t)(j >> 1);
              tc_mma_mxf4(d, da, db, idesc_mx(1u, 1u, n_mma, sf), (t_sfw + cs) | (sf << 30), (t_sfa + cs) | (sf << 30),
                          acc);
            } else {
              tc_mma_mxf8f6f4(d, da, db, idesc_mx(5u, 0u, n_mma, (uint32_t)j), t_sfw | ((uint32_t)j << 30),
                              t_sfa | ((uint32_t)j << 30), acc);
            }
          }
          tc_commit(&s.empty[st]);
        }
        if (!ok) break;
        tc_commit(&s.accf[ab]);
      }
      if (!ok) {
        // abort: let every MMA already issued retire before TMEM is released
        tc_commit(&s.mdone);
        mbar_drain(&s.mdone, 0);
      }
    }
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16);
    int uc = 0;
    for (int u = blockIdx.x; u < U; u += gridDim.x, ++uc) {
      const Unit x = unit_of<MODE>(s, p.E, u);
      const int ab = uc & 1;
      if (!mbar_wait(&s.accf[ab], (uc >> 1) & 1, err, abort)) break;
      tc_fence_after();
      const int n = x.j * kBW + q * 32 + lane;
      __nv_bfloat16* ycol = p.y + (size_t)x.row0 * p.N + n;
      const int nsplit = SPLIT ? 1 : acc_split(x.rows);
      // kSplit: the lo term of row i sits hrows columns after its hi term
      const int hrows = kBox * ((x.rows + kBox - 1) / kBox);
      for (int c = 0; c * 32 < x.rows; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_lane + (uint32_t)(ab * G::kAccW + c * 32), v);
        tmem_wait_ld();
        const int nparts = SPLIT ? 2 : nsplit;
        for (int j = 1; j < nparts; ++j) {  // partial accumulators (or the lo term), summed in a fixed order
          uint32_t w2[32];
          const int off = SPLIT ? hrows : j * (G::kAccW / nsplit);
          tmem_ld_32x32b_x32(t_lane + (uint32_t)(ab * G::kAccW + off + c * 32), w2);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) + __uint_as_float(w2[i]));
        }
        const int lim = min(32, x.rows - c * 32);
        if (n < p.N) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < lim) ycol[(size_t)(c * 32 + i) * p.N] = __float2bfloat16_rn(__uint_as_float(v[i]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s.acce[ab]);
    }
  }

  // Normal path: the epilogue has consumed every accumulator, so every MMA
  // and TMEM access has completed here.
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_quant_mxfp8(const __nv_bfloat16* x, long long elems, uint8_t* codes, uint8_t* scales,
                               uint8_t* lo_codes, uint8_t* lo_scales, cudaStream_t stream) {
  const long long octets = elems / 8;
  if (octets == 0) return cudaSuccess;
  const long long blocks = (octets + kQThreads - 1) / kQThreads;
  if (lo_codes != nullptr)
    return launch_pdl(quant_mxfp8_kernel<true>, dim3((unsigned)blocks), dim3(kQThreads), 0, stream, x, octets, codes,
                      scales, lo_codes, lo_scales);
  return launch_pdl(quant_mxfp8_kernel<false>, dim3((unsigned)blocks), dim3(kQThreads), 0, stream, x, octets, codes,
                    scales, lo_codes, lo_scales);
}

cudaError_t launch_quant_mxfp8_split_rows(const __nv_bfloat16* x, int K, const int* offsets, const int* counts,
                                          int E, int M, int max_rows, unsigned* err, uint8_t* hi_codes,
                                          uint8_t* hi_scales, uint8_t* lo_codes, uint8_t* lo_scales, int num_sms,
                                          cudaStream_t stream) {
  const int grid = num_sms * (2048 / kQThreads);
  return launch_pdl(quant_mxfp8_rows_kernel<true>, dim3((unsigned)grid), dim3(kQThreads), 0, stream, x, K, offsets,
                    counts, E, M, max_rows, err, hi_codes, hi_scales, lo_codes, lo_scales);
}

cudaError_t launch_quant_mxfp4_act(const __nv_bfloat16* x, long long elems, uint8_t* blocks, uint8_t* scales,
                                   cudaStream_t stream) {
  const long long octets = elems / 8;
  if (octets == 0) return cudaSuccess;
  const long long nb = (octets + kQThreads - 1) / kQThreads;
  return launch_pdl(quant_mxfp4_act_kernel, dim3((unsigned)nb), dim3(kQThreads), 0, stream, x, octets, blocks, scales);
}

template <int MODE>
static size_t smem_bytes_t() { return sizeof(MxSmem<MODE>) + 1024; }

size_t gemm_mx_smem_bytes(int mode) {
  return mode == kW4A4 ? smem_bytes_t<kW4A4>() : (mode == kSplit ? smem_bytes_t<kSplit>() : smem_bytes_t<kW4A8>());
}
int gemm_mx_rows_per_unit(int mode) {
  return mode == kW4A4 ? Geo<kW4A4>::kBT : (mode == kSplit ? Geo<kSplit>::kBT : Geo<kW4A8>::kBT);
}
int gemm_mx_k_per_stage(int mode) { return mode == kW4A4 ? Geo<kW4A4>::kBK : Geo<kW4A8>::kBK; }
int gemm_mx_weight_rows_per_unit() { return kBW; }
int gemm_mx_small_box_rows() { return kBox; }

template <int MODE>
static cudaError_t launch_gemm_mx_t(const CUtensorMap& tm_a, const CUtensorMap& tm_a_big, const CUtensorMap& tm_w,
                                    const CUtensorMap& tm_w_tail, const MxArgs& p, int grid, cudaStream_t stream) {
  static std::atomic<bool> configured[64];
  const cudaError_t e = set_smem_limit_once(gemm_mx_kernel<MODE>, (int)smem_bytes_t<MODE>(), configured);
  if (e != cudaSuccess) return e;
  return launch_pdl(gemm_mx_kernel<MODE>, dim3(grid), dim3(kThreads), smem_bytes_t<MODE>(), stream, tm_a, tm_a_big,
                    tm_w, tm_w_tail, p);
}

cudaError_t launch_gemm_mx(int mode, const CUtensorMap& tm_a, const CUtensorMap& tm_a_big, const CUtensorMap& tm_w,
                           const CUtensorMap& tm_w_tail, const uint8_t* a_scales, const uint8_t* lo_scales,
                           const uint8_t* w_scales, const int* offsets, const int* counts, __nv_bfloat16* y,
                           unsigned* err, int E, int N, int K, int M, int grid, cudaStream_t stream,
                           int max_rows) {
  MxArgs p{a_scales, lo_scales, w_scales, offsets, counts, y, err, E, N, K, M, max_rows};
  if (mode == kW4A4) return launch_gemm_mx_t<kW4A4>(tm_a, tm_a_big, tm_w, tm_w_tail, p, grid, stream);
  if (mode == kSplit) return launch_gemm_mx_t<kSplit>(tm_a, tm_a_big, tm_w, tm_w_tail, p, grid, stream);
  return launch_gemm_mx_t<kW4A8>(tm_a, tm_a_big, tm_w, tm_w_tail, p, grid, stream);
}

}  // namespace gnf4
