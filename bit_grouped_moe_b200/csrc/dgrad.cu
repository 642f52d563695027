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
//  * a decode group of four warps decodes it through the pair table in its natural
//    order, weight row n with k contiguous, as two 128B-swizzled halves
//    [64 n][64 k] bf16.  The MMA reads this tile as an MN-major B operand
//    (MN = k, the output width; K = n, the contraction), so no transpose
//    happens anywhere: a quarter warp stores one 128-byte row with eight
//    conflict-free 16-byte stores, and a warp reads 128 contiguous packed bytes.
// D[r, k] accumulates in TMEM (lane = row r, column = k).  Work unit = (expert
// e, chunk of <= 128 of its rows, 128-wide k tile); a persistent grid strides
// over the units.  Warp roles: four decode groups of 4 warps that take the
// stages in turn (one group's waits, proxy fence and barrier overlap the
// others' decode), a dY producer, a weight producer, an MMA issuer, 4
// epilogue warps and a stage poller (it tests the dY and decoded-tile
// barriers and publishes a count of complete stages that the MMA thread
// reads with a load-acquire).
//
// Every stage waits on memory twice, for the packed weights and block scales
// (mostly DRAM: the stacks are larger than L2) and for the dY tile (mostly L2:
// the k tiles of one row chunk run side by side).  Each source has its own
// queue, deep enough to cover its latency:
//  * dY tiles: a 4-deep TMA ring, released by the MMAs' commit;
//  * packed weight blocks: an 8-deep TMA ring of 4 KB slots, released by the
//    decode group once it has read a block;
//  * block scales: each decode thread keeps the raw scales of its group's
//    next 4 stages (16 stages of the CTA) in registers, a plain load issued
//    that far ahead, and stores one stage ahead into the group's
//    double-buffered table.
// Four decoded weight tiles are in flight (one per group) and two
// accumulators, so copies, MMAs, decode and the epilogue of the previous unit
// overlap.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace gnf4 {
namespace {

constexpr int kDecWarps = 4;                    // warps of one decode group
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecGroups = 4;                   // groups take stages in turn
constexpr int kProdWarp = kDecGroups * kDecWarps, kWProdWarp = kProdWarp + 1, kMmaWarp = kProdWarp + 2;
constexpr int kEpiWarp0 = kProdWarp + 3;
constexpr int kPollWarp = kEpiWarp0 + 4;        // tests the stage barriers for the MMA thread
constexpr int kThreads = (kPollWarp + 1) * 32;  // 768
constexpr int kRing = 4;                       // dY stages in flight
constexpr int kWRing = 8;                      // packed-weight stages in flight
constexpr int kSQ = 4;                         // stages of block scales queued in registers
constexpr int kTBuf = 4;                       // decoded weight tiles in flight
static_assert(kTBuf <= kRing, "a decoded tile is released through the ring's MMA-done barriers");
// A group waits on a ring slot's phase P only after it has itself waited on
// phase P-1 (a parity wait cannot tell the two apart): the stage that used
// the slot one lap earlier must belong to the same group.
static_assert(kRing % kDecGroups == 0 && kWRing % kDecGroups == 0, "ring depths must be multiples of the group count");
constexpr int kBR = 128;                   // rows per unit (MMA M)
constexpr int kBKt = 128;                  // k per unit (MMA N)
constexpr int kBN = 64;                    // n per stage (four k-steps of 16)
constexpr int kYBytes = kBR * kBN * 2;     // 16 KB
constexpr int kTBytes = kBKt * kBN * 2;    // 16 KB
constexpr int kTHalf = kBN * 128;          // one 64-k half of the decoded tile: 64 rows of 128 bytes
constexpr int kWBytes = kBN * kBKt / 2;    // 4 KB
constexpr int kTmemCols = 2 * kBKt;  // two accumulators

struct DSmem {
  uint8_t y[kRing][kYBytes];  // dY tiles (1024-aligned for the 128-byte swizzle)
  uint8_t t[kTBuf][kTBytes];  // decoded W tiles, two 64-k halves each
  uint8_t w[kWRing][kWBytes];  // packed weight blocks
  uint32_t lut[kLutWords];    // pair table, 128-byte entries (32 lanes)
  uint32_t sc[kDecGroups][2][kBN][4];  // per decode group, two stages of block scales (bf16x2): 64 rows x (2 NF4 | 4 MXFP4) blocks of the k tile
  int off[kMaxExperts + 1];
  int upre[kMaxExperts + 1];
  int scratch[kMaxExperts];
  uint64_t full[kRing], mdone[kRing], wfull[kWRing], wempty[kWRing], decoded[kTBuf], accf[2], acce[2], drain;
  uint32_t tmem_base;
  uint32_t sready;  // stages whose dY tile and decoded tile are complete (the poller counts, the MMA thread reads)
  int abort;
};

static_assert(sizeof(DSmem) + 1024 <= 227 * 1024, "shared memory budget");

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

// Shared-memory descriptor of an MN-major operand in the 128-byte swizzle:
// 64 consecutive MN elements (bf16) fill a 128-byte row, eight rows of
// consecutive K form a 1 KB atom; lbo = bytes to the next 64 MN elements,
// sbo = bytes to the next 8 K rows.
__device__ __forceinline__ uint64_t sdesc_mn_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);  // start address
  d |= (uint64_t)(lbo >> 4) << 16;           // leading byte offset: next 64 MN elements
  d |= (uint64_t)(sbo >> 4) << 32;           // stride byte offset: next 8 K rows
  d |= (uint64_t)1u << 46;                   // descriptor version for tcgen05
  d |= (uint64_t)2u << 61;                   // 128-byte swizzle
  return d;
}

__device__ __forceinline__ void sts_u128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// a read of the pair table, which is constant once built: free to schedule
__device__ __forceinline__ uint32_t lds_lut(uint32_t addr) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
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
  build_pair_lut<FMT>(s.lut, tid, kThreads);
  griddep_wait();
  if (!load_groups(p.offsets, p.counts, p.E, p.M, s.off, s.scratch, err)) return;
  const int nkt = (K + kBKt - 1) / kBKt;
  block_exclusive_scan(p.E, s.upre, s.scratch, [&](int e) { return ((s.off[e + 1] - s.off[e] + kBR - 1) / kBR) * nkt; });
  const int U = s.upre[p.E];
  if ((int)blockIdx.x >= U) return;  // uniform over the block
  const int ns = (N + kBN - 1) / kBN;

  if (tid == 0) {
    for (int i = 0; i < kRing; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.mdone[i], 1);
    }
    for (int i = 0; i < kWRing; ++i) {
      mbar_init(&s.wfull[i], 1);
      mbar_init(&s.wempty[i], 1);
    }
    for (int i = 0; i < kTBuf; ++i) mbar_init(&s.decoded[i], kDecWarps);  // one arrival per warp of a group
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s.accf[i], 1);
      mbar_init(&s.acce[i], 128);
    }
    mbar_init(&s.drain, 1);
    s.abort = 0;
    s.sready = 0;
    fence_mbar_init();
    prefetch_tmap(&tm_y);
    prefetch_tmap(&tm_w);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&s.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  const int nsc = FMT == 0 ? K / 64 : K / 32;        // scales per weight row
  constexpr int spk = FMT == 0 ? kBKt / 64 : kBKt / 32;                  // scale blocks of a row in one k tile
  constexpr int kSpt = (kBN * spk + kDecThreads - 1) / kDecThreads;  // block scales per decode thread per stage
  constexpr int kItems = kBN * (kBKt / 8) / kDecThreads;             // 16-byte chunks per decode thread per stage

  // The CTA's stage stream: stage g = (unit u, n block sb), units strided by the grid.
  struct Pos {
    int u, sb;
  };
  auto next = [&](Pos q) {
    if (++q.sb >= ns) {
      q.sb = 0;
      q.u += (int)gridDim.x;
    }
    return q;
  };

  if (warp == kProdWarp) {
    // ------------------------------------------------------------ dY producer
    if (lane == 0) {
      int g = 0, xu = -1;
      DUnit x{};
      for (Pos q{(int)blockIdx.x, 0}; q.u < U && !*abort; q = next(q), ++g) {
        const int b = g % kRing;
        if (g >= kRing && !mbar_wait(&s.mdone[b], (uint32_t)((g - kRing) / kRing) & 1u, err, abort)) break;
        if (q.u != xu) {
          x = dunit_of(s, p.E, nkt, q.u);
          xu = q.u;
        }
        mbar_arrive_expect_tx(&s.full[b], kYBytes);
        tma_load_2d(s.y[b], &tm_y, &s.full[b], q.sb * kBN, x.row0);
      }
      if (*abort)  // let the last copies land before shared memory goes away
        for (int i = max(0, g - kRing); i < g; ++i) mbar_drain(&s.full[i % kRing], (uint32_t)(i / kRing) & 1u);
    }
  } else if (warp == kWProdWarp) {
    // ------------------------------------------------------------ weight producer
    if (lane == 0) {
      int g = 0, xu = -1;
      DUnit x{};
      for (Pos q{(int)blockIdx.x, 0}; q.u < U && !*abort; q = next(q), ++g) {
        const int b = g % kWRing;
        if (g >= kWRing && !mbar_wait(&s.wempty[b], (uint32_t)((g - kWRing) / kWRing) & 1u, err, abort)) break;
        if (q.u != xu) {
          x = dunit_of(s, p.E, nkt, q.u);
          xu = q.u;
        }
        mbar_arrive_expect_tx(&s.wfull[b], kWBytes);
        tma_load_3d(s.w[b], &tm_w, &s.wfull[b], x.kt * (kBKt / 2), q.sb * kBN, x.e);
      }
      if (*abort)
        for (int i = max(0, g - kWRing); i < g; ++i) mbar_drain(&s.wfull[i % kWRing], (uint32_t)(i / kWRing) & 1u);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_m128((uint32_t)kBKt) | (1u << 16);  // B (the decoded W tile) MN-major
      int g = 0, uc = 0;
      uint32_t ready = 0;  // stages the poller had counted complete at the last read
      bool ok = true;
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x, ++uc) {
        const int ab = uc & 1;
        if (uc >= 2 && !(ok = mbar_wait(&s.acce[ab], (uint32_t)((uc >> 1) - 1) & 1u, err, abort))) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(ab * kBKt);
        for (int sb = 0; sb < ns; ++sb, ++g) {
          const int b = g % kRing, tb = g % kTBuf;
          // The poller warp tests the dY and decoded-tile barriers and counts
          // the complete stages; this thread re-reads the count only when it
          // has used up the last one it read (an mbarrier test here costs
          // ~220 cycles while MMAs are in flight, measured in the forward
          // GEMM), and one fence after each fresh read covers every stage it
          // counted.
          if ((int)ready <= g) {
            ready = ld_acquire_shared(&s.sready);
            if ((int)ready <= g) {
              const long long t0 = clock64();
              while ((int)(ready = ld_acquire_shared(&s.sready)) <= g) {
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
          }
          const uint32_t ya = smem_u32(s.y[b]), ta = smem_u32(s.t[tb]);
#pragma unroll
          for (int q = 0; q < kBN / 16; ++q)
            tc_mma_ss(d_tmem, sdesc_k_sw128(ya + q * 32), sdesc_mn_sw128(ta + q * 16 * 128, kTHalf, 1024), idesc,
                      (sb | q) != 0);
          tc_commit(&s.mdone[b]);
        }
        if (!ok) break;
        tc_commit(&s.accf[ab]);
      }
      if (!ok) {  // let every issued MMA retire before TMEM is released
        tc_commit(&s.drain);
        mbar_drain(&s.drain, 0);
      }
    }
  } else if (warp == kPollWarp) {
    // ------------------------------------------------------------ stage poller
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < U && ok; u += gridDim.x)
        for (int sb = 0; sb < ns; ++sb, ++g) {
          if (!(ok = mbar_wait(&s.full[g % kRing], (uint32_t)(g / kRing) & 1u, err, abort))) break;
          if (!(ok = mbar_wait(&s.decoded[g % kTBuf], (uint32_t)(g / kTBuf) & 1u, err, abort))) break;
          st_release_shared(&s.sready, (uint32_t)(g + 1));
        }
    }
  } else if (warp < kProdWarp) {
    // ------------------------------------------------------------ decode
    // group grp takes the stages g = grp (mod kDecGroups); gtid = thread of the group
    const int grp = warp / kDecWarps, gtid = tid - grp * kDecThreads;
    const uint32_t lut_lane = smem_u32(s.lut) + (uint32_t)lane * 4u;  // this lane's column of the pair table
    // Raw block scale j (of kSpt) of this thread for the stage at position q;
    // the unit's view is recomputed only when q moves to another unit.  A row
    // past N has no scale and reads as 0, which stores as a zero factor: NF4
    // keeps the fp32 bits (+0 converts to the bf16 zero), MXFP4 marks a real
    // e8m0 byte with bit 8.
    int xs_u = -1;
    DUnit xs{};
    auto scale_raw = [&](Pos q, int j) -> uint32_t {
      const int vi = gtid + kDecThreads * j;
      if (q.u >= U || vi >= kBN * spk) return 0u;
      if (q.u != xs_u) {
        xs = dunit_of(s, p.E, nkt, q.u);
        xs_u = q.u;
      }
      const DUnit& x = xs;
      const int rr = vi / spk, bb = vi - rr * spk;
      const int n = q.sb * kBN + rr;
      if (n >= N) return 0u;
      const int blk = min(x.kt * spk + bb, nsc - 1);  // past K: any valid scale, never stored
      const size_t idx = ((size_t)x.e * N + (size_t)n) * (size_t)nsc + (size_t)blk;
      return FMT == 0 ? __float_as_uint(__ldg(reinterpret_cast<const float*>(p.scales) + idx))
                      : 0x100u | (uint32_t)__ldg(reinterpret_cast<const uint8_t*>(p.scales) + idx);
    };
    // bf16x2 scale pair into the group's sc[buf]
    auto scale_store = [&](int buf, int j, uint32_t raw) {
      const int vi = gtid + kDecThreads * j;
      if (vi >= kBN * spk) return;
      const int rr = vi / spk, bb = vi - rr * spk;
      s.sc[grp][buf][rr][bb] = FMT == 0 ? f32_to_bf16x2_rn(__uint_as_float(raw))
                                        : ((raw & 0x100u) ? e8m0_to_bf16x2(raw & 0xFFu) : 0u);
    };
    auto dec_barrier = [&]() { asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(kDecThreads) : "memory"); };
    auto next_own = [&](Pos q) {  // this group's next stage
#pragma unroll
      for (int i = 0; i < kDecGroups; ++i) q = next(q);
      return q;
    };

    Pos sp{(int)blockIdx.x, 0};
    for (int i = 0; i < grp; ++i) sp = next(sp);  // the group's first stage
#pragma unroll
    for (int j = 0; j < kSpt; ++j) scale_store(0, j, scale_raw(sp, j));
    // Raw block scales of the group's next kSQ stages wait in registers (its
    // i-th stage in slot i % kSQ): a load is issued kSQ of the group's stages
    // before its value is stored.
    uint32_t rq[kSQ][kSpt];
#pragma unroll
    for (int i = 1; i <= kSQ; ++i) {
      sp = next_own(sp);
#pragma unroll
      for (int j = 0; j < kSpt; ++j) rq[i % kSQ][j] = scale_raw(sp, j);
    }
    sp = next_own(sp);  // the group's stage kSQ + 1
    dec_barrier();
    // The group's stages, flattened and unrolled by kSQ so that every queue
    // slot index is a compile-time constant.  After an abort the loop still
    // runs to its end (no waits, garbage results), so every decode warp
    // reaches every named barrier.
    const int G = ((U - 1 - (int)blockIdx.x) / (int)gridDim.x + 1) * ns;  // the CTA's stages
    const int Gi = (G - grp + kDecGroups - 1) / kDecGroups;               // this group's
    for (int i0 = 0; i0 < Gi; i0 += kSQ) {
#pragma unroll
      for (int d = 0; d < kSQ; ++d) {
        const int i = i0 + d, g = grp + kDecGroups * i;
        if (i < Gi) {  // uniform over the group
          const int wb = g % kWRing, tb = g % kTBuf, sb2 = i & 1;  // sb2: scale table of this stage
          // this stage's packed weights have landed, and the MMAs of stage g-kTBuf no longer read t[tb]
          if (!*abort) mbar_wait(&s.wfull[wb], (uint32_t)(g / kWRing) & 1u, err, abort);
          if (g >= kTBuf && !*abort)
            mbar_wait(&s.mdone[(g - kTBuf) % kRing], (uint32_t)((g - kTBuf) / kRing) & 1u, err, abort);
          // item (n, c): packed bytes 4c .. 4c+3 of weight row n, i.e. k = 8c .. 8c+7
          // of the tile, decoded into the 16-byte chunk c % 8 of row n in half c / 8
          const uint32_t wbase = smem_u32(s.w[wb]);
          const uint32_t tbase = smem_u32(s.t[tb]);
          // item (n, c): packed bytes 4c .. 4c+3 of weight row n, i.e. k = 8c .. 8c+7
          // of the tile, decoded into the 16-byte chunk c % 8 of row n in half c / 8
#pragma unroll
          for (int j = 0; j < kItems; ++j) {
            const int item = gtid + kDecThreads * j;
            const int c = item & 15, n = item >> 4;
            const uint32_t word = lds_u32(wbase + (uint32_t)(n * (kBKt / 2) + 4 * c));
            const uint32_t sc = s.sc[grp][sb2][n][FMT == 0 ? (c >> 3) : (c >> 2)];
            // byte i holds k = 8c+2i (low half of its pair) and 8c+2i+1
            const uint32_t p0 = bf16x2_mul(lds_lut(lut_lane + ((word << 7) & 0x7F80u)), sc);
            const uint32_t p1 = bf16x2_mul(lds_lut(lut_lane + ((word >> 1) & 0x7F80u)), sc);
            const uint32_t p2 = bf16x2_mul(lds_lut(lut_lane + ((word >> 9) & 0x7F80u)), sc);
            const uint32_t p3 = bf16x2_mul(lds_lut(lut_lane + ((word >> 17) & 0x7F80u)), sc);
            sts_u128(tbase + (uint32_t)((c >> 3) * kTHalf + n * 128 + (((c & 7) ^ (n & 7)) << 4)), p0, p1, p2, p3);
          }
          // every thread orders its generic-proxy writes of t[tb] before the
          // MMA's reads; one lane per warp then signals (32 arrivals on one
          // word would serialise)
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&s.decoded[tb]);
          const int q1 = (d + 1) % kSQ;  // slot of the group's stage i+1, refilled with its stage i+1+kSQ
#pragma unroll
          for (int j = 0; j < kSpt; ++j) {
            scale_store(sb2 ^ 1, j, rq[q1][j]);
            rq[q1][j] = scale_raw(sp, j);
          }
          sp = next_own(sp);
          dec_barrier();  // sc[sb2 ^ 1] written, sc[sb2] and w[wb] no longer read
          if (gtid == 0) mbar_arrive(&s.wempty[wb]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // a warp reaches TMEM lanes 32 (warp % 4) .. +31: these rows
    const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16);
    const int r = q * 32 + lane;
    int uc = 0;
    for (int u = blockIdx.x; u < U; u += gridDim.x, ++uc) {
      const DUnit x = dunit_of(s, p.E, nkt, u);
      const int ab = uc & 1;
      if (!mbar_wait(&s.accf[ab], (uint32_t)(uc >> 1) & 1u, err, abort)) break;
      tc_fence_after();
      const int k0 = x.kt * kBKt;
      for (int c = 0; c < kBKt / 32; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_lane + (uint32_t)(ab * kBKt + c * 32), v);
        tmem_wait_ld();
        const int kc = k0 + c * 32;
        if (r < x.rows && kc < K) {
          __nv_bfloat16* dst = p.y + (size_t)(x.row0 + r) * K + kc;
          if (kc + 32 <= K) {
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              __nv_bfloat162 h0 = __floats2bfloat162_rn(__uint_as_float(v[8 * qq + 0]), __uint_as_float(v[8 * qq + 1]));
              __nv_bfloat162 h1 = __floats2bfloat162_rn(__uint_as_float(v[8 * qq + 2]), __uint_as_float(v[8 * qq + 3]));
              __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(v[8 * qq + 4]), __uint_as_float(v[8 * qq + 5]));
              __nv_bfloat162 h3 = __floats2bfloat162_rn(__uint_as_float(v[8 * qq + 6]), __uint_as_float(v[8 * qq + 7]));
              uint4 o;
              o.x = *reinterpret_cast<uint32_t*>(&h0);
              o.y = *reinterpret_cast<uint32_t*>(&h1);
              o.z = *reinterpret_cast<uint32_t*>(&h2);
              o.w = *reinterpret_cast<uint32_t*>(&h3);
              reinterpret_cast<uint4*>(dst)[qq] = o;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i)  // static indices keep v in registers
              if (kc + i < K) dst[i] = __float2bfloat16_rn(__uint_as_float(v[i]));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&s.acce[ab]);
    }
  }

  // Normal path: the epilogue has read every accumulator, so every MMA and
  // TMEM access has completed.
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
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
  static std::atomic<bool> configured[64];
  const cudaError_t e = set_smem_limit_once(dgrad_tc_kernel<FMT>, (int)dgrad_tc_smem_bytes(), configured);
  if (e != cudaSuccess) return e;
  return launch_pdl(dgrad_tc_kernel<FMT>, dim3(grid), dim3(kThreads), dgrad_tc_smem_bytes(), stream, tm_y, tm_w, p);
}

cudaError_t launch_dgrad_tc(int fmt, const CUtensorMap& tm_y, const CUtensorMap& tm_w, const GroupedArgs& p,
                            int grid, cudaStream_t stream) {
  return fmt == 0 ? launch_dgrad_t<0>(tm_y, tm_w, p, grid, stream) : launch_dgrad_t<1>(tm_y, tm_w, p, grid, stream);
}

}  // namespace gnf4
