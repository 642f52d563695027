// gemm_tc.cu -- grouped 4-bit expert GEMM on tcgen05 tensor cores (sm_100a),
// one MMA per CTA pair.
//
// Y[r, n] = sum_k A[r, k] * W_e[n, k] for the rows r of every expert e, in
// one launch for all experts (grouped-nf4-gemm 0.33.1 on PyPI, opening
// paragraphs: decode in registers, blockwise scaling, fp32 accumulation,
// bf16 epilogue; no bf16 copy of a weight ever reaches global memory).
//
// Design (B200):
//  * The MMA is computed transposed, D^T[n, r] = W_e[n, :] . A[r, :], and
//    spans a cluster of two CTAs (tcgen05 cta_group::2, M = 256): each CTA
//    decodes its own 128 weight rows x 64 k into its own TMEM (the MMA's A
//    operand) and loads its half of the unit's token rows by TMA into
//    128B-swizzled shared memory (the B operand, N/2 rows each); each CTA's
//    TMEM receives its 128 rows of the accumulator.  The even CTA issues the
//    MMAs; its commits are multicast to both CTAs.
//  * Why a pair with 256-row units: (1) the thread that issues the MMAs
//    tests one barrier per 64-k stage, and that test costs it 200-250
//    cycles whenever MMAs are in flight (measured on B200), so a stage must
//    hold 4 x 128 cycles of MMA work: N = 256 tokens.  (2) Per CTA, a
//    256-token tile costs 32 KB of activation traffic per stage; the pair
//    halves it, so shared memory (TMA writes, MMA reads, decode table) stays
//    within its bandwidth and an 8-deep activation ring covers the L2
//    latency (a 4-deep ring of full tiles did not: measured).  (3) Each
//    activation tile serves 256 weight rows, halving its re-reads from L2.
//  * Work unit = (expert e, 256-row weight tile j, chunk of <= 256 of the
//    expert's rows), derived on the device from the group offsets (no host
//    sync, no tile list in global memory); both CTAs of a pair derive the
//    same list.  Experts are taken largest first (a stable rank sort of the
//    row counts), then weight tile, then chunk, so under a skewed routing the
//    long experts start first and small ones fill the tail of the grid.
//  * MMA N = the chunk's rows rounded up to 32 (at least 32), so small groups
//    are not padded to a full tile; each CTA holds N/2 token rows.
//  * Rings per CTA: packed weights (4 stages x 4 KB, two TMA threads taking
//    stages in turn), activation half-tiles (8 stages x 16 KB, 16- or 64-row
//    boxes), decoded weights in TMEM (8 stages x 32 columns).  The
//    accumulator (256 columns) is single: the next unit's MMAs wait until
//    both CTAs' epilogues have drained it.
//  * Synchronisation: per stage, each CTA's decode group meets at a named
//    barrier and one of its threads reports the decoded stage on the even
//    CTA's barrier (remote arrive, cluster scope) once its CTA's activation
//    half-tile has landed, so the MMA thread tests a single barrier per
//    stage.  Both epilogues report the drained accumulator there too.  All
//    waits are bounded.
//  * Epilogue: TMEM -> registers -> bf16 tile in shared memory -> one TMA
//    store per 32 tokens (double-buffered); a ragged last chunk is stored
//    element by element.
//  * Fused combine (CMB, the second projection): once a unit's accumulator
//    is drained and released (the next unit's MMAs already run), its stores
//    are waited for and published, and each of its rows counts its (token,
//    128-column tile) in with an atomic; the thread that completes a token's
//    last valid pair queues it, and the epilogue warps then compute the
//    queued tokens' 128 output columns with the same fp32 fmaf sequence as
//    the separate combine (pairs in slot order), reading the rows through L2,
//    so the fused output equals GEMM + combine bit for bit.  The work
//    overlaps the next unit's mainloop instead of holding the accumulator.
//  * Warp roles per CTA (26 warps): 0 and 24 = weight TMA, 1 = TMEM owner
//    (both CTAs) + MMA issuer (even CTA), 25 = stage poller (even CTA: tests
//    the stage barriers and publishes a ready count the MMA thread reads with
//    a load-acquire), 2 = activation TMA, 3 = scale loader
//    (raw block scales copied into a shared-memory ring with cp.async, 8
//    k-stages per chunk, 3 chunks ahead), 4..19 = decode (four groups of
//    four; group g takes the stages it = g mod 4, so every ring slot is
//    waited on by one group only), 20..23 = epilogue.
//  * Decode: a thread owns one weight row; per 64-k stage it reads its 32
//    packed bytes from shared memory, and for every byte builds the address
//    of a lane-private pair-table entry (PRMT + shift), loads the two bf16
//    codes, multiplies them by the block scale in bf16x2 and finally stores
//    32 columns to TMEM with tcgen05.st.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "internal.h"

namespace gnf4 {
namespace {

constexpr int kBT = 256;   // activation rows (tokens) per unit = max MMA N
constexpr int kHT = kBT / 2;  // token rows held by each CTA
constexpr int kBW = 128;   // weight rows per CTA (M = 256 per pair)
constexpr int kBK = 64;    // k per stage
constexpr int kWStages = 4;
constexpr int kAStages = 8;
constexpr int kTStages = 8;
constexpr int kSChunk = 8;       // k-stages per scale chunk
constexpr int kSStages = 3;      // scale chunks in flight
constexpr int kSRowWords = 9;    // raw scale words per row per chunk (NF4 8, MXFP4 5), padded
constexpr int kDecGroups = 4;
constexpr int kDecWarp0 = 4;
constexpr int kEpiWarp0 = kDecWarp0 + 4 * kDecGroups;  // 20
constexpr int kWProd2 = kEpiWarp0 + 4;                 // 24: second weight producer
constexpr int kPoller = kWProd2 + 1;                   // 25: tests the stage barriers for the MMA thread
constexpr int kThreads = (kPoller + 1) * 32;           // 832
constexpr int kSmallBox = 16;                          // activation rows per box, half-tiles of <= 16 rows
constexpr int kBigBox = 64;                            // activation rows per box otherwise
constexpr int kACol0 = kBT;                            // decoded-weight ring after the accumulator
constexpr int kTmemCols = 512;
constexpr int kActStageBytes = kHT * kBK * 2;          // 16 KB
constexpr int kWStageBytes = kBW * kBK / 2;            // 4 KB
static_assert(kACol0 + kTStages * (kBK / 2) <= kTmemCols, "TMEM budget");
static_assert(kAStages % kDecGroups == 0 && kTStages % kDecGroups == 0 && kWStages % kDecGroups == 0,
              "each ring slot must belong to one decode group");
static_assert(kAStages == kTStages, "one commit per stage releases the activation and decoded-weight slots");
constexpr int kOutRows = 32;                           // tokens per epilogue store
constexpr int kOutBytes = kOutRows * kBW * 2;          // 8 KB: 32 tokens x 128 weight rows, bf16
constexpr int kBarEpi = 1 + kDecGroups;                // named barrier of the epilogue warps (decode groups: 1..4)

struct Smem {
  uint8_t act[kAStages][kActStageBytes];  // 1024-aligned (offset 0); the same offsets in both CTAs
  uint32_t lut[kLutWords];                // 32 KB pair table, entry b of lane l at word 32 b + l
  uint8_t wq[kWStages][kWStageBytes];
  uint32_t sring[kSStages][kBW][kSRowWords];  // raw block scales of kSChunk k-stages per row
  uint8_t out[2][kOutBytes];                  // epilogue staging: [32 tokens][128 columns] bf16 (SwiGLU: 64)
  int off[kMaxExperts + 1];
  int upre[kMaxExperts + 1];
  int scratch[kMaxExperts];
  int order[kMaxExperts];  // experts by descending row count (stable)
  int done[kBT];           // fused combine: tokens this unit's rows completed
  int ndone;
  uint64_t wfull[kWStages], wempty[kWStages];
  uint64_t afull[kAStages];
  uint64_t sdone[kAStages];  // a stage's MMAs completed: frees its activation slot and its decoded-weight slot
  uint64_t tfull[kTStages];  // even CTA only, one arrival per CTA
  uint64_t sfull[kSStages], sempty[kSStages];
  uint64_t accf, acce;  // acce: even CTA only, 8 arrivals (both CTAs' epilogue warps)
  uint64_t mdone;       // abort path only: every issued MMA has retired
  uint32_t tmem_base;
  uint32_t tready;  // even CTA: stages whose report is complete (the poller counts, the MMA thread reads)
  int abort;
};
static_assert(sizeof(Smem) + 1024 <= 227 * 1024, "shared memory budget");

struct Unit {
  int e, j, row0, rows, n;  // n: MMA N (rows rounded up to 32)
};

// Fused combine: pairs of token t whose sorted row lies in [0, nvalid).
__device__ __forceinline__ int cmb_valid_pairs(const CombineArgs& c, int t, int nvalid) {
  int need = 0;
  for (int j = 0; j < c.k; ++j) {
    const int r = __ldg(c.f2s + (size_t)t * c.k + j);
    need += (r >= 0 && r < nvalid) ? 1 : 0;
  }
  return need;
}

// out[t, n0 .. n0+8) = bf16(sum_j w[t, j] * y[f2s[t*k + j], n0 ..]) over the
// valid pairs in slot order, fp32 fmaf from 0 (the separate combine's
// sequence); rows read through L2.  Loads of 8 slots are issued together.
__device__ __forceinline__ void cmb_token_cols8(const CombineArgs& c, const __nv_bfloat16* y, int N, int t, int n0,
                                                int nvalid) {
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  for (int j0 = 0; j0 < c.k; j0 += 8) {
    uint4 yv[8];
    float wv[8];
    bool ok[8];
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const int j = j0 + jj;
      const int r = j < c.k ? __ldg(c.f2s + (size_t)t * c.k + j) : -1;
      ok[jj] = r >= 0 && r < nvalid;
      yv[jj] = ok[jj] ? __ldcg(reinterpret_cast<const uint4*>(y + (size_t)r * N + n0)) : make_uint4(0u, 0u, 0u, 0u);
      wv[jj] = ok[jj] ? __ldg(c.w + (size_t)t * c.k + j) : 0.f;
    }
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      if (!ok[jj]) continue;
      const uint32_t qq[4] = {yv[jj].x, yv[jj].y, yv[jj].z, yv[jj].w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        acc[2 * h] = fmaf(wv[jj], __uint_as_float(qq[h] << 16), acc[2 * h]);
        acc[2 * h + 1] = fmaf(wv[jj], __uint_as_float(qq[h] & 0xFFFF0000u), acc[2 * h + 1]);
      }
    }
  }
  uint32_t o[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * h], acc[2 * h + 1]);
    o[h] = *reinterpret_cast<const uint32_t*>(&b);
  }
  *reinterpret_cast<uint4*>(c.out + (size_t)t * N + n0) = make_uint4(o[0], o[1], o[2], o[3]);
}

// Weight row (within the expert) held by TMEM lane nl of this CTA in pair
// tile j (cta = 0 or 1).  SwiGLU: single tile jj = 2j + cta takes 64 gate
// rows and the matching 64 up rows of a gate_up stack [E, 2I, K]; inside
// every 32-lane quarter q, lanes 0..15 are gate rows 64jj + 16q + x and lanes
// 16..31 the up rows I + 64jj + 16q + x, so the epilogue pairs them with one
// shuffle.
template <bool SWI>
__device__ __forceinline__ int tile_row(int jj, int nl, int I) {
  if (!SWI) return jj * kBW + nl;
  const int q = nl >> 5, x = nl & 31;
  return (x < 16 ? 0 : I) + 64 * jj + 16 * q + (x & 15);
}
// Row of lane nl's packed bytes inside a weight stage (SwiGLU stages hold the
// gate box in rows 0..63 and the up box in rows 64..127).
template <bool SWI>
__device__ __forceinline__ int stage_row(int nl) {
  if (!SWI) return nl;
  const int q = nl >> 5, x = nl & 31;
  return (x < 16 ? 0 : 64) + 16 * q + (x & 15);
}

// Unit u: position p of the largest-first expert order, then pair weight
// tile, then chunk of kBT rows.
__device__ __forceinline__ Unit unit_of(const Smem& s, int E, int u) {
  Unit x;
  const int p = find_group(s.upre, E, u);
  x.e = s.order[p];
  const int local = u - s.upre[p];
  const int rows_e = s.off[x.e + 1] - s.off[x.e];
  const int nch = (rows_e + kBT - 1) / kBT;
  x.j = local / nch;
  const int c = local - x.j * nch;
  x.row0 = s.off[x.e] + c * kBT;
  x.rows = min(kBT, s.off[x.e + 1] - x.row0);
  x.n = max(32, (x.rows + 31) & ~31);
  return x;
}

// Two bf16 codes of byte j of `word` (pair table, 128-byte stride per entry).
// lane8 = 8 * lane: the PRMT puts the byte in bits 8..15, 8 * lane in bits
// 0..7 and zeros above, and the shift turns that into 128 * byte + 4 * lane.
__device__ __forceinline__ uint32_t lut_get(uint32_t lut, uint32_t word, uint32_t lane8, uint32_t j) {
  uint32_t v;
  const uint32_t off = prmt_b32(word, lane8, 0x5504u | (j << 4)) >> 1;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(lut + off));
  return v;
}

template <int FMT, bool SWI, bool CMB>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_a_big,
                   const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_y, GroupedArgs p,
                   CombineArgs cmb) {
  static_assert(!(SWI && CMB), "the combine follows the second projection, not the fused gate_up");
  extern __shared__ uint8_t smem_raw[];
  Smem& s = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t cta = cluster_ctarank();  // 0: issues the MMAs
  const int pair = (int)blockIdx.x >> 1, npairs = (int)gridDim.x >> 1;
  unsigned* err = p.err;
  volatile int* abort = &s.abort;

  griddep_launch_dependents();
  griddep_wait();
  // Both CTAs read the same offsets, so they agree on validity, on U and on
  // every unit; a malformed description makes both return here.
  if (!load_groups(p.offsets, p.counts, p.E, p.M, s.off, s.scratch, err)) return;
  // largest-first expert order: rank = experts with more rows, ties by index
  for (int e = tid; e < p.E; e += kThreads) {
    const int re = s.off[e + 1] - s.off[e];
    int rank = 0;
    for (int f = 0; f < p.E; ++f) {
      const int rf = s.off[f + 1] - s.off[f];
      rank += (rf > re || (rf == re && f < e)) ? 1 : 0;
    }
    s.scratch[rank] = e;
  }
  __syncthreads();
  for (int i = tid; i < p.E; i += kThreads) s.order[i] = s.scratch[i];
  __syncthreads();
  const int I = p.N / 2;  // SwiGLU: output columns
  // pair tiles: 256 weight rows, or (SwiGLU) two single tiles of 64 gate + 64 up rows
  const int nwt = SWI ? ((I / (kBW / 2)) + 1) / 2 : (p.N + 2 * kBW - 1) / (2 * kBW);
  block_exclusive_scan(p.E, s.upre, s.scratch, [&](int q) {
    const int e = s.order[q];
    const int r = s.off[e + 1] - s.off[e];
    return r >= p.min_rows ? ((r + kBT - 1) / kBT) * nwt : 0;
  });
  const int U = s.upre[p.E];
  if (CMB) {
    if (tid == 0) s.ndone = 0;
    if (blockIdx.x == 0) {  // tokens without a valid pair get a zero row (no unit ever completes them)
      const int nvalid = s.off[p.E];
      for (int t = tid; t < cmb.T; t += kThreads)
        if (cmb_valid_pairs(cmb, t, nvalid) == 0)
          for (int n = 0; n < p.N; n += 8)
            *reinterpret_cast<uint4*>(cmb.out + (size_t)t * p.N + n) = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  if (pair >= U) return;  // uniform over the pair
  const int nk = (p.K + kBK - 1) / kBK;

  build_pair_lut<FMT>(s.lut, tid, kThreads);
  if (tid == 0) {
    for (int i = 0; i < kWStages; ++i) {
      mbar_init(&s.wfull[i], 1);
      mbar_init(&s.wempty[i], 4);
    }
    for (int i = 0; i < kAStages; ++i) {
      mbar_init(&s.afull[i], 1);
      mbar_init(&s.sdone[i], 1);
    }
    for (int i = 0; i < kTStages; ++i) mbar_init(&s.tfull[i], 2);
    for (int i = 0; i < kSStages; ++i) {
      mbar_init(&s.sfull[i], 32);
      mbar_init(&s.sempty[i], 4 * kDecGroups);
    }
    mbar_init(&s.accf, 1);
    mbar_init(&s.acce, 8);
    mbar_init(&s.mdone, 1);
    s.tready = 0;
    s.abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_a);
    prefetch_tmap(&tm_a_big);
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_y);
  }
  if (warp == 1) {
    tmem_alloc_pair(&s.tmem_base, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // the other CTA's barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem = s.tmem_base;
  // this CTA's weight tile inside pair tile j
  auto my_tile = [&](int j) { return 2 * j + (int)cta; };

  if (warp == 0 || warp == kWProd2) {
    // ------------------------------------------------------------ weight TMA
    // Two producer threads take the k-stages in turn: an SM completes about
    // one box per issuing thread per memory latency, so one producer alone
    // would cap the weight stream (measured on B200).
    const int pi = warp == 0 ? 0 : 1;
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int u = pair; u < U && ok; u += npairs) {
        const Unit x = unit_of(s, p.E, u);
        const int jj = my_tile(x.j);
        for (int kt = 0; kt < nk; ++kt, ++it) {
          if ((it & 1) != pi) continue;
          const int st = it % kWStages, use = it / kWStages;
          if (it >= kWStages && !(ok = mbar_wait(&s.wempty[st], (use - 1) & 1, err, abort))) break;
          mbar_arrive_expect_tx(&s.wfull[st], kWStageBytes);
          if (SWI) {  // one box of 64 gate rows followed by the matching 64 up rows (zeros past I)
            tma_load_5d(s.wq[st], &tm_w, &s.wfull[st], kt * (kBK / 2), 0, 0, jj, x.e);
          } else {  // rows past N read as zero
            tma_load_3d(s.wq[st], &tm_w, &s.wfull[st], kt * (kBK / 2), jj * kBW, x.e);
          }
        }
      }
      if (!ok)  // drain loads still in flight before shared memory goes away
        for (int i = max(0, it - kWStages); i < it; ++i)
          if ((i & 1) == pi) mbar_drain(&s.wfull[i % kWStages], (i / kWStages) & 1);
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ activation TMA
    // This CTA's half of the unit's rows: [row0 + cta * n/2, + n/2), as one
    // 16-row box (n/2 <= 16) or ceil(n/2 / 64) boxes of 64 rows.  Rows past
    // the group are read but never stored; rows past M read as zero.
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int u = pair; u < U && ok; u += npairs) {
        const Unit x = unit_of(s, p.E, u);
        const int h = x.n / 2;
        const int r0 = x.row0 + (int)cta * h;
        const bool big = h > kSmallBox;
        const int nb = big ? (h + kBigBox - 1) / kBigBox : 1;
        for (int kt = 0; kt < nk; ++kt, ++it) {
          const int st = it % kAStages, use = it / kAStages;
          if (it >= kAStages && !(ok = mbar_wait_cl(&s.sdone[st], (use - 1) & 1, err, abort))) break;
          if (big) {
            mbar_arrive_expect_tx(&s.afull[st], nb * kBigBox * 128);
            for (int b = 0; b < nb; ++b)
              tma_load_2d(s.act[st] + b * kBigBox * 128, &tm_a_big, &s.afull[st], kt * kBK, r0 + b * kBigBox);
          } else {
            mbar_arrive_expect_tx(&s.afull[st], kSmallBox * 128);
            tma_load_2d(s.act[st], &tm_a, &s.afull[st], kt * kBK, r0);
          }
        }
      }
      if (!ok)
        for (int i = max(0, it - kAStages); i < it; ++i) mbar_drain(&s.afull[i % kAStages], (i / kAStages) & 1);
    }
  } else if (warp == 3) {
    // ------------------------------------------------------------ scale loader
    // Copies the raw block scales of the next kSChunk k-stages of every
    // weight row into a shared-memory ring with 4-byte cp.async, three
    // chunks ahead, so decode never waits on a global load.  NF4: the 8
    // absmax floats of the chunk; MXFP4: the 5 aligned words that cover the
    // chunk's 16 scale bytes.  Lane l serves rows l, l+32, l+64, l+96.
    const int nsc = FMT == 0 ? p.K / 64 : p.K / 32;
    int ci = 0;
    bool ok = true;
    for (int u = pair; u < U && ok; u += npairs) {
      const Unit x = unit_of(s, p.E, u);
      const int jj = my_tile(x.j);
      for (int kt0 = 0; kt0 < nk; kt0 += kSChunk, ++ci) {
        const int slot = ci % kSStages;
        if (ci >= kSStages && !(ok = mbar_wait(&s.sempty[slot], ((ci / kSStages) - 1) & 1, err, abort))) break;
#pragma unroll
        for (int m = 0; m < kBW / 32; ++m) {
          const int r = lane + 32 * m;
          const int n = tile_row<SWI>(jj, r, I);
          if (n >= p.N) continue;  // never stored
          const size_t rowsc = ((size_t)x.e * p.N + (size_t)n) * (size_t)nsc;
          if (FMT == 0) {
            const float* src = reinterpret_cast<const float*>(p.scales) + rowsc + kt0;
            const int cnt = min(kSChunk, nk - kt0);
            for (int q = 0; q < cnt; ++q) cp_async_4(&s.sring[slot][r][q], src + q);
          } else {
            const uint8_t* base = reinterpret_cast<const uint8_t*>(p.scales);
            const size_t b0 = rowsc + 2 * (size_t)kt0;                     // first scale byte of the chunk
            const size_t b1 = min(rowsc + (size_t)nsc, b0 + 2 * kSChunk);  // one past the last
            const size_t w0 = b0 & ~(size_t)3;
            for (size_t wq = w0, q = 0; wq < b1; wq += 4, ++q) cp_async_4(&s.sring[slot][r][q], base + wq);
          }
        }
        cp_async_arrive_noinc(&s.sfull[slot]);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (even CTA)
    if (lane == 0 && cta == 0) {
      int it = 0, uc = 0;
      uint32_t ready = 0;  // stages the poller had counted complete at the last read
      bool ok = true;
      for (int u = pair; u < U && ok; u += npairs, ++uc) {
        const Unit x = unit_of(s, p.E, u);
        if (uc >= 1 && !(ok = mbar_wait_cl(&s.acce, (uc - 1) & 1, err, abort))) break;
        tc_fence_after();
        const uint32_t idesc = idesc_bf16_m256((uint32_t)x.n);
        for (int kt = 0; kt < nk; ++kt, ++it) {
          const int sa = it % kAStages, sT = it % kTStages;
          // Both CTAs report a stage only after its activation half-tiles have
          // landed.  The poller warp tests those barriers and counts the
          // complete stages; this thread re-reads the count only when it has
          // used up the last one it read.  Any shared-memory access here waits
          // ~220 cycles behind the decode warps' table lookups (measured), long
          // enough to let the tensor pipe run dry if paid every stage; the
          // poller runs several stages ahead, so one read covers several.
          // One fence after each fresh read orders the MMAs of every stage
          // that read covers after the decode warps' TMEM stores (measured in
          // isolation: a fence and an acquire per stage add ~110 cycles to the
          // ~200 of four small-N pair MMAs).
          if ((int)ready <= it) {
            ready = ld_acquire_shared(&s.tready);
            if ((int)ready <= it) {
              const long long t0 = clock64();
              while ((int)(ready = ld_acquire_shared(&s.tready)) <= it) {
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
          const uint32_t a_col = tmem + (uint32_t)(kACol0 + sT * (kBK / 2));
          const uint32_t b_addr = smem_u32(s.act[sa]);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            tc_mma_ts_pair(tmem, a_col + kk * 8, sdesc_k_sw128(b_addr + kk * 32), idesc, (kt | kk) != 0);
          tc_commit_pair(&s.sdone[sa]);  // sa == sT: one commit frees both slots
        }
        if (!ok) break;
        tc_commit_pair(&s.accf);
      }
      if (!ok) {
        // abort: let every MMA already issued retire before TMEM is released
        tc_commit_pair(&s.mdone);
        mbar_drain(&s.mdone, 0);
      }
    }
  } else if (warp == kPoller) {
    // ------------------------------------------------------------ stage poller (even CTA)
    if (lane == 0 && cta == 0) {
      int it = 0;
      bool ok = true;
      for (int u = pair; u < U && ok; u += npairs)
        for (int kt = 0; kt < nk; ++kt, ++it) {
          if (!(ok = mbar_wait_cl(&s.tfull[it % kTStages], (it / kTStages) & 1, err, abort))) break;
          st_release_shared(&s.tready, (uint32_t)(it + 1));
        }
    }
  } else if (warp >= kDecWarp0 && warp < kEpiWarp0) {
    // ------------------------------------------------------------ decode
    // A failed wait (timeout, or another role's abort) marks the warp dead:
    // it keeps walking the stage list and meets its group's named barrier
    // every owned stage, doing nothing else, so no warp of the group is left
    // waiting at that barrier for one that has stopped.
    const int grp = (warp - kDecWarp0) >> 2, q = warp & 3;
    const int nl = q * 32 + lane;
    const uint32_t lut = smem_u32(s.lut);
    const uint32_t lane8 = (uint32_t)lane * 8u;
    const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16);
    int it = 0, ci = 0;
    bool live = true;
    for (int u = pair; u < U; u += npairs) {
      const Unit xu = unit_of(s, p.E, u);
      const int jj = my_tile(xu.j);
      for (int kt = 0; kt < nk; ++kt, ++it) {
        const int q8 = kt % kSChunk, slot = ci % kSStages;
        if (live && q8 == 0) live = mbar_wait(&s.sfull[slot], (ci / kSStages) & 1, err, abort);
        if (it % kDecGroups == grp) {
          const int sw = it % kWStages, sT = it % kTStages, sa = it % kAStages;
          if (live) live = mbar_wait(&s.wfull[sw], (it / kWStages) & 1, err, abort);
          if (live && it >= kTStages) live = mbar_wait_cl(&s.sdone[sT], ((it / kTStages) - 1) & 1, err, abort);
          live = __all_sync(0xffffffffu, live);
          if (live) {
            uint32_t sc0, sc1;
            if (FMT == 0) {
              sc0 = sc1 = f32_to_bf16x2_rn(__uint_as_float(s.sring[slot][nl][q8]));
            } else {
              // bytes of the chunk start at (row offset & 3) inside the copied words
              const size_t rowsc = ((size_t)xu.e * p.N + (size_t)tile_row<SWI>(jj, nl, I)) * (size_t)(p.K / 32);
              const uint32_t b = (uint32_t)(rowsc & 3u) + 2u * (uint32_t)q8;
              const uint8_t* bytes = reinterpret_cast<const uint8_t*>(s.sring[slot][nl]);
              sc0 = e8m0_to_bf16x2(bytes[b]);
              sc1 = (2 * kt + 1 < p.K / 32) ? e8m0_to_bf16x2(bytes[b + 1]) : 0u;
            }
            // two 16-byte reads of this row's 32 bytes, ordered so a quarter warp
            // touches 8 distinct 16-byte bank groups
            const uint32_t srow = (uint32_t)stage_row<SWI>(nl);
            const uint32_t wrow = smem_u32(s.wq[sw]) + srow * 32u;
            const uint32_t c_first = (srow >> 2) & 1u;
            uint4 c0 = lds_u128(wrow + 16u * c_first), c1 = lds_u128(wrow + 16u * (c_first ^ 1u));
            if (c_first) {
              const uint4 tmp = c0;
              c0 = c1;
              c1 = tmp;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.wempty[sw]);  // packed bytes are in registers now
            uint32_t v[32];
            {
              const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                const uint32_t sc = i < 4 ? sc0 : sc1;
#pragma unroll
                for (int j = 0; j < 4; ++j) v[4 * i + j] = bf16x2_mul(lut_get(lut, w[i], lane8, (uint32_t)j), sc);
              }
            }
            tmem_st_32x32b_x32(t_lane + (uint32_t)(kACol0 + sT * (kBK / 2)), v);
            tmem_wait_st();
            tc_fence_before();
          }
          // One report per CTA and stage: the group's four warps meet at their
          // named barrier (their TMEM stores have completed), then one thread
          // waits for this CTA's activation half-tile and reports on the even
          // CTA's barrier.  The report publishes no generic-memory write, so
          // the arrive is relaxed: a release would hold the thread ~1.5k
          // cycles under this kernel's load (measured).
          named_bar(1 + grp, 128);
          if (q == 0) {
            if (lane == 0 && live) {
              live = mbar_wait(&s.afull[sa], (it / kAStages) & 1, err, abort);
              if (live) mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(&s.tfull[sT]), 0));
            }
            live = __shfl_sync(0xffffffffu, live, 0);
          }
        }
        if (q8 == kSChunk - 1 || kt == nk - 1) {  // this warp is done with the chunk
          __syncwarp();
          if (lane == 0 && live) mbar_arrive(&s.sempty[slot]);
          ++ci;
        }
      }
    }
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + 4) {
    // ------------------------------------------------------------ epilogue
    // Full 32-token chunks are converted into a shared-memory tile and
    // written by one TMA store (double-buffered); a ragged last chunk is
    // stored element by element.  Per-element stores of whole chunks cost
    // ~2.3k cycles each (measured), the TMA path a few hundred.
    const int q = warp & 3;
    const bool issuer = q == 0 && lane == 0;
    const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16);
    constexpr int kCols = SWI ? kBW / 2 : kBW;  // output columns of this CTA's tile
    int uc = 0, nbuf = 0;
    for (int u = pair; u < U; u += npairs, ++uc) {
      const Unit x = unit_of(s, p.E, u);
      const int jj = my_tile(x.j);
      // the four warps agree on the outcome, so none is left at a named barrier
      if (!named_bar_and(kBarEpi, 128, mbar_wait_cl(&s.accf, uc & 1, err, abort))) break;
      tc_fence_after();
      const int n = jj * kBW + q * 32 + lane;
      const int col0 = jj * kCols;                          // first output column of the tile
      const bool any_col = col0 < (SWI ? I : p.N);
      __nv_bfloat16* ycol = p.y + (size_t)x.row0 * p.N + n;
      for (int c = 0; c * 32 < x.rows; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_lane + (uint32_t)(c * 32), v);
        tmem_wait_ld();
        const int lim = min(32, x.rows - c * 32);
        const bool staged = lim == kOutRows;  // uniform over the four warps
        uint8_t* st = s.out[nbuf & 1];
        if (staged) {
          if (issuer) bulk_wait_read<1>();  // this buffer's store of two chunks ago has read it
          named_bar(kBarEpi, 128);
        }
        if (SWI) {
          // lane x < 16 holds gate(col), lane x + 16 up(col).  Per pair of rows
          // (2m, 2m+1) the low lane finishes row 2m and the high lane row 2m+1:
          // each sends its partner the value the partner lacks.
          const bool up_lane = lane >= 16;
          const int cl = q * 16 + (lane & 15);
          const int col = col0 + cl;
          __nv_bfloat16* hcol = p.y + (size_t)x.row0 * I + col;
#pragma unroll
          for (int m = 0; m < 16; ++m) {
            // select between two static indices so v stays in registers
            const float even = __uint_as_float(v[2 * m]), odd = __uint_as_float(v[2 * m + 1]);
            const float keep = up_lane ? odd : even;
            const float send = up_lane ? even : odd;
            const float got = __shfl_xor_sync(0xffffffffu, send, 16);
            const int i = 2 * m + (up_lane ? 1 : 0);
            // low lane: gate = keep (row 2m), up = got; high lane: up = keep (row 2m+1), gate = got
            const float g = up_lane ? got : keep, uu = up_lane ? keep : got;
            const __nv_bfloat16 hv = __float2bfloat16_rn(silu_mul_tanh(g, uu));
            if (staged)
              reinterpret_cast<__nv_bfloat16*>(st)[i * kCols + cl] = hv;
            else if (i < lim && col < I)
              hcol[(size_t)(c * 32 + i) * I] = hv;
          }
        } else if (staged) {
          const int cl = q * 32 + lane;
#pragma unroll
          for (int i = 0; i < 32; ++i)
            reinterpret_cast<__nv_bfloat16*>(st)[i * kCols + cl] = __float2bfloat16_rn(__uint_as_float(v[i]));
        } else if (n < p.N) {
#pragma unroll
          for (int i = 0; i < 32; ++i)
            if (i < lim) ycol[(size_t)(c * 32 + i) * p.N] = __float2bfloat16_rn(__uint_as_float(v[i]));
        }
        if (staged) {
          fence_proxy_async_smem();
          named_bar(kBarEpi, 128);
          if (issuer) {
            // columns past the output's end are not written by the store
            if (any_col) tma_store_2d(&tm_y, st, col0, x.row0 + c * 32);
            bulk_commit();
          }
          ++nbuf;
        }
      }
      tc_fence_before();
      __syncwarp();
      // the accumulator's TMEM loads have completed (tcgen05.wait::ld): relaxed
      if (lane == 0) mbar_arrive_cluster_relaxed(mapa_shared(smem_u32(&s.acce), 0));
      if (CMB) {
        // The unit's rows of y are published before they are counted: the
        // TMA stores have completed (not only read their source), the proxy
        // fence orders them before the issuer's generic accesses, the
        // barrier before every epilogue thread's, and each counting thread's
        // fence (cumulative) before its count.
        if (issuer) {
          bulk_wait_all();
          fence_proxy_async_all();
        }
        named_bar(kBarEpi, 128);
        const int et = q * 32 + lane;
        const int nvalid = s.off[p.E];
        const int ntile = (p.N + kBW - 1) / kBW;
        for (int rr = et; rr < x.rows; rr += 128) {
          const int f = __ldg(cmb.s2f + x.row0 + rr);
          if (f < 0 || f >= cmb.T * cmb.k) continue;
          const int t = f / cmb.k;
          int* ctr = cmb.cnt + (size_t)t * ntile + jj;
          __threadfence();
          if (atomicAdd(ctr, 1) == cmb_valid_pairs(cmb, t, nvalid) - 1) {
            __threadfence();  // the other units' rows of t are visible to this thread from here on
            *ctr = 0;         // every pair of this tile is in: ready for the next call
            s.done[atomicAdd(&s.ndone, 1)] = t;
          }
        }
        named_bar(kBarEpi, 128);
        const int nd = s.ndone;
        if (nd > 0) __threadfence();  // the completing threads' acquisitions, for every reader
        // 16 threads per token (8 columns each), 8 tokens at a time
        for (int o = et; o < nd * 16; o += 128) {
          const int n0 = col0 + (o & 15) * 8;
          if (n0 < p.N) cmb_token_cols8(cmb, p.y, p.N, s.done[o >> 4], n0, nvalid);
        }
        named_bar(kBarEpi, 128);
        if (et == 0) s.ndone = 0;
      }
    }
    if (issuer) bulk_wait_all();  // every store has completed before the CTA ends
  }

  // Normal path: both epilogues have consumed the accumulator, so every MMA
  // and TMEM access of the pair has completed.  The cluster barrier also
  // keeps each CTA's shared memory alive until the other's remote arrivals
  // have landed.
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace

size_t gemm_tc_smem_bytes() { return sizeof(Smem) + 1024; }

// Cluster of two CTAs (the MMA pair) with programmatic stream serialization.
template <typename... KArgs, typename... Args>
static cudaError_t launch_pair(void (*kernel)(KArgs...), int grid, size_t smem, cudaStream_t stream,
                               Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int FMT, bool SWI, bool CMB>
cudaError_t launch_gemm_tc_t(const CUtensorMap& tm_a, const CUtensorMap& tm_a_big, const CUtensorMap& tm_w,
                             const CUtensorMap& tm_y, const GroupedArgs& p, const CombineArgs& c, int grid,
                             cudaStream_t stream) {
  static std::atomic<bool> configured[64];
  const cudaError_t e = set_smem_limit_once(gemm_tc_kernel<FMT, SWI, CMB>, (int)gemm_tc_smem_bytes(), configured);
  if (e != cudaSuccess) return e;
  return launch_pair(gemm_tc_kernel<FMT, SWI, CMB>, grid, gemm_tc_smem_bytes(), stream, tm_a, tm_a_big, tm_w, tm_y,
                     p, c);
}

cudaError_t launch_gemm_tc(int fmt, bool swiglu, const CUtensorMap& tm_a, const CUtensorMap& tm_a_big,
                           const CUtensorMap& tm_w, const CUtensorMap& tm_y, const GroupedArgs& p, int grid,
                           cudaStream_t stream, const CombineArgs* combine) {
  const CombineArgs none{};
  if (combine != nullptr) {
    if (swiglu) return cudaErrorInvalidValue;
    return fmt == 0 ? launch_gemm_tc_t<0, false, true>(tm_a, tm_a_big, tm_w, tm_y, p, *combine, grid, stream)
                    : launch_gemm_tc_t<1, false, true>(tm_a, tm_a_big, tm_w, tm_y, p, *combine, grid, stream);
  }
  if (fmt == 0)
    return swiglu ? launch_gemm_tc_t<0, true, false>(tm_a, tm_a_big, tm_w, tm_y, p, none, grid, stream)
                  : launch_gemm_tc_t<0, false, false>(tm_a, tm_a_big, tm_w, tm_y, p, none, grid, stream);
  return swiglu ? launch_gemm_tc_t<1, true, false>(tm_a, tm_a_big, tm_w, tm_y, p, none, grid, stream)
                : launch_gemm_tc_t<1, false, false>(tm_a, tm_a_big, tm_w, tm_y, p, none, grid, stream);
}

int gemm_tc_rows_per_unit() { return kBT; }
int gemm_tc_weight_rows_per_unit() { return 2 * kBW; }
int gemm_tc_weight_box_rows() { return kBW; }
int gemm_tc_out_box_rows() { return kOutRows; }

// CTAs for a launch over `units` pair units: whole pairs, at most as many as
// can be resident at once (queried once per device).
int gemm_tc_grid(long long units, int num_sms) {
  static std::atomic<int> max_clusters[64];
  int dev = 0;
  int mc = 0;
  if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) mc = max_clusters[dev].load();
  if (mc == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(num_sms & ~1));
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = gemm_tc_smem_bytes();
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    static std::atomic<bool> configured[64];
    int n = 0;
    if (set_smem_limit_once(gemm_tc_kernel<0, false, false>, (int)gemm_tc_smem_bytes(), configured) == cudaSuccess &&
        cudaOccupancyMaxActiveClusters(&n, gemm_tc_kernel<0, false, false>, &cfg) == cudaSuccess && n > 0)
      mc = n;
    else
      mc = num_sms / 2;
    cudaGetLastError();
    if (dev >= 0 && dev < 64) max_clusters[dev].store(mc);
  }
  const long long pairs = units < mc ? units : mc;
  return (int)(2 * (pairs > 0 ? pairs : 1));
}
int gemm_tc_small_box_rows() { return kSmallBox; }
int gemm_tc_big_box_rows() { return kBigBox; }

}  // namespace gnf4
