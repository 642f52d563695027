// common.cuh -- device helpers shared by the libgnf4 kernels (sm_100a).
//
// Hand-written PTX wrappers for mbarriers, TMA (cp.async.bulk.tensor),
// tcgen05 (TMEM alloc, MMA, loads and stores) and the warp-level MMA, plus the
// decode tables.  Every wait on an mbarrier is bounded: after about two
// seconds of spinning it sets GNF4_DEVERR_TIMEOUT in the device error word and
// returns false so the kernel can drain and exit instead of hanging the GPU.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gnf4.h"

namespace gnf4 {

// ---------------------------------------------------------------- limits
constexpr int kMaxExperts = 1024;               // group table held in shared memory
constexpr long long kSpinLimitCycles = 1ll << 32;  // ~2.2 s at 1.965 GHz

// ---------------------------------------------------------------- decode tables
// NF4 codebook (NormalFloat-4 of the QLoRA paper): index 7 is the exact zero.
__device__ __constant__ float kNf4Code[16] = {
    -1.0f, -0.6961928009986877f, -0.5250730514526367f, -0.39491748809814453f,
    -0.28444138169288635f, -0.18477343022823334f, -0.09105003625154495f, 0.0f,
    0.07958029955625534f, 0.16093020141124725f, 0.24611230194568634f, 0.33791524171829224f,
    0.44070982933044434f, 0.5626170039176941f, 0.7229568362236023f, 1.0f};
// OCP e2m1: bit 3 sign, bits 2..0 index the magnitude.
__device__ __constant__ float kE2m1Mag[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

__device__ __forceinline__ float e2m1_value(uint32_t code) {
  float m = kE2m1Mag[code & 7u];
  return (code & 8u) ? -m : m;
}

// 2^(e-127) as fp32, exact; e = 0 is the subnormal 2^-127; e = 255 is NaN.
__device__ __forceinline__ float e8m0_to_f32(uint32_t e) {
  if (e == 0u) return __uint_as_float(0x00400000u);
  if (e == 255u) return __uint_as_float(0x7fc00000u);
  return __uint_as_float(e << 23);
}

// 2^(e-127) as a bf16 pattern duplicated in both halves (bf16 shares fp32's
// exponent field, so the power of two is exact; e = 0 is the bf16 subnormal).
__device__ __forceinline__ uint32_t e8m0_to_bf16x2(uint32_t e) {
  uint32_t h = (e == 0u) ? 0x0040u : (e == 255u ? 0x7fc0u : (e << 7));
  return h | (h << 16);
}

// Pair lookup table in shared memory: entry b (a packed byte) holds the two
// decoded codes of that byte as bf16x2, element 2i in the low half.  The
// table is replicated 32 times, word index b*32 + lane, so a warp's 32 lookups
// always hit 32 different banks.  NF4 stores element 2i in the high nibble,
// MXFP4 in the low nibble.  Values are the unscaled codes (exact in bf16 for
// e2m1, rounded to nearest bf16 for NF4).
constexpr int kLutWords = 256 * 32;
constexpr int kLutBytes = kLutWords * 4;

template <int FMT>  // 0 = NF4, 1 = MXFP4
__device__ __forceinline__ void build_pair_lut(uint32_t* lut, int tid, int nthreads) {
  for (int i = tid; i < kLutWords; i += nthreads) {
    uint32_t b = (uint32_t)i >> 5;
    float lo, hi;
    if (FMT == 0) {
      lo = kNf4Code[b >> 4];
      hi = kNf4Code[b & 15u];
    } else {
      lo = e2m1_value(b & 15u);
      hi = e2m1_value(b >> 4);
    }
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    lut[i] = *reinterpret_cast<uint32_t*>(&v);
  }
}

// Same pair table with a 256-byte entry stride (entry b, lane l at byte
// b*256 + 4*l; the upper 128 bytes of every entry are unused).  The address
// of a lookup is then one PRMT: byte 0 = 4*lane, byte 1 = the packed byte,
// bytes 2..3 = 0 -- one integer instruction and one shared load per byte.
constexpr int kLut256Words = 256 * 64;
constexpr int kLut256Bytes = kLut256Words * 4;

template <int FMT>
__device__ __forceinline__ void build_pair_lut256(uint32_t* lut, int tid, int nthreads) {
  for (int i = tid; i < 256 * 32; i += nthreads) {
    const uint32_t b = (uint32_t)i >> 5, l = (uint32_t)i & 31u;
    float lo, hi;
    if (FMT == 0) {
      lo = kNf4Code[b >> 4];
      hi = kNf4Code[b & 15u];
    } else {
      lo = e2m1_value(b & 15u);
      hi = e2m1_value(b >> 4);
    }
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    lut[b * 64u + l] = *reinterpret_cast<uint32_t*>(&v);
  }
}

// fp32 -> bf16 round-to-nearest-even on the integer pipe, duplicated in both
// halves (the hardware conversion runs on the narrow XU pipe, which a decode
// loop would saturate).  Exact RNE for every finite input and +-Inf; a NaN
// stays a NaN.
__device__ __forceinline__ uint32_t f32_to_bf16x2_rn(float f) {
  const uint32_t u = __float_as_uint(f);
  uint32_t h = (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
  if ((u & 0x7FFFFFFFu) > 0x7F800000u) h = (u >> 16) | 0x0040u;  // NaN: keep it quiet
  return h | (h << 16);
}

__device__ __forceinline__ uint32_t prmt_b32(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&a);
  __nv_bfloat162 y = *reinterpret_cast<__nv_bfloat162*>(&b);
  __nv_bfloat162 z = __hmul2(x, y);
  return *reinterpret_cast<uint32_t*>(&z);
}

// silu(g) * u = g / (1 + e^-g) * u in fp32 with the fast exponential and
// division intrinsics (a few ulp; a denominator above 2^126 gives 0, the
// limit of silu for g -> -inf).
__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// The same product through silu(g) = (g/2) (1 + tanh(g/2)): one special-
// function instruction (tanh.approx, absolute error about 2^-11) and no
// division.  For an epilogue that shares the issue path with heavy shared-
// memory traffic, where each special-function op waits behind it (measured:
// the exponential + division form cost the fused gate_up GEMM 33 us of 283
// on the Qwen3-shaped prefill).  Relative error about 2^-11 for g >= 0; for
// g < 0 the absolute error is at most |g u| 2^-12.
__device__ __forceinline__ float silu_mul_tanh(float g, float u) {
  const float hg = 0.5f * g;
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(hg));
  return fmaf(hg, t, hg) * u;
}

// ---------------------------------------------------------------- stream order
// Programmatic dependent launch: let the next kernel of the stream be
// scheduled now, and wait until every earlier kernel of the stream has
// completed and its memory is visible.  Without the launch attribute both
// are no-ops.
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------- misc
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 lds_u128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

__device__ __forceinline__ uint2 ldg_nc_u64(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ldg_nc_u128(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ldg_u128(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Decodes the 16 packed bytes of `w` (byte i = elements 2i, 2i+1 of 32
// codes) into 16 bf16x2 pairs multiplied by the bf16x2 scale `sc`.
// `lane4` = 4 * lane; the table is the 256-byte-stride pair table.
// Table lookup with 32-bit shared-memory addressing: the PRMT result is the
// byte offset inside the table and `lut` its shared-window address, so the
// lookup is one PRMT and one shared load.  (Not volatile: the table is
// read-only once built, so the compiler may schedule the loads freely.)
__device__ __forceinline__ uint32_t lut256_get(uint32_t lut, uint32_t word, uint32_t lane4, uint32_t j) {
  uint32_t v;
  asm("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(lut + prmt_b32(word, lane4, 0x5504u | (j << 4))));
  return v;
}

__device__ __forceinline__ void decode16_lut256(uint32_t lut, uint32_t lane4, uint4 w, uint32_t sc,
                                                uint32_t (&out)[16]) {
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
#pragma unroll
    for (int j = 0; j < 4; ++j) out[4 * i + j] = bf16x2_mul(lut256_get(lut, words[i], lane4, (uint32_t)j), sc);
  }
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0u;
}

// Waits for the phase with the given parity to complete.  Gives up after
// `limit` cycles (raising GNF4_DEVERR_TIMEOUT and *abort), or as soon as
// another role of the CTA has raised *abort.
__device__ __forceinline__ bool mbar_wait_for(uint64_t* bar, uint32_t parity, unsigned* err, volatile int* abort,
                                              long long limit) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > limit) {
      atomicOr(err, GNF4_DEVERR_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned* err,
                                          volatile int* abort) {
  return mbar_wait_for(bar, parity, err, abort, kSpinLimitCycles);
}

// Short bounded wait used while draining after an abort (no error raised).
__device__ __forceinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > (1ll << 28)) return;
  }
}

// ---------------------------------------------------------------- TMA
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void tma_load_5d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2,
                                            int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6, %7}], "
      "[%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}

// TMA store of a 2-D box from shared memory (bulk-group completion).  The
// caller fences its generic-proxy writes to `src` first.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Wait until at most N committed bulk groups still read their shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
// Wait until every committed bulk group has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Named barrier over `n` threads (ids 1..15; 0 is __syncthreads).
__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Named barrier that also returns the AND of `v` over its `n` threads.
__device__ __forceinline__ bool named_bar_and(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"((uint32_t)v), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// 4-byte asynchronous global -> shared copy (both addresses 4-byte aligned).
__device__ __forceinline__ void cp_async_4(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}

// Arrives on `bar` once every cp.async this thread issued so far has landed
// (the barrier's expected count must include this arrival).
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (TMA) accesses to the same memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// Orders this thread's async-proxy accesses (completed bulk stores) with its
// later generic-proxy accesses, in every state space.
__device__ __forceinline__ void fence_proxy_async_all() { asm volatile("fence.proxy.async;" ::: "memory"); }

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* holder, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(holder)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive once on `bar` when every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// D[tmem] (+)= A[tmem] x B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Acquire / release accesses of a shared-memory counter (CTA scope).
__device__ __forceinline__ uint32_t ld_acquire_shared(const void* p) {
  uint32_t v;
  asm volatile("ld.acquire.cta.shared::cta.u32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_shared(void* p, uint32_t v) {
  asm volatile("st.release.cta.shared::cta.u32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

// ---------------------------------------------------------------- CTA pairs
// Two CTAs of a cluster share one MMA (cta_group::2): the even CTA issues it,
// both hold half of each operand and their own half of the accumulator.
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank) {
  uint32_t d;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(d) : "r"(saddr), "r"(rank));
  return d;
}
// Arrive (release, cluster scope) on an mbarrier given by its cluster address.
// The release makes the arriving thread wait until its earlier memory
// operations are visible cluster-wide: ~320 cycles on an idle SM, ~1.5k
// under a GEMM's load (measured on B200).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cl_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cl_addr) : "memory");
}
// Relaxed arrive on an mbarrier given by its cluster address (~2 cycles).
// For signals that publish no generic-memory writes: the TMEM stores or loads
// they report have completed (tcgen05.wait::st / ::ld) and the shared-memory
// tiles were written by TMA and observed complete before the arrive issues.
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t cl_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cl_addr) : "memory");
}
// try_wait with cluster-scope acquire (arrivals come from the other CTA too).
__device__ __forceinline__ bool mbar_try_wait_cl(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0u;
}
__device__ __forceinline__ bool mbar_wait_cl(uint64_t* bar, uint32_t parity, unsigned* err, volatile int* abort) {
  if (mbar_try_wait_cl(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait_cl(bar, parity)) return true;
    if (*abort) return false;
    if (clock64() - t0 > kSpinLimitCycles) {
      atomicOr(err, GNF4_DEVERR_TIMEOUT);
      *abort = 1;
      return false;
    }
  }
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t* holder, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(holder)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
// Arrive once on `bar` in both CTAs of the pair when every tcgen05 operation
// this thread issued so far has completed.
__device__ __forceinline__ void tc_commit_pair(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"((uint16_t)3)
      : "memory");
}
// D[tmem] (+)= A[tmem] x B[smem]^T over the CTA pair: M = 256 (128 rows of A
// and of D in each CTA's TMEM), B's N columns split in halves between the
// CTAs' shared memory at the same offset.
__device__ __forceinline__ void tc_mma_ts_pair(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Instruction descriptor: kind::f16, bf16 x bf16 -> fp32, both K-major, M = 256 (a CTA pair), N = n.
__device__ __forceinline__ uint32_t idesc_bf16_m256(uint32_t n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((256u >> 4) << 24);
}

// Shared-memory matrix descriptor for a K-major operand stored with the 128B
// swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sdesc_k_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);  // start address
  d |= (uint64_t)1u << 16;                   // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32;         // stride byte offset: next 8-row group
  d |= (uint64_t)1u << 46;                   // descriptor version for tcgen05
  d |= (uint64_t)2u << 61;                   // 128-byte swizzle
  return d;
}

// Instruction descriptor: kind::f16, A = B = bf16, D = fp32, both K-major,
// M = 128, N = n (multiple of 16, 16..256).
__device__ __forceinline__ uint32_t idesc_bf16_m128(uint32_t n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((n >> 3) << 17) | ((128u >> 4) << 24);
}

#define GNF4_R32(v)                                                                                             \
  "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]), "r"(v[9]), \
      "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]),         \
      "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]),         \
      "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
#define GNF4_W32(v)                                                                                           \
  "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), \
      "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), \
      "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), \
      "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])

// Each thread of the warp writes 32 consecutive 32-bit columns of its own
// lane (the warp covers the 32 lanes of its quarter of TMEM).
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(taddr),
      GNF4_R32(v)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : GNF4_W32(v)
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// ---------------------------------------------------------------- warp MMA
// D (16x8 fp32) += A (16x16 bf16, row) x B (16x8 bf16, col).
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------- groups
// Warp 0 does the group bookkeeping (E <= kMaxExperts): lane l owns the
// contiguous run of groups [l*per, l*per + per), per = ceil(E/32), so an
// exclusive scan is one pass over the run, five shuffles and a second pass.
// A block-wide Hillis-Steele scan took ~5k cycles for 64 groups (14 block
// barriers); this takes about one global-load latency.

// Exclusive scan of the lanes' partial sums (warp 0).
__device__ __forceinline__ int warp_exclusive_sum(int v, int lane, int* total) {
  int incl = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += o;
  }
  *total = __shfl_sync(0xffffffffu, incl, 31);
  return incl - v;
}

// Loads the group description into shared memory as row offsets off[0..E]
// (from `offsets`, or as the exclusive scan of `counts`) and checks it.
// Returns false (and flags GNF4_DEVERR_BAD_OFFSETS) if it is malformed.  All
// threads of the block must call it; it ends with __syncthreads().
__device__ __forceinline__ bool load_groups(const int* offsets, const int* counts, int E, int M, int* off,
                                            int* scratch, unsigned* err) {
  (void)scratch;
  __shared__ int s_bad;
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int per = (E + 31) >> 5;
    const int b = min(lane * per, E), e_end = min(b + per, E);
    bool bad = false;
    if (offsets != nullptr) {
      for (int i = lane; i <= E; i += 32) off[i] = offsets[i];
      __syncwarp();
      for (int i = b; i < e_end; ++i) bad |= off[i + 1] < off[i];
    } else {
      int sum = 0;
      for (int i = b; i < e_end; ++i) {
        const int c = __ldg(counts + i);
        bad |= c < 0;
        sum += c;
      }
      int total = 0;
      int run = warp_exclusive_sum(sum, lane, &total);
      for (int i = b; i < e_end; ++i) {
        off[i] = run;
        run += __ldg(counts + i);
      }
      if (lane == 0) off[E] = total;
      __syncwarp();
    }
    if (lane == 0) bad |= off[0] != 0 || off[E] > M;
    bad = __any_sync(0xffffffffu, bad);
    if (lane == 0) s_bad = bad ? 1 : 0;
  }
  __syncthreads();
  const bool bad = s_bad != 0;
  if (bad && threadIdx.x == 0 && blockIdx.x == 0) atomicOr(err, GNF4_DEVERR_BAD_OFFSETS);
  return !bad;
}

// Exclusive scan over e of val(e), written to pre[0..E]; all threads call
// (warp 0 computes; val is evaluated twice per e and must be pure).
template <class F>
__device__ __forceinline__ void block_exclusive_scan(int E, int* pre, int* scratch, F val) {
  (void)scratch;
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int per = (E + 31) >> 5;
    const int b = min(lane * per, E), e_end = min(b + per, E);
    int sum = 0;
    for (int i = b; i < e_end; ++i) sum += val(i);
    int total = 0;
    int run = warp_exclusive_sum(sum, lane, &total);
    for (int i = b; i < e_end; ++i) {
      pre[i] = run;
      run += val(i);
    }
    if (lane == 0) pre[E] = total;
  }
  __syncthreads();
}

// Largest e in [0, E) with pre[e] <= u (pre non-decreasing, pre[0] = 0).
__device__ __forceinline__ int find_group(const int* pre, int E, int u) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= u)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

}  // namespace gnf4
